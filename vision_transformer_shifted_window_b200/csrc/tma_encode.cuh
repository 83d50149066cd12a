// The driver's tensor-map encoder (cuTensorMapEncodeTiled), looked up once
// through the runtime's entry-point query; shared by the kernels that build
// TMA descriptors.
#pragma once

#include <cuda.h>

namespace swin {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// nullptr when the driver does not provide it.
EncodeTiledFn tma_encode_fn();

}  // namespace swin
