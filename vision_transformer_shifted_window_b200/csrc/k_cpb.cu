// Log-CPB meta network evaluation ("Swin Transformer V2" wiki card, Method
// §3.3, eq. 3 and eq. 4; continuous_bias pseudocode).  For every offset of an
// MxM window it maps (dx, dy) to (sign(dx) ln(1+|dx|), sign(dy) ln(1+|dy|)),
// runs the two-layer ReLU MLP G and writes one bias per head.  The page's
// "Paper vs code" notes give the released code's form, also built: offsets
// scaled by 8 / (Mp - 1) and mapped by sign(d) log2(1+|d|) / log2(8), and the
// output bounded as 16 sigmoid(G).  §3.3 notes
// that the biases can be computed once and stored for inference: this kernel
// is that precompute; the attention kernels then read the table.
//
// One CTA per offset row: the hidden layer (hidden <= 4096 fp32) goes to shared
// memory, then one warp per head reduces w2[h] . hidden with shuffles.
// Work is (2M-1)^2 * hidden * (2 + heads) FMAs: negligible next to attention.
#include "swin_common.cuh"

namespace swin {
namespace {

__device__ __forceinline__ float log_map(int delta) {
  float a = log1pf((float)(delta < 0 ? -delta : delta));
  return delta < 0 ? -a : a;
}

// The code form: d' = d * scale (scale = 8 / (Mp - 1), or 0 for Mp = 1),
// sign(d') log2(1 + |d'|) / 3.
__device__ __forceinline__ float log2_map(int delta, float scale) {
  const float a = log2f(1.0f + fabsf((float)delta) * scale) / 3.0f;
  return delta < 0 ? -a : a;
}

__global__ void __launch_bounds__(256) cpb_eval_kernel(int M, int heads, int hidden, int form, float scale,
                                                       const float* __restrict__ w1,
                                                       const float* __restrict__ b1,
                                                       const float* __restrict__ w2,
                                                       const float* __restrict__ b2,
                                                       float* __restrict__ table) {
  extern __shared__ float hid[];
  const int R = 2 * M - 1;
  const int row = blockIdx.x;
  const int dy = row / R - (M - 1), dx = row % R - (M - 1);
  const float in_x = form == SWIN_CPB_CODE ? log2_map(dx, scale) : log_map(dx);
  const float in_y = form == SWIN_CPB_CODE ? log2_map(dy, scale) : log_map(dy);
  for (int j = threadIdx.x; j < hidden; j += blockDim.x) {
    float a = fmaf(w1[2 * j + 0], in_x, fmaf(w1[2 * j + 1], in_y, b1 ? b1[j] : 0.0f));
    hid[j] = a > 0.0f ? a : 0.0f;
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarp = blockDim.x >> 5;
  for (int h = warp; h < heads; h += nwarp) {
    const float* wr = w2 + (size_t)h * hidden;
    float acc = 0.0f;
    for (int j = lane; j < hidden; j += 32) acc = fmaf(wr[j], hid[j], acc);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) {
      const float z = acc + (b2 ? b2[h] : 0.0f);
      table[(size_t)row * heads + h] = form == SWIN_CPB_CODE ? 16.0f / (1.0f + expf(-z)) : z;
    }
  }
}

}  // namespace

swin_status launch_cpb_eval(int M, int heads, const swin_cpb_weights& g, float* table,
                            cudaStream_t stream, int form, int pretrained_M) {
  const int R = 2 * M - 1;
  const int mp = pretrained_M > 0 ? pretrained_M : M;
  const float scale = mp > 1 ? 8.0f / (float)(mp - 1) : 0.0f;
  size_t smem = sizeof(float) * (size_t)g.hidden;
  cpb_eval_kernel<<<R * R, 256, smem, stream>>>(M, heads, g.hidden, form, scale, g.w1, g.b1, g.w2, g.b2,
                                                table);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(SWIN_ERR_CUDA, "cpb_eval launch: %s", cudaGetErrorString(e));
  return SWIN_OK;
}

}  // namespace swin
