// swin_window_attn_fwd_noalloc: the forward pass for callers that cannot
// allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocator) around this call: a
// runtime that owns every device byte through its own pool, code running
// inside stream capture where allocation is not allowed, or an embedding that
// forbids allocation after start-up.  The regular entry point asks them for a
// workspace when the cosine mode has to evaluate the Log-CPB meta network; this
// one keeps that bias table in a fixed device array of this library instead.
//
// The array (kNoallocTableFloats floats = 512 KiB) is a file-scope __device__
// variable: every GPU that loads the library holds it until the process exits,
// and every call on a device shares it.  Calls whose kernels overlap on the
// GPU (different streams, or different host threads) race on it and must be
// serialised by the caller.  The CPB kernel overwrites every table entry it
// uses on each call, so nothing has to start at zero; the array keeps the last
// call's table afterwards.
//
// Host code may not use the array's name as a device address (it is a host
// stand-in).  The first call on each device looks the address up with
// cudaGetSymbolAddress while that device is current; make that first call
// before any stream capture.  The address is cached per device ordinal for the
// life of the process, so the library must not be used across a
// cudaDeviceReset (which unloads the module and invalidates it).  No
// cudaMalloc, cudaFree or allocating library routine is called here, and an
// argument error returns before anything is enqueued.
#include <mutex>

#include "swin_common.cuh"

namespace swin {
namespace {

// (2M-1)^2 * heads floats: enough for M = 32 with 32 heads (508 KiB).
constexpr size_t kNoallocTableFloats = 131072;

static __device__ __align__(256) float g_noalloc_table[kNoallocTableFloats];

constexpr int kMaxDev = 64;
float* g_noalloc_ptr[kMaxDev] = {};
std::mutex g_noalloc_mu;

// Device address of g_noalloc_table on the current device (looked up once).
swin_status noalloc_table(float** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(SWIN_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDev) return fail(SWIN_ERR_UNSUPPORTED, "device ordinal %d above %d", dev, kMaxDev - 1);
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_table);
    if (e != cudaSuccess)
      return fail(SWIN_ERR_CUDA, "cudaGetSymbolAddress(no-alloc table): %s", cudaGetErrorString(e));
    g_noalloc_ptr[dev] = static_cast<float*>(p);
  }
  *out = g_noalloc_ptr[dev];
  return SWIN_OK;
}

}  // namespace
}  // namespace swin

extern "C" swin_status swin_window_attn_fwd_noalloc(
    const void* q, const void* k, const void* v, void* out, swin_dtype dt, swin_dtype out_dt, int B,
    int H, int W, int heads, int d, int M, int shift, swin_mode mode, const float* tau,
    const float* bias_table, const swin_cpb_weights* cpb, const float* rope_freqs,
    swin_stream_t stream) {
  // every argument check first, so that a rejected call launches nothing and
  // leaves the shared table as it was
  swin_status st = swin::check_fwd_args(q, k, v, out, dt, out_dt, B, H, W, heads, d, M, shift, mode, tau,
                                        bias_table, cpb, rope_freqs);
  if (st != SWIN_OK) return st;
  const bool needs_table = mode == SWIN_MODE_COSINE_CPB && !bias_table && cpb;
  if (!needs_table)
    return swin_window_attn_fwd(q, k, v, out, dt, out_dt, B, H, W, heads, d, M, shift, mode, tau,
                                bias_table, cpb, rope_freqs, nullptr, 0, stream);
  const size_t need = (size_t)(2 * M - 1) * (2 * M - 1) * heads;
  if (need > swin::kNoallocTableFloats)
    return swin::fail(SWIN_ERR_UNSUPPORTED,
                      "no-alloc entry point: (2M-1)^2*heads = %zu floats exceeds its fixed table of "
                      "%zu floats; use swin_window_attn_fwd with a workspace",
                      need, swin::kNoallocTableFloats);
  float* table = nullptr;
  st = swin::noalloc_table(&table);
  if (st != SWIN_OK) return st;
  st = swin::launch_cpb_eval(M, heads, *cpb, table, reinterpret_cast<cudaStream_t>(stream));
  if (st != SWIN_OK) return st;
  return swin_window_attn_fwd(q, k, v, out, dt, out_dt, B, H, W, heads, d, M, shift, mode, tau, table,
                              nullptr, rope_freqs, nullptr, 0, stream);
}
