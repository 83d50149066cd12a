// Writes the kernels' view of Swin's bookkeeping (rolled-frame window, band and
// local index per token; relative-position row per window pair) so that tests
// can compare it bit for bit with an independent enumeration.
#include "swin_common.cuh"

namespace swin {
namespace {

__global__ void token_tables_kernel(int H, int W, int M, int s, int32_t* tw, int32_t* tr,
                                    int32_t* tl) {
  int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= H * W) return;
  SwinRolled r = swin_rolled(t / W, t % W, H, W, M, s);
  if (tw) tw[t] = r.window;
  if (tr) tr[t] = r.band;
  if (tl) tl[t] = r.local;
}

__global__ void rel_index_kernel(int M, int32_t* ri) {
  int N = M * M;
  int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= N * N) return;
  int i = t / N, j = t % N;
  ri[t] = swin_rel_row(i / M - j / M, i % M - j % M, M);
}

}  // namespace

swin_status launch_index_tables(int H, int W, int M, int shift, int32_t* tw, int32_t* tr,
                                int32_t* tl, int32_t* ri, cudaStream_t stream) {
  if (tw || tr || tl) {
    int n = H * W;
    token_tables_kernel<<<(n + 255) / 256, 256, 0, stream>>>(H, W, M, shift, tw, tr, tl);
  }
  if (ri) {
    int n = M * M * M * M;
    rel_index_kernel<<<(n + 255) / 256, 256, 0, stream>>>(M, ri);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess)
    return fail(SWIN_ERR_CUDA, "index_tables launch: %s", cudaGetErrorString(e));
  return SWIN_OK;
}

}  // namespace swin
