// The steps either side of the window attention in a Swin V2 block
// ("Swin Transformer V2" wiki card, Method item 1 "Residual post-norm", §3.2,
// fig. 1, and the swin_v2_block pseudocode): the projection of the block's
// input into q, k and v, and after the attention the output projection, whose
// result is layer-normalised before it joins the residual path:
//   q | k | v = x W_qkv^T + b_qkv
//   out       = x + LN(a W_o^T + b_o) * gamma + beta
// bf16 inputs with C = heads * d a multiple of 32 up to 128 (96 for the qkv
// projection, whose weights must stay in shared memory) take the fused
// tensor-core kernels of k_block_tc.cu.  Otherwise the projections are plain
// GEMMs (cuBLASLt, fp32 accumulation, no cuBLAS workspace) whose fp32 results
// land in the caller's workspace, and the bias, the post-norm and the
// residual add are this file's kernels.  Either way the arithmetic after the
// products is fp32 and each output element is rounded once (a bf16 output is
// the fp32 one rounded to nearest even).
#include <cublasLt.h>

#include <map>
#include <mutex>
#include <tuple>

#include "swin_common.cuh"

namespace swin {
namespace {

std::mutex g_lt_mu;
constexpr int kMaxDevices = 64;
cublasLtHandle_t g_lt[kMaxDevices] = {};  // one per device ordinal

// (device, dtype, m, n, k) -> heuristic algorithm; a GEMM shape is planned
// once per device.
std::map<std::tuple<int, int, int, int, int>, cublasLtMatmulAlgo_t> g_algos;

swin_status lt_fail(const char* what, cublasStatus_t st) {
  return fail(SWIN_ERR_CUDA, "cuBLASLt %s failed (status %d)", what, (int)st);
}

// Y[rows][n] = X[rows][k] W[n][k]^T (row-major, dense), fp32 accumulation;
// X and W fp32 or bf16, Y fp32.
swin_status gemm_xwt(const void* X, const void* Wt, float* Y, bool bf16, int rows, int n, int k,
                     cudaStream_t stream) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return fail(SWIN_ERR_CUDA, "could not resolve the current device");
  std::lock_guard<std::mutex> lock(g_lt_mu);
  cublasStatus_t st;
  if (!g_lt[dev]) {
    st = cublasLtCreate(&g_lt[dev]);
    if (st != CUBLAS_STATUS_SUCCESS) return lt_fail("create", st);
  }
  cublasLtHandle_t lt = g_lt[dev];
  const cudaDataType_t t = bf16 ? CUDA_R_16BF : CUDA_R_32F, to = CUDA_R_32F;
  // Column-major view: Y^T (n x rows) = W (n x k) . X^T (k x rows), where the
  // row-major W buffer is W^T in column-major (k x n), hence op(A) = T.
  cublasLtMatmulDesc_t op = nullptr;
  cublasLtMatrixLayout_t la = nullptr, lb = nullptr, lc = nullptr;
  swin_status ret = SWIN_OK;
  const cublasOperation_t ta = CUBLAS_OP_T, tb = CUBLAS_OP_N;
  const float one = 1.0f, zero = 0.0f;
  do {
    if ((st = cublasLtMatmulDescCreate(&op, CUBLAS_COMPUTE_32F, CUDA_R_32F)) != CUBLAS_STATUS_SUCCESS) {
      ret = lt_fail("descriptor", st);
      break;
    }
    cublasLtMatmulDescSetAttribute(op, CUBLASLT_MATMUL_DESC_TRANSA, &ta, sizeof(ta));
    cublasLtMatmulDescSetAttribute(op, CUBLASLT_MATMUL_DESC_TRANSB, &tb, sizeof(tb));
    if ((st = cublasLtMatrixLayoutCreate(&la, t, k, n, k)) != CUBLAS_STATUS_SUCCESS ||
        (st = cublasLtMatrixLayoutCreate(&lb, t, k, rows, k)) != CUBLAS_STATUS_SUCCESS ||
        (st = cublasLtMatrixLayoutCreate(&lc, to, n, rows, n)) != CUBLAS_STATUS_SUCCESS) {
      ret = lt_fail("layout", st);
      break;
    }
    const auto key = std::make_tuple(dev, (int)bf16, n, rows, k);
    auto it = g_algos.find(key);
    if (it == g_algos.end()) {
      cublasLtMatmulPreference_t pref = nullptr;
      size_t zero_ws = 0;
      cublasLtMatmulPreferenceCreate(&pref);
      cublasLtMatmulPreferenceSetAttribute(pref, CUBLASLT_MATMUL_PREF_MAX_WORKSPACE_BYTES, &zero_ws,
                                           sizeof(zero_ws));
      cublasLtMatmulHeuristicResult_t res;
      int found = 0;
      st = cublasLtMatmulAlgoGetHeuristic(lt, op, la, lb, lc, lc, pref, 1, &res, &found);
      cublasLtMatmulPreferenceDestroy(pref);
      if (st != CUBLAS_STATUS_SUCCESS || found < 1) {
        ret = fail(SWIN_ERR_UNSUPPORTED, "cuBLASLt has no algorithm for a %d x %d x %d GEMM", rows, n, k);
        break;
      }
      it = g_algos.emplace(key, res.algo).first;
    }
    st = cublasLtMatmul(lt, op, &one, Wt, la, X, lb, &zero, Y, lc, Y, lc, &it->second, nullptr, 0, stream);
    if (st != CUBLAS_STATUS_SUCCESS) ret = lt_fail("matmul", st);
  } while (false);
  if (lc) cublasLtMatrixLayoutDestroy(lc);
  if (lb) cublasLtMatrixLayoutDestroy(lb);
  if (la) cublasLtMatrixLayoutDestroy(la);
  if (op) cublasLtMatmulDescDestroy(op);
  return ret;
}

template <typename T>
__device__ __forceinline__ float to_f(T x);
template <>
__device__ __forceinline__ float to_f<float>(float x) {
  return x;
}
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}
template <typename T>
__device__ __forceinline__ T from_f(float x);
template <>
__device__ __forceinline__ float from_f<float>(float x) {
  return x;
}
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Four consecutive values of T from fp32, rounded once each.
__device__ __forceinline__ void store4(float* dst, float4 v) { *reinterpret_cast<float4*>(dst) = v; }
__device__ __forceinline__ void store4(__nv_bfloat16* dst, float4 v) {
  __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y), hi = __floats2bfloat162_rn(v.z, v.w);
  uint2 w;
  w.x = *reinterpret_cast<uint32_t*>(&lo);
  w.y = *reinterpret_cast<uint32_t*>(&hi);
  *reinterpret_cast<uint2*>(dst) = w;
}

// q, k, v = the fp32 product y [tokens][3C] plus b (NULL: 0), split by
// channel thirds and rounded once to T; each thread takes four consecutive
// channels (C % 8 == 0: every 16-byte load and store is aligned), grid-stride
// over tokens x C / 4.
template <typename T>
__global__ void bias_split_kernel(const float* __restrict__ y, const float* b, T* q, T* k, T* v, long long n,
                                  int C) {
  const long long n4 = n / 4;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n4;
       i += (long long)gridDim.x * blockDim.x) {
    const long long e = 4 * i, t = e / C;
    const int c = (int)(e - t * C);
    const float* yr = y + t * 3 * C + c;
    T* outs[3] = {q + e, k + e, v + e};
#pragma unroll
    for (int part = 0; part < 3; ++part) {
      float4 val = *reinterpret_cast<const float4*>(yr + part * C);
      if (b) {
        const float* bb = b + part * C + c;
        val.x += __ldg(bb);
        val.y += __ldg(bb + 1);
        val.z += __ldg(bb + 2);
        val.w += __ldg(bb + 3);
      }
      store4(outs[part], val);
    }
  }
}

// out[t] = x[t] + gamma * (y[t] + b - mean) / sqrt(var + eps) + beta, one warp
// per token row; y is the fp32 projection.  Mean and variance are two passes
// over the row held in registers (fp32): kPer values per lane, the row's C
// channels rounded up to a multiple of 32, so a narrow row keeps few
// registers and many warps resident (C <= kMaxC).
constexpr int kMaxC = 1024;

// kTok tokens per warp at a time, all their loads issued before the first
// reduction (kTok x kPer values per lane in flight).
template <typename T, typename TO, int kPer, int kTok>
__global__ void __launch_bounds__(256) postnorm_residual_kernel(const T* __restrict__ x,
                                                                const float* __restrict__ yall, TO* out,
                                                                const float* b, const float* gamma, const float* beta,
                                                                float eps, long long tokens, int C) {
  const int lane = threadIdx.x & 31;
  const long long warp = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5;
  const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;
  for (long long t0 = warp * kTok; t0 < tokens; t0 += nwarps * kTok) {
    float y[kTok][kPer], xv[kTok][kPer];
#pragma unroll
    for (int u = 0; u < kTok; ++u)
#pragma unroll
      for (int j = 0; j < kPer; ++j) {
        const int c = lane + 32 * j;
        const bool ok = c < C && t0 + u < tokens;
        y[u][j] = ok ? yall[(t0 + u) * C + c] + (b ? __ldg(b + c) : 0.f) : 0.f;
        xv[u][j] = ok ? to_f(x[(t0 + u) * C + c]) : 0.f;
      }
    float mean[kTok], rstd[kTok];
#pragma unroll
    for (int u = 0; u < kTok; ++u) {
      float s = 0.f;
#pragma unroll
      for (int j = 0; j < kPer; ++j) s += y[u][j];  // padding lanes hold 0
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      mean[u] = s / (float)C;
      float ss = 0.f;
#pragma unroll
      for (int j = 0; j < kPer; ++j)
        if (lane + 32 * j < C) ss += (y[u][j] - mean[u]) * (y[u][j] - mean[u]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      rstd[u] = rsqrtf(ss / (float)C + eps);
    }
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int c = lane + 32 * j;
      if (c >= C) continue;
      const float g = gamma ? __ldg(gamma + c) : 1.f, be = beta ? __ldg(beta + c) : 0.f;
#pragma unroll
      for (int u = 0; u < kTok; ++u)
        if (t0 + u < tokens) out[(t0 + u) * C + c] = from_f<TO>(xv[u][j] + (y[u][j] - mean[u]) * rstd[u] * g + be);
    }
  }
}

int grid_for(long long work, int per_block) {
  long long g = (work + per_block - 1) / per_block;
  return (int)(g < 148 * 16 ? (g < 1 ? 1 : g) : 148 * 16);
}

template <int kPer>
void launch_postnorm(const void* x, const float* y, void* out, const float* b_o, const float* gamma,
                     const float* beta, float eps, bool bf16, bool f32_out, int tokens, int C, cudaStream_t stream) {
  using bf = __nv_bfloat16;
  // one token per warp: batching 2-4 tokens per warp measured slower (fewer
  // warps in flight); 8 warps per block, every token in one wave
  constexpr int kTok = 1;
  const int blocks = (int)(((long long)tokens + 8 * kTok - 1) / (8 * kTok));
  if (bf16 && !f32_out)
    postnorm_residual_kernel<bf, bf, kPer, kTok><<<blocks, 256, 0, stream>>>(
        static_cast<const bf*>(x), y, static_cast<bf*>(out), b_o, gamma, beta, eps, tokens, C);
  else if (bf16)
    postnorm_residual_kernel<bf, float, kPer, kTok><<<blocks, 256, 0, stream>>>(
        static_cast<const bf*>(x), y, static_cast<float*>(out), b_o, gamma, beta, eps, tokens, C);
  else
    postnorm_residual_kernel<float, float, kPer, kTok><<<blocks, 256, 0, stream>>>(
        static_cast<const float*>(x), y, static_cast<float*>(out), b_o, gamma, beta, eps, tokens, C);
}

}  // namespace

swin_status launch_qkv_proj(const void* x, const void* w_qkv, const float* b_qkv, void* q, void* k, void* v,
                            bool bf16, bool f32_out, int tokens, int C, float* y, cudaStream_t stream) {
  if (block_tc_supported(C, bf16, false)) return launch_qkv_proj_tc(x, w_qkv, b_qkv, q, k, v, f32_out, tokens, C, stream);
  swin_status s = gemm_xwt(x, w_qkv, y, bf16, tokens, 3 * C, C, stream);
  if (s != SWIN_OK) return s;
  const long long n = (long long)tokens * C;
  if (bf16 && !f32_out)
    bias_split_kernel<__nv_bfloat16><<<grid_for(n / 4, 256), 256, 0, stream>>>(
        y, b_qkv, static_cast<__nv_bfloat16*>(q), static_cast<__nv_bfloat16*>(k), static_cast<__nv_bfloat16*>(v), n,
        C);
  else
    bias_split_kernel<float><<<grid_for(n / 4, 256), 256, 0, stream>>>(
        y, b_qkv, static_cast<float*>(q), static_cast<float*>(k), static_cast<float*>(v), n, C);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(SWIN_ERR_CUDA, "bias launch: %s", cudaGetErrorString(e));
  return SWIN_OK;
}

swin_status launch_proj_postnorm(const void* a, const void* w_o, const float* b_o, const void* x,
                                 const float* gamma, const float* beta, float eps, void* out, bool bf16, bool f32_out,
                                 int tokens, int C, float* y, cudaStream_t stream) {
  if (C > kMaxC) return fail(SWIN_ERR_UNSUPPORTED, "post-norm supports C <= %d, got %d", kMaxC, C);
  if (block_tc_supported(C, bf16, true))
    return launch_proj_postnorm_tc(a, w_o, b_o, x, gamma, beta, eps, out, f32_out, tokens, C, stream);
  swin_status s = gemm_xwt(a, w_o, y, bf16, tokens, C, C, stream);
  if (s != SWIN_OK) return s;
  const int per = (C + 31) / 32;
  switch (per <= 2 ? 2 : per <= 3 ? 3 : per <= 4 ? 4 : per <= 8 ? 8 : per <= 16 ? 16 : 32) {
    case 2: launch_postnorm<2>(x, y, out, b_o, gamma, beta, eps, bf16, f32_out, tokens, C, stream); break;
    case 3: launch_postnorm<3>(x, y, out, b_o, gamma, beta, eps, bf16, f32_out, tokens, C, stream); break;
    case 4: launch_postnorm<4>(x, y, out, b_o, gamma, beta, eps, bf16, f32_out, tokens, C, stream); break;
    case 8: launch_postnorm<8>(x, y, out, b_o, gamma, beta, eps, bf16, f32_out, tokens, C, stream); break;
    case 16: launch_postnorm<16>(x, y, out, b_o, gamma, beta, eps, bf16, f32_out, tokens, C, stream); break;
    default: launch_postnorm<32>(x, y, out, b_o, gamma, beta, eps, bf16, f32_out, tokens, C, stream); break;
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(SWIN_ERR_CUDA, "post-norm launch: %s", cudaGetErrorString(e));
  return SWIN_OK;
}

}  // namespace swin
