// Shifted-window attention on the CUDA cores, for fp32 tensors (and for bf16
// tensors the tensor-core path does not cover: d != 32, a bias table with
// M > 32, interleaved windows).  Inputs and outputs keep their dtype.  For
// fp32 tensors the arithmetic inside is double precision — normalisation or
// rotation of q and k, logits, the exponentials and the running sums — so
// that the fp32 result stays within 1e-5 of the exact one (max error over the
// output's RMS) even for the sharpest softmax the pages' settings give
// (tau = 0.05, i.e. logits scaled by 20): in fp32, the logit roundings and the
// running-sum roundings each came to a few 1e-6 on a 16 x 16 window.  For bf16
// tensors (a 2e-2 bound) it is fp32.
//
// Scores follow "Swin Transformer V2" eq. 1 (mode 0) and eq. 2 (mode 1, tau
// clamped at 0.01, §3.2), or FlashSwin's window-local 2-D RoPE (mode 2); the
// softmax is the exact online form FlashSwin relies on: a running maximum and
// rescaled running sums, so no score row is stored.
//
// Decomposition: one CTA per (image, head, rectangle, block of queries), of
// 128 threads, or 64 when a window has at most 64 tokens (M <= 8); a
// rectangle is one window per axis, a segment of the shifted partition or a
// strided window of the interleaved one (see swin_index.cuh), i.e. one
// independent attention problem of up to M*M tokens.  Each thread owns one
// query row; keys and values stream through shared memory 16 at a time
// (normalised or rotated once per key), and every thread reads them as
// broadcasts; each logit is four independent FMA chains.
#include "swin_common.cuh"

namespace swin {
namespace {

constexpr int kThreads = 128;  // threads per CTA (64 when a window has at most 64 tokens)
constexpr int kKeyTile = 16;
constexpr int kMaxM = 64;

template <typename T>
__device__ __forceinline__ float load_elem(const T* p);
template <>
__device__ __forceinline__ float load_elem<float>(const float* p) {
  return __ldg(p);
}
template <>
__device__ __forceinline__ float load_elem<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}
template <typename T>
__device__ __forceinline__ T store_conv(double x);
template <>
__device__ __forceinline__ float store_conv<float>(double x) {
  return (float)x;
}
template <>
__device__ __forceinline__ __nv_bfloat16 store_conv<__nv_bfloat16>(double x) {
  // round once, from the fp32 result: a bf16 output is the fp32 output rounded
  return __float2bfloat16_rn((float)x);
}

__device__ __forceinline__ double a_exp(double x) { return exp(x); }
__device__ __forceinline__ float a_exp(float x) { return expf(x); }

// Rotate channel pairs of one half (row or column axis) by position p.
template <typename A, int D>
__device__ __forceinline__ void rope_rotate(A* x, int half, int p, const A* cs, const A* sn) {
  constexpr int Q = D / 4;
#pragma unroll
  for (int t = 0; t < Q; ++t) {
    const A c = cs[p * Q + t], s = sn[p * Q + t];
    const A a = x[half * (D / 2) + 2 * t], b = x[half * (D / 2) + 2 * t + 1];
    x[half * (D / 2) + 2 * t] = a * c - b * s;
    x[half * (D / 2) + 2 * t + 1] = a * s + b * c;
  }
}

template <typename T, typename TO, typename A, int D, int MODE>
__global__ void __launch_bounds__(kThreads) attn_simt_kernel(AttnArgs a, int nsx, int chunks) {
  __shared__ A ks[kKeyTile][D];
  __shared__ float vs[kKeyTile][D];  // V entries are fp32 or bf16 values: exact in fp32
  // RoPE tables: [axis][p][t] for p < M, t < D/4
  __shared__ A rcos[(MODE == 2) ? 2 * kMaxM * (D / 4) : 1];
  __shared__ A rsin[(MODE == 2) ? 2 * kMaxM * (D / 4) : 1];

  const int M = a.M, s = a.shift;
  const int rect = blockIdx.x / chunks, chunk = blockIdx.x % chunks;
  const int sy = rect / nsx, sx = rect % nsx;
  const int h = blockIdx.y, b = blockIdx.z;
  const SwinAxis ay = swin_axis(a.part, sy, a.H, M, s), ax = swin_axis(a.part, sx, a.W, M, s);
  const int ly = ay.len, lx = ax.len;
  const int n = ly * lx;
  const int nt = blockDim.x;
  if (chunk * nt >= n) return;  // whole CTA idle (uniform)
  const int C = a.heads * D;
  const T* Q = static_cast<const T*>(a.q);
  const T* K = static_cast<const T*>(a.k);
  const T* V = static_cast<const T*>(a.v);
  TO* O = static_cast<TO*>(a.out);

  if (MODE == 2) {
    constexpr int Qd = D / 4;
    for (int i = threadIdx.x; i < 2 * M * Qd; i += nt) {
      const int axis = i / (M * Qd), p = (i / Qd) % M, t = i % Qd;
      double sv, cv;
      sincos((double)p * (double)a.rope[axis * Qd + t], &sv, &cv);
      rcos[axis * kMaxM * Qd + p * Qd + t] = (A)cv;
      rsin[axis * kMaxM * Qd + p * Qd + t] = (A)sv;
    }
    __syncthreads();
  }

  const int qi = chunk * nt + threadIdx.x;
  const bool active = qi < n;
  const int iyq = active ? qi / lx : 0, ixq = active ? qi % lx : 0;
  const int yq = ay.start + ay.stride * iyq, xq = ax.start + ax.stride * ixq;
  A q[D], o[D];
  {
    const T* src = Q + (((size_t)b * a.H + yq) * a.W + xq) * C + (size_t)h * D;
#pragma unroll
    for (int e = 0; e < D; ++e) q[e] = active ? (A)load_elem(src + e) : (A)0;
  }
  // logit = (q . k) * scale (+ bias): mode 1 scale = 1 / (|q| max(tau, 0.01)),
  // k unit-normalised; modes 0 and 2 scale = 1 / sqrt(d)
  A scale = (A)(1.0 / sqrt((double)D));
  if (MODE == 1) {
    A ss = 0;
#pragma unroll
    for (int e = 0; e < D; ++e) ss = fma(q[e], q[e], ss);
    scale = (A)1 / (fmax(sqrt(ss), (A)kNormEps) * fmax((A)__ldg(a.tau + h), (A)kTauMin));
  }
  if (MODE == 2) {
    rope_rotate<A, D>(q, 0, ay.base + iyq, rcos, rsin);
    rope_rotate<A, D>(q, 1, ax.base + ixq, rcos + kMaxM * (D / 4), rsin + kMaxM * (D / 4));
  }
#pragma unroll
  for (int e = 0; e < D; ++e) o[e] = 0;
  A m = -INFINITY, l = 0;

  for (int j0 = 0; j0 < n; j0 += kKeyTile) {
    const int nk = min(kKeyTile, n - j0);
    __syncthreads();
    for (int i = threadIdx.x; i < nk * D; i += nt) {
      const int j = i / D, e = i % D, kk = j0 + j;
      const int yk = ay.start + ay.stride * (kk / lx), xk = ax.start + ax.stride * (kk % lx);
      const size_t off = (((size_t)b * a.H + yk) * a.W + xk) * C + (size_t)h * D + e;
      SWIN_DCHECK(a.status, yk >= 0 && yk < a.H && xk >= 0 && xk < a.W && off < (size_t)a.B * a.H * a.W * C);
      ks[j][e] = (A)load_elem(K + off);
      vs[j][e] = load_elem(V + off);
    }
    __syncthreads();
    if (MODE != 0 && threadIdx.x < nk) {
      A* kr = ks[threadIdx.x];
      if (MODE == 1) {
        A ss = 0;
        for (int e = 0; e < D; ++e) ss = fma(kr[e], kr[e], ss);
        const A inv = (A)1 / fmax(sqrt(ss), (A)kNormEps);
        for (int e = 0; e < D; ++e) kr[e] *= inv;
      } else {
        const int kk = j0 + threadIdx.x;
        A tmp[D];
        for (int e = 0; e < D; ++e) tmp[e] = kr[e];
        rope_rotate<A, D>(tmp, 0, ay.base + kk / lx, rcos, rsin);
        rope_rotate<A, D>(tmp, 1, ax.base + kk % lx, rcos + kMaxM * (D / 4),
                       rsin + kMaxM * (D / 4));
        for (int e = 0; e < D; ++e) kr[e] = tmp[e];
      }
    }
    __syncthreads();
    if (!active) continue;
    for (int j = 0; j < nk; ++j) {
      // four partial sums: independent FMA chains
      A d0 = 0, d1 = 0, d2 = 0, d3 = 0;
#pragma unroll
      for (int e = 0; e < D; e += 4) {
        d0 = fma(q[e], ks[j][e], d0);
        d1 = fma(q[e + 1], ks[j][e + 1], d1);
        d2 = fma(q[e + 2], ks[j][e + 2], d2);
        d3 = fma(q[e + 3], ks[j][e + 3], d3);
      }
      A lg = ((d0 + d1) + (d2 + d3)) * scale;
      if (MODE != 2 && a.table) {
        const int kk = j0 + j;
        const int r = swin_rel_row(iyq - kk / lx, ixq - kk % lx, M);
        lg += (A)__ldg(a.table + (size_t)r * a.heads + h);
      }
      if (lg > m) {
        const A c = a_exp(m - lg);
        l = fma(l, c, (A)1);
#pragma unroll
        for (int e = 0; e < D; ++e) o[e] = fma(o[e], c, (A)vs[j][e]);
        m = lg;
      } else {
        const A p = a_exp(lg - m);
        l += p;
#pragma unroll
        for (int e = 0; e < D; ++e) o[e] = fma(p, (A)vs[j][e], o[e]);
      }
    }
  }
  if (active) {
    const A inv = (A)1 / l;
    SWIN_DCHECK(a.status, yq >= 0 && yq < a.H && xq >= 0 && xq < a.W);
    TO* dst = O + (((size_t)b * a.H + yq) * a.W + xq) * C + (size_t)h * D;
#pragma unroll
    for (int e = 0; e < D; ++e) dst[e] = store_conv<TO>((double)(o[e] * inv));
  }
}

template <typename T, typename TO, typename A, int D>
swin_status launch_typed(const AttnArgs& a, cudaStream_t stream) {
  const int nsy = swin_nwin(a.part, a.H, a.M, a.shift), nsx = swin_nwin(a.part, a.W, a.M, a.shift);
  const int nt = a.M * a.M <= 64 ? 64 : kThreads;
  const int chunks = (a.M * a.M + nt - 1) / nt;
  dim3 grid(nsy * nsx * chunks, a.heads, a.B);
  switch (a.mode) {
    case 0: attn_simt_kernel<T, TO, A, D, 0><<<grid, nt, 0, stream>>>(a, nsx, chunks); break;
    case 1: attn_simt_kernel<T, TO, A, D, 1><<<grid, nt, 0, stream>>>(a, nsx, chunks); break;
    default:
      if constexpr (D % 4 == 0) attn_simt_kernel<T, TO, A, D, 2><<<grid, nt, 0, stream>>>(a, nsx, chunks);
      break;
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(SWIN_ERR_CUDA, "attn_simt launch: %s", cudaGetErrorString(e));
  return SWIN_OK;
}

template <typename T, typename TO, typename A>
swin_status launch_d(const AttnArgs& a, cudaStream_t stream) {
  switch (a.d) {
    case 8: return launch_typed<T, TO, A, 8>(a, stream);
    case 16: return launch_typed<T, TO, A, 16>(a, stream);
    case 32: return launch_typed<T, TO, A, 32>(a, stream);
    case 64: return launch_typed<T, TO, A, 64>(a, stream);
    default: return fail(SWIN_ERR_UNSUPPORTED, "CUDA-core path supports d in {8,16,32,64}, got %d", a.d);
  }
}

}  // namespace

swin_status launch_attn_simt(const AttnArgs& a, bool bf16_in, bool f32_out, cudaStream_t stream) {
  if (a.M > kMaxM) return fail(SWIN_ERR_UNSUPPORTED, "M=%d above %d", a.M, kMaxM);
  if (!bf16_in) return launch_d<float, float, double>(a, stream);
  return f32_out ? launch_d<__nv_bfloat16, float, float>(a, stream)
                 : launch_d<__nv_bfloat16, __nv_bfloat16, float>(a, stream);
}

}  // namespace swin
