// Gradients of shifted-window attention on the CUDA cores: dq, dk, dv, and
// the parameter gradients d(bias table), d(tau) and d(RoPE frequencies).
//
// With L = sum(dout . out), P_ij the softmax weights of query i over its key
// set and g_i = dout_i, the chain rule through the forward definition
// ("Swin Transformer V2" eq. 1 and eq. 2 with tau clamped at 0.01, §3.2;
// FlashSwin's window-local 2-D RoPE) gives
//   dv_j  = sum_i P_ij g_i
//   dl_ij = P_ij (g_i . v_j - D_i),   D_i = sum_j P_ij (g_i . v_j) = g_i . o_i
// and dl flows into the score.  Every mode is written as a dot product of
// transformed vectors plus a bias, l_ij = qt_i . kt_j + T[r]:
//   mode 0  qt = q / sqrt(d)          kt = k
//   mode 1  qt = q / (|q| t)          kt = k / |k|       (t = max(tau, 0.01))
//   mode 2  qt = R(p_i) q / sqrt(d)   kt = R(p_j) k
// so dqt_i = sum_j dl_ij kt_j and dkt_j = sum_i dl_ij qt_i, mapped back to q
// and k by each transform's Jacobian (the normalisation's projection, the
// rotation's transpose); dT[r] = sum of dl over the pairs at offset r;
// dtau = -(1/t) sum_i qt_i . dqt_i where tau >= 0.01 (below, the clamp is a
// constant); domega_t = sum over queries and keys of p * (dxt . J xt) on the
// channel pair that omega_t rotates, J the quarter turn.
//
// Nothing is kept from the forward pass: the softmax statistics are
// recomputed.  Three launches, all on the caller's stream:
//   1. bwd_q: one thread per query row (the forward's decomposition: one CTA
//      of 128 threads, 64 for windows of <= 64 tokens, per image, head,
//      rectangle and block of queries).
//      Pass 1 recomputes the row's log-sum-exp and D_i = g_i . o_i by an online
//      softmax over the rectangle's keys, and stores both; pass 2 forms dl,
//      accumulates dqt in registers and the bias gradient in shared memory
//      (in double).
//   2. bwd_kv: one thread per key row; queries stream through shared memory
//      with their stored statistics; accumulates dkt and dv in registers.
//   3. bwd_finish: converts the double accumulators of the parameter
//      gradients to the caller's fp32 arrays.
// Arithmetic type: double for fp32 tensors (the 1e-5 bound on gradients,
// which subtract nearly equal terms in dl), float for bf16 tensors.
#include "swin_common.cuh"

namespace swin {
namespace {

constexpr int kThreads = 128;
constexpr int kMaxM = 64;

// Rows per shared-memory tile: 16, or 8 for double rows of 64 channels (the
// static shared-memory limit of 48 KB with the RoPE tables).
template <typename A, int D>
constexpr int tile_rows() {
  return (sizeof(A) == 8 && D >= 64) ? 8 : 16;
}

template <typename A>
__device__ __forceinline__ A a_exp(A x);
template <>
__device__ __forceinline__ double a_exp<double>(double x) {
  return exp(x);
}
template <>
__device__ __forceinline__ float a_exp<float>(float x) {
  return expf(x);
}
template <typename A>
__device__ __forceinline__ A a_log(A x);
template <>
__device__ __forceinline__ double a_log<double>(double x) {
  return log(x);
}
template <>
__device__ __forceinline__ float a_log<float>(float x) {
  return logf(x);
}
template <typename A>
__device__ __forceinline__ A a_sqrt(A x);
template <>
__device__ __forceinline__ double a_sqrt<double>(double x) {
  return sqrt(x);
}
template <>
__device__ __forceinline__ float a_sqrt<float>(float x) {
  return sqrtf(x);
}

template <typename T>
__device__ __forceinline__ float ld(const T* p);
template <>
__device__ __forceinline__ float ld<float>(const float* p) {
  return __ldg(p);
}
template <>
__device__ __forceinline__ float ld<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}
template <typename TG>
__device__ __forceinline__ TG st_conv(double x);
template <>
__device__ __forceinline__ float st_conv<float>(double x) {
  return (float)x;
}
template <>
__device__ __forceinline__ __nv_bfloat16 st_conv<__nv_bfloat16>(double x) {
  return __float2bfloat16_rn((float)x);  // a bf16 gradient is the fp32 one rounded
}

// RoPE tables [axis][p][t] (p < M, t < D/4) for the caller's frequencies.
template <typename A, int D>
__device__ void build_rope_tables(const float* freqs, int M, A* rc, A* rs) {
  constexpr int Qd = D / 4;
  for (int i = threadIdx.x; i < 2 * M * Qd; i += blockDim.x) {
    const int axis = i / (M * Qd), p = (i / Qd) % M, t = i % Qd;
    double sv, cv;
    sincos((double)p * (double)freqs[axis * Qd + t], &sv, &cv);
    rc[axis * kMaxM * Qd + p * Qd + t] = (A)cv;
    rs[axis * kMaxM * Qd + p * Qd + t] = (A)sv;
  }
}

// x <- R(p) x on one half (axis) of the channels; sign = -1 applies R^T.
template <typename A, int D>
__device__ __forceinline__ void rotate_half(A* x, int half, int p, const A* rc, const A* rs, A sign) {
  constexpr int Qd = D / 4;
  const A* c = rc + half * kMaxM * Qd + p * Qd;
  const A* s = rs + half * kMaxM * Qd + p * Qd;
#pragma unroll
  for (int t = 0; t < Qd; ++t) {
    const A a = x[half * (D / 2) + 2 * t], b = x[half * (D / 2) + 2 * t + 1];
    const A sn = sign * s[t];
    x[half * (D / 2) + 2 * t] = a * c[t] - b * sn;
    x[half * (D / 2) + 2 * t + 1] = a * sn + b * c[t];
  }
}

// Clamped norm of a row under the forward's rule: |x| if |x| > 1e-12, else
// 1e-12 (and then the norm is a constant).
template <typename A, int D>
__device__ __forceinline__ A clamped_norm(const A* x, bool& clamped) {
  A ss = 0;
#pragma unroll
  for (int e = 0; e < D; ++e) ss += x[e] * x[e];
  const A n = a_sqrt(ss);
  clamped = !(n > (A)kNormEps);
  return clamped ? (A)kNormEps : n;
}

template <typename A>
__device__ __forceinline__ A tau_eff(const float* tau, int h) {
  return (A)fmaxf(__ldg(tau + h), kTauMin);
}

// qt of one query row in place (see the header comment); returns the clamped
// norm in mode 1 (1 otherwise).
template <typename A, int D, int MODE>
__device__ __forceinline__ A prep_q(A* x, A t, int py, int px, const A* rc, const A* rs, bool& clamped) {
  const A rsd = (A)(1.0 / sqrt((double)D));
  clamped = false;
  A n = 1;
  if (MODE == 1) {
    n = clamped_norm<A, D>(x, clamped);
    const A sc = (A)1 / (n * t);
#pragma unroll
    for (int e = 0; e < D; ++e) x[e] *= sc;
  } else {
    if (MODE == 2) {
      rotate_half<A, D>(x, 0, py, rc, rs, (A)1);
      rotate_half<A, D>(x, 1, px, rc, rs, (A)1);
    }
#pragma unroll
    for (int e = 0; e < D; ++e) x[e] *= rsd;
  }
  return n;
}

// kt of one key row in place.
template <typename A, int D, int MODE>
__device__ __forceinline__ A prep_k(A* x, int py, int px, const A* rc, const A* rs, bool& clamped) {
  clamped = false;
  A n = 1;
  if (MODE == 1) {
    n = clamped_norm<A, D>(x, clamped);
    const A sc = (A)1 / n;
#pragma unroll
    for (int e = 0; e < D; ++e) x[e] *= sc;
  } else if (MODE == 2) {
    rotate_half<A, D>(x, 0, py, rc, rs, (A)1);
    rotate_half<A, D>(x, 1, px, rc, rs, (A)1);
  }
  return n;
}

// RoPE frequency gradient of one transformed row xt with gradient g: on each
// rotated pair, p * (g . J xt), added to acc[half * D/4 + t].
template <typename A, int D>
__device__ __forceinline__ void rope_grad(const A* xt, const A* g, int py, int px, A* acc) {
  constexpr int Qd = D / 4;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const A p = (A)(half == 0 ? py : px);
#pragma unroll
    for (int t = 0; t < Qd; ++t) {
      const int i0 = half * (D / 2) + 2 * t;
      acc[half * Qd + t] += p * (g[i0 + 1] * xt[i0] - g[i0] * xt[i0 + 1]);
    }
  }
}

// Adds the warp's sum of v (v = 0 on idle threads) to a double in shared
// memory.  Parameter-gradient partials are kept in double whatever the
// arithmetic type, so the varying order of the atomic additions moves the
// result by far less than one fp32 ulp.
template <typename A>
__device__ __forceinline__ void warp_sum_to(A v, double* smem_slot) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if ((threadIdx.x & 31) == 0) atomicAdd(smem_slot, (double)v);
}

// The CTA's rectangle (one window per axis) and its block of 128 rows.  Row
// kk of the rectangle is the token (Y(kk), X(kk)) with window-local
// coordinates (PY(kk), PX(kk)); offsets are differences of kk / lx, kk % lx.
struct Geometry {
  SwinAxis ay, ax;
  int lx, n, chunk;
  __device__ __forceinline__ int Y(int kk) const { return ay.start + ay.stride * (kk / lx); }
  __device__ __forceinline__ int X(int kk) const { return ax.start + ax.stride * (kk % lx); }
  __device__ __forceinline__ int PY(int kk) const { return ay.base + kk / lx; }
  __device__ __forceinline__ int PX(int kk) const { return ax.base + kk % lx; }
  __device__ __forceinline__ int rel(int qq, int kk, int M) const {
    return swin_rel_row(qq / lx - kk / lx, qq % lx - kk % lx, M);
  }
};

// Dot product of two rows, one FMA chain: split chains cost registers that
// lowered the occupancy of these kernels by a third and measured slower.
template <typename A, int D>
__device__ __forceinline__ A row_dot(const A* x, const A* y) {
  A d = 0;
#pragma unroll
  for (int e = 0; e < D; ++e) d += x[e] * y[e];
  return d;
}

__device__ __forceinline__ Geometry geometry(const BwdArgs& a, int nsx, int chunks) {
  Geometry g;
  const int rect = blockIdx.x / chunks;
  g.chunk = blockIdx.x % chunks;
  const int sy = rect / nsx, sx = rect % nsx;
  g.ay = swin_axis(a.part, sy, a.H, a.M, a.shift);
  g.ax = swin_axis(a.part, sx, a.W, a.M, a.shift);
  g.lx = g.ax.len;
  g.n = g.ay.len * g.lx;
  return g;
}

__device__ __forceinline__ size_t row_off(const BwdArgs& a, int b, int y, int x, int h, int D) {
  SWIN_DCHECK(a.status, b >= 0 && b < a.B && y >= 0 && y < a.H && x >= 0 && x < a.W && h >= 0 && h < a.heads);
  return (((size_t)b * a.H + y) * a.W + x) * (size_t)a.heads * D + (size_t)h * D;
}

template <typename A, int D, int MODE, int kTile = tile_rows<A, D>()>
struct Smem {
  A kv0[kTile][D];  // bwd_q: transformed keys; bwd_kv: transformed queries
  A kv1[kTile][D];  // bwd_q: values;          bwd_kv: output gradients
  A st0[kTile], st1[kTile];  // bwd_kv: lse and D of the query tile
  A rc[(MODE == 2) ? 2 * kMaxM * (D / 4) : 1];
  A rs[(MODE == 2) ? 2 * kMaxM * (D / 4) : 1];
  double red[1 + D / 2];  // CTA sums: d(tau), d(omega)
};

// NT threads per CTA (128, or 64 for windows of <= 64 tokens).  The register
// bound keeps three 128-thread CTAs per SM for fp32 arithmetic (170
// registers); one more register per thread would drop it to two.
template <typename T, typename TG, typename A, int D, int MODE, int NT>
__global__ void __launch_bounds__(NT, sizeof(A) == 4 ? 384 / NT : 1) bwd_q_kernel(BwdArgs a, int nsx, int chunks) {
  constexpr int kTile = tile_rows<A, D>();
  extern __shared__ __align__(16) unsigned char dyn[];  // double[(2M-1)^2]: this head's d(table)
  __shared__ Smem<A, D, MODE> sm;
  const Geometry G = geometry(a, nsx, chunks);
  constexpr int nt = NT;
  if (G.chunk * nt >= G.n) return;  // whole CTA idle (uniform)
  const int M = a.M, s = a.shift, h = blockIdx.y, b = blockIdx.z, R = 2 * M - 1;
  const bool want_T = MODE != 2 && a.acc_table != nullptr;
  double* sT = reinterpret_cast<double*>(dyn);
  if (want_T)
    for (int i = threadIdx.x; i < R * R; i += nt) sT[i] = 0;
  for (int i = threadIdx.x; i < 1 + D / 2; i += nt) sm.red[i] = 0;
  if (MODE == 2) build_rope_tables<A, D>(a.rope, M, sm.rc, sm.rs);
  __syncthreads();

  const T* Q = static_cast<const T*>(a.q);
  const T* K = static_cast<const T*>(a.k);
  const T* V = static_cast<const T*>(a.v);
  const T* GO = static_cast<const T*>(a.dout);
  const int qi = G.chunk * nt + threadIdx.x;
  const bool active = qi < G.n;
  const int qrow = active ? qi : 0;
  const int yq = G.Y(qrow), xq = G.X(qrow);
  const int pyq = G.PY(qrow), pxq = G.PX(qrow);
  const A t = MODE == 1 ? tau_eff<A>(a.tau, h) : (A)1;
  A qt[D], g[D];
  {
    const size_t off = row_off(a, b, yq, xq, h, D);
#pragma unroll
    for (int e = 0; e < D; ++e) {
      qt[e] = active ? (A)ld(Q + off + e) : (A)0;
      g[e] = active ? (A)ld(GO + off + e) : (A)0;
    }
  }
  bool qclamped;
  const A qn = prep_q<A, D, MODE>(qt, t, pyq, pxq, sm.rc, sm.rs, qclamped);

  // One tile of the rectangle's keys: kt into kv0, v into kv1.
  auto load_tile = [&](int j0, int nk) {
    __syncthreads();
    for (int i = threadIdx.x; i < nk * D; i += nt) {
      const int j = i / D, e = i % D, kk = j0 + j;
      const size_t off = row_off(a, b, G.Y(kk), G.X(kk), h, D) + e;
      sm.kv0[j][e] = (A)ld(K + off);
      sm.kv1[j][e] = (A)ld(V + off);
    }
    __syncthreads();
    if (MODE != 0 && threadIdx.x < nk) {
      const int kk = j0 + threadIdx.x;
      A row[D];
#pragma unroll
      for (int e = 0; e < D; ++e) row[e] = sm.kv0[threadIdx.x][e];
      bool c;
      prep_k<A, D, MODE>(row, G.PY(kk), G.PX(kk), sm.rc, sm.rs, c);
#pragma unroll
      for (int e = 0; e < D; ++e) sm.kv0[threadIdx.x][e] = row[e];
    }
    __syncthreads();
  };
  auto logit = [&](int j, int kk) {
    A dot = row_dot<A, D>(qt, sm.kv0[j]);
    if (MODE != 2 && a.table) {
      dot += (A)__ldg(a.table + (size_t)G.rel(qrow, kk, M) * a.heads + h);
    }
    return dot;
  };
  auto gdotv = [&](int j) { return row_dot<A, D>(g, sm.kv1[j]); };

  // pass 1: log-sum-exp and D = g . o by an online softmax
  A m = -INFINITY, l = 0, u = 0;
  for (int j0 = 0; j0 < G.n; j0 += kTile) {
    const int nk = min(kTile, G.n - j0);
    load_tile(j0, nk);
    if (!active) continue;
    for (int j = 0; j < nk; ++j) {
      const A lg = logit(j, j0 + j), gv = gdotv(j);
      if (lg > m) {
        const A c = a_exp(m - lg);
        l = l * c + (A)1;
        u = u * c + gv;
        m = lg;
      } else {
        const A p = a_exp(lg - m);
        l += p;
        u += p * gv;
      }
    }
  }
  const A lse = m + a_log(l), Dq = u / l;
  if (active) {
    const size_t si = ((((size_t)b * a.H + yq) * a.W + xq) * a.heads + h);
    a.stats[si] = make_double2((double)lse, (double)Dq);
  }

  // pass 2: dl, dqt, d(table)
  A dqt[D];
#pragma unroll
  for (int e = 0; e < D; ++e) dqt[e] = 0;
  for (int j0 = 0; j0 < G.n; j0 += kTile) {
    const int nk = min(kTile, G.n - j0);
    load_tile(j0, nk);
    if (!active) continue;
    for (int j = 0; j < nk; ++j) {
      const int kk = j0 + j;
      const A p = a_exp(logit(j, kk) - lse);
      const A dl = p * (gdotv(j) - Dq);
#pragma unroll
      for (int e = 0; e < D; ++e) dqt[e] += dl * sm.kv0[j][e];
      SWIN_DCHECK(a.status, !want_T || (G.rel(qrow, kk, M) >= 0 && G.rel(qrow, kk, M) < R * R));
      if (want_T) atomicAdd(&sT[G.rel(qrow, kk, M)], (double)dl);
    }
  }

  // back to q; parameter gradients of this query
  A dq[D];
  A dtau = 0;
  A drope[(MODE == 2) ? D / 2 : 1];
  if (MODE == 0) {
    const A rsd = (A)(1.0 / sqrt((double)D));
#pragma unroll
    for (int e = 0; e < D; ++e) dq[e] = dqt[e] * rsd;
  } else if (MODE == 1) {
    A qd = 0;
#pragma unroll
    for (int e = 0; e < D; ++e) qd += qt[e] * dqt[e];
    // the clamp passes the gradient where tau >= 0.01 as a real number (the
    // fp32 value nearest 0.01 lies just below it and is clamped)
    if ((double)__ldg(a.tau + h) >= 0.01) dtau = -qd / t;
    const A inv = (A)1 / (qn * t), tt = qclamped ? (A)0 : t * t * qd;
#pragma unroll
    for (int e = 0; e < D; ++e) dq[e] = (dqt[e] - tt * qt[e]) * inv;
  } else {
#pragma unroll
    for (int e = 0; e < D / 2; ++e) drope[e] = 0;
    rope_grad<A, D>(qt, dqt, pyq, pxq, drope);
    const A rsd = (A)(1.0 / sqrt((double)D));
#pragma unroll
    for (int e = 0; e < D; ++e) dq[e] = dqt[e] * rsd;
    rotate_half<A, D>(dq, 0, pyq, sm.rc, sm.rs, (A)-1);
    rotate_half<A, D>(dq, 1, pxq, sm.rc, sm.rs, (A)-1);
  }
  if (active) {
    TG* dst = static_cast<TG*>(a.dq) + row_off(a, b, yq, xq, h, D);
#pragma unroll
    for (int e = 0; e < D; ++e) dst[e] = st_conv<TG>((double)dq[e]);
  }
  if (!active) {
    dtau = 0;
    if (MODE == 2)
#pragma unroll
      for (int e = 0; e < D / 2; ++e) drope[e] = 0;
  }
  if (MODE == 1 && a.acc_tau) warp_sum_to(dtau, &sm.red[0]);
  if (MODE == 2 && a.acc_rope)
#pragma unroll
    for (int e = 0; e < D / 2; ++e) warp_sum_to(drope[e], &sm.red[1 + e]);
  __syncthreads();
  if (want_T)
    for (int i = threadIdx.x; i < R * R; i += nt)
      if (sT[i] != 0.0) atomicAdd(a.acc_table + (size_t)i * a.heads + h, sT[i]);
  if (MODE == 1 && a.acc_tau && threadIdx.x == 0) atomicAdd(a.acc_tau + h, sm.red[0]);
  if (MODE == 2 && a.acc_rope && threadIdx.x < D / 2) atomicAdd(a.acc_rope + threadIdx.x, sm.red[1 + threadIdx.x]);
}

template <typename T, typename TG, typename A, int D, int MODE, int NT>
__global__ void __launch_bounds__(NT, sizeof(A) == 4 ? 256 / NT : 1) bwd_kv_kernel(BwdArgs a, int nsx, int chunks) {
  constexpr int kTile = tile_rows<A, D>();
  __shared__ Smem<A, D, MODE> sm;
  const Geometry G = geometry(a, nsx, chunks);
  constexpr int nt = NT;
  if (G.chunk * nt >= G.n) return;
  const int M = a.M, s = a.shift, h = blockIdx.y, b = blockIdx.z;
  for (int i = threadIdx.x; i < 1 + D / 2; i += nt) sm.red[i] = 0;
  if (MODE == 2) build_rope_tables<A, D>(a.rope, M, sm.rc, sm.rs);
  __syncthreads();

  const T* Q = static_cast<const T*>(a.q);
  const T* K = static_cast<const T*>(a.k);
  const T* V = static_cast<const T*>(a.v);
  const T* GO = static_cast<const T*>(a.dout);
  const int kj = G.chunk * nt + threadIdx.x;
  const bool active = kj < G.n;
  const int krow = active ? kj : 0;
  const int yk = G.Y(krow), xk = G.X(krow);
  const int pyk = G.PY(krow), pxk = G.PX(krow);
  const A t = MODE == 1 ? tau_eff<A>(a.tau, h) : (A)1;
  A kt[D], vr[D];
  {
    const size_t off = row_off(a, b, yk, xk, h, D);
#pragma unroll
    for (int e = 0; e < D; ++e) {
      kt[e] = active ? (A)ld(K + off + e) : (A)0;
      vr[e] = active ? (A)ld(V + off + e) : (A)0;
    }
  }
  bool kclamped;
  const A kn = prep_k<A, D, MODE>(kt, pyk, pxk, sm.rc, sm.rs, kclamped);
  A dkt[D], dv[D];
#pragma unroll
  for (int e = 0; e < D; ++e) dkt[e] = dv[e] = 0;

  for (int i0 = 0; i0 < G.n; i0 += kTile) {
    const int nq = min(kTile, G.n - i0);
    __syncthreads();
    for (int i = threadIdx.x; i < nq * D; i += nt) {
      const int r = i / D, e = i % D, qq = i0 + r;
      const size_t off = row_off(a, b, G.Y(qq), G.X(qq), h, D) + e;
      sm.kv0[r][e] = (A)ld(Q + off);
      sm.kv1[r][e] = (A)ld(GO + off);
    }
    if (threadIdx.x < nq) {
      const int qq = i0 + threadIdx.x;
      const double2 st = a.stats[(((size_t)b * a.H + G.Y(qq)) * a.W + G.X(qq)) * a.heads + h];
      sm.st0[threadIdx.x] = (A)st.x;
      sm.st1[threadIdx.x] = (A)st.y;
    }
    __syncthreads();
    if (threadIdx.x < nq) {
      const int qq = i0 + threadIdx.x;
      A row[D];
#pragma unroll
      for (int e = 0; e < D; ++e) row[e] = sm.kv0[threadIdx.x][e];
      bool c;
      prep_q<A, D, MODE>(row, t, G.PY(qq), G.PX(qq), sm.rc, sm.rs, c);
#pragma unroll
      for (int e = 0; e < D; ++e) sm.kv0[threadIdx.x][e] = row[e];
    }
    __syncthreads();
    if (!active) continue;
    for (int i = 0; i < nq; ++i) {
      const int qq = i0 + i;
      A dot = row_dot<A, D>(sm.kv0[i], kt), gv = row_dot<A, D>(sm.kv1[i], vr);
      if (MODE != 2 && a.table) {
        dot += (A)__ldg(a.table + (size_t)G.rel(qq, krow, M) * a.heads + h);
      }
      const A p = a_exp(dot - sm.st0[i]);
      const A dl = p * (gv - sm.st1[i]);
#pragma unroll
      for (int e = 0; e < D; ++e) {
        dv[e] += p * sm.kv1[i][e];
        dkt[e] += dl * sm.kv0[i][e];
      }
    }
  }

  A dk[D];
  A drope[(MODE == 2) ? D / 2 : 1];
  if (MODE == 0) {
#pragma unroll
    for (int e = 0; e < D; ++e) dk[e] = dkt[e];
  } else if (MODE == 1) {
    A kd = 0;
#pragma unroll
    for (int e = 0; e < D; ++e) kd += kt[e] * dkt[e];
    const A inv = (A)1 / kn, kk = kclamped ? (A)0 : kd;
#pragma unroll
    for (int e = 0; e < D; ++e) dk[e] = (dkt[e] - kk * kt[e]) * inv;
  } else {
#pragma unroll
    for (int e = 0; e < D / 2; ++e) drope[e] = 0;
    rope_grad<A, D>(kt, dkt, pyk, pxk, drope);
#pragma unroll
    for (int e = 0; e < D; ++e) dk[e] = dkt[e];
    rotate_half<A, D>(dk, 0, pyk, sm.rc, sm.rs, (A)-1);
    rotate_half<A, D>(dk, 1, pxk, sm.rc, sm.rs, (A)-1);
  }
  if (active) {
    const size_t off = row_off(a, b, yk, xk, h, D);
    TG* dkd = static_cast<TG*>(a.dk) + off;
    TG* dvd = static_cast<TG*>(a.dv) + off;
#pragma unroll
    for (int e = 0; e < D; ++e) {
      dkd[e] = st_conv<TG>((double)dk[e]);
      dvd[e] = st_conv<TG>((double)dv[e]);
    }
  }
  if (MODE == 2 && a.acc_rope) {
    if (!active)
#pragma unroll
      for (int e = 0; e < D / 2; ++e) drope[e] = 0;
#pragma unroll
    for (int e = 0; e < D / 2; ++e) warp_sum_to(drope[e], &sm.red[1 + e]);
    __syncthreads();
    if (threadIdx.x < D / 2) atomicAdd(a.acc_rope + threadIdx.x, sm.red[1 + threadIdx.x]);
  }
}

__global__ void bwd_finish_kernel(const double* acc, int n_table, int n_tau, int n_rope, float* dtable,
                                  float* dtau, float* drope) {
  const int n = n_table + n_tau + n_rope;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    const float v = (float)acc[i];
    if (i < n_table) {
      if (dtable) dtable[i] = v;
    } else if (i < n_table + n_tau) {
      if (dtau) dtau[i - n_table] = v;
    } else if (drope) {
      drope[i - n_table - n_tau] = v;
    }
  }
}

template <typename T, typename TG, typename A, int D, int MODE, int NT>
swin_status launch_nt(const BwdArgs& a, cudaStream_t stream) {
  const int nsy = swin_nwin(a.part, a.H, a.M, a.shift), nsx = swin_nwin(a.part, a.W, a.M, a.shift);
  constexpr int nt = NT;
  const int chunks = (a.M * a.M + nt - 1) / nt;
  const dim3 grid(nsy * nsx * chunks, a.heads, a.B);
  const size_t dyn = (MODE != 2 && a.acc_table) ? sizeof(double) * (size_t)(2 * a.M - 1) * (2 * a.M - 1) : 0;
  auto kq = bwd_q_kernel<T, TG, A, D, MODE, NT>;
  if (dyn > 0) {  // static plus dynamic shared memory may pass the 48 KB default
    cudaError_t e = cudaFuncSetAttribute(kq, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn);
    if (e != cudaSuccess) return fail(SWIN_ERR_CUDA, "attn_bwd smem attribute: %s", cudaGetErrorString(e));
  }
  kq<<<grid, nt, dyn, stream>>>(a, nsx, chunks);
  bwd_kv_kernel<T, TG, A, D, MODE, NT><<<grid, nt, 0, stream>>>(a, nsx, chunks);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(SWIN_ERR_CUDA, "attn_bwd launch: %s", cudaGetErrorString(e));
  return SWIN_OK;
}

template <typename T, typename TG, typename A, int D, int MODE>
swin_status launch_mode(const BwdArgs& a, cudaStream_t stream) {
  // windows of <= 64 tokens: 64 threads, so fewer of them idle
  return a.M * a.M <= 64 ? launch_nt<T, TG, A, D, MODE, 64>(a, stream)
                         : launch_nt<T, TG, A, D, MODE, kThreads>(a, stream);
}

template <typename T, typename TG, typename A, int D>
swin_status launch_d(const BwdArgs& a, cudaStream_t stream) {
  switch (a.mode) {
    case 0: return launch_mode<T, TG, A, D, 0>(a, stream);
    case 1: return launch_mode<T, TG, A, D, 1>(a, stream);
    default:
      if constexpr (D % 4 == 0) return launch_mode<T, TG, A, D, 2>(a, stream);
      return fail(SWIN_ERR_INVALID_ARG, "RoPE mode needs d %% 4 == 0");
  }
}

template <typename T, typename TG, typename A>
swin_status launch_typed(const BwdArgs& a, cudaStream_t stream) {
  switch (a.d) {
    case 8: return launch_d<T, TG, A, 8>(a, stream);
    case 16: return launch_d<T, TG, A, 16>(a, stream);
    case 32: return launch_d<T, TG, A, 32>(a, stream);
    case 64: return launch_d<T, TG, A, 64>(a, stream);
    default: return fail(SWIN_ERR_UNSUPPORTED, "backward supports d in {8,16,32,64}, got %d", a.d);
  }
}

}  // namespace

swin_status launch_attn_bwd(const BwdArgs& a, bool bf16_in, bool f32_grad, float* dtable, float* dtau,
                            float* drope, cudaStream_t stream) {
  if (a.M > kMaxM) return fail(SWIN_ERR_UNSUPPORTED, "M=%d above %d", a.M, kMaxM);
  const int n_table = a.acc_table ? (2 * a.M - 1) * (2 * a.M - 1) * a.heads : 0;
  const int n_tau = a.acc_tau ? a.heads : 0;
  const int n_rope = a.acc_rope ? 2 * (a.d / 4) : 0;
  const int n_acc = n_table + n_tau + n_rope;
  if (n_acc) {
    cudaError_t e = cudaMemsetAsync(a.acc_base, 0, sizeof(double) * (size_t)n_acc, stream);
    if (e != cudaSuccess) return fail(SWIN_ERR_CUDA, "attn_bwd memset: %s", cudaGetErrorString(e));
  }
  swin_status st;
  if (attn_bwd_tc_supported(a, bf16_in))
    st = launch_attn_bwd_tc(a, f32_grad, stream);
  else if (!bf16_in)
    st = launch_typed<float, float, double>(a, stream);
  else if (f32_grad)
    st = launch_typed<__nv_bfloat16, float, float>(a, stream);
  else
    st = launch_typed<__nv_bfloat16, __nv_bfloat16, float>(a, stream);
  if (st != SWIN_OK || !n_acc) return st;
  bwd_finish_kernel<<<(n_acc + 255) / 256, 256, 0, stream>>>(a.acc_base, n_table, n_tau, n_rope, dtable, dtau,
                                                             drope);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(SWIN_ERR_CUDA, "attn_bwd finish launch: %s", cudaGetErrorString(e));
  return SWIN_OK;
}

}  // namespace swin
