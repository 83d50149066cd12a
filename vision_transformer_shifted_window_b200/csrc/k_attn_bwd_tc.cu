// Gradients of shifted-window attention on the tensor cores (bf16 tensors,
// d = 32): the five products of the backward pass — S = Q K^T, dP = dO V^T,
// dV = P^T dO, dK = dS^T Q, dQ = dS K — as tcgen05 MMAs with TMEM
// accumulators, in two kernels that never materialise a score matrix:
//
//   bwd_tc_q   one CTA per query tile (<= 128 tokens of a rectangle, one TMEM
//              lane each).  Pass 1 sweeps the rectangle's key blocks (64 keys)
//              with S and dP and keeps each row's log-sum-exp and
//              D = sum_j P dP = dO . O (online, like the forward's softmax);
//              pass 2 repeats S and dP, forms dl = P (dP - D) and
//              dS = dl * (the score's derivative), stores dS as fp16 into TMEM
//              and accumulates dQ += dS K there.  The statistics go to the
//              workspace; the bias-table gradient is summed in shared memory.
//   bwd_tc_kv  one CTA per key tile; query blocks of 64 stream by with their
//              statistics: S^T = K Q^T, dP^T = V dO^T, P^T and dS^T into TMEM,
//              dV += P^T dO and dK += dS^T Q.
//
// The math is the chain rule of the forward definition ("Swin Transformer V2"
// eq. 1 and eq. 2, tau clamped at 0.01, §3.2; FlashSwin's window-local RoPE),
// the same as the CUDA-core backward; every mode is q~ . k~ + T[r]:
//   mode 0  q~ = q / sqrt(d), k~ = k;  mode 1  q~ = q / (|q| t), k~ = k / |k|;
//   mode 2  q~ = R q / sqrt(d), k~ = R k,
// with the per-row factors applied to the raw (or rotated) operands' products
// in fp32 and folded into dS, and each transform's Jacobian applied to the
// accumulated gradient in the epilogue.
//
// Operands.  Every MMA is kind::f16 with fp16 A and B (one type per MMA):
// Q, K, V and dO are converted from bf16 to fp16 in shared memory (exact for
// bf16 values inside fp16's range); RoPE rows are rotated in fp32 and kept as
// two fp16 parts, hi and lo, so that S = Q_hi K_hi^T + Q_lo K_hi^T +
// Q_hi K_lo^T and the dQ, dK products against both parts carry the rotated
// operands to about 22 bits (a float64 replay of these roundings on the
// FlashSwin workload: with single fp16 rotated operands dq and dk reach 1.5-2 %
// of their RMS on one image, with the split about 0.5 %); P and dS are fp16 in
// TMEM.  An operand at or beyond fp16's range
// (65504) saturates and the call reports SWIN_ERR_UNSUPPORTED through the
// status word, as the forward does.  Rows are loaded by the CTA's threads
// with 16-byte loads into the 64-byte-swizzled layout the MMA descriptors
// describe (a tile is the next tokens of the rectangle in row-major order), so
// both window partitions are served.  Synchronisation is one mbarrier for MMA
// completion plus CTA barriers: a simple, fully synchronous pipeline; several
// CTAs per SM overlap one another's latencies.  Every wait is bounded; on time
// -out the kernel records SWIN_ERR_TIMEOUT and leaves its loops.
#include <algorithm>

#include "sm100_ptx.cuh"
#include "swin_common.cuh"

namespace swin {
namespace {

constexpr int kD = 32;
constexpr int kRows = 128;  // TMEM lanes = tile rows
constexpr int kBlk = 64;    // keys (bwd_tc_q) or queries (bwd_tc_kv) per block
constexpr int kThreads = 128;
constexpr int kTileB = kRows * 64;  // bytes of a 128-row tile of 32 fp16
constexpr int kBlkB = kBlk * 64;
constexpr float kLog2e = 1.4426950408889634f;
constexpr long long kWaitLimit = 2000000000ll;  // clock64 cycles (about one second)

__device__ __forceinline__ uint32_t swz(int row, int chunk) {
  // byte offset of 16-byte chunk `chunk` of 64-byte row `row` under the 64-byte swizzle
  return (uint32_t)(row * 64 + ((chunk ^ ((row >> 1) & 3)) << 4));
}

// One token's head row (32 bf16) as four 16-byte words, and those words as floats.
__device__ __forceinline__ void load_raw(const __nv_bfloat16* src, uint4 (&w)[4]) {
  const uint4* s4 = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int c = 0; c < 4; ++c) w[c] = __ldg(s4 + c);
}

__device__ __forceinline__ void unpack_row(const uint4 (&w)[4], float (&v)[kD]) {
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const uint32_t u[4] = {w[c].x, w[c].y, w[c].z, w[c].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      v[8 * c + 2 * e] = __uint_as_float(u[e] << 16);
      v[8 * c + 2 * e + 1] = __uint_as_float(u[e] & 0xFFFF0000u);
    }
  }
}

// One token's head row (32 bf16) into floats.
__device__ __forceinline__ void load_row(const __nv_bfloat16* src, float (&v)[kD]) {
  const uint4* s4 = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const uint4 w = __ldg(s4 + c);
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      v[8 * c + 2 * e] = __uint_as_float(u[e] << 16);
      v[8 * c + 2 * e + 1] = __uint_as_float(u[e] & 0xFFFF0000u);
    }
  }
}

// One token's head row (32 bf16) as raw 16-byte words, loaded ahead of use.
struct RawRow {
  uint4 w[4];
};
__device__ __forceinline__ void fetch_row(const __nv_bfloat16* src, RawRow& r) {
  const uint4* s4 = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int c = 0; c < 4; ++c) r.w[c] = __ldg(s4 + c);
}
__device__ __forceinline__ void unpack_row(const RawRow& r, float (&v)[32]) {
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const uint32_t u[4] = {r.w[c].x, r.w[c].y, r.w[c].z, r.w[c].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      v[8 * c + 2 * e] = __uint_as_float(u[e] << 16);
      v[8 * c + 2 * e + 1] = __uint_as_float(u[e] & 0xFFFF0000u);
    }
  }
}

// A row of 32 values as fp16 into a swizzled tile; returns whether an entry
// reached fp16's range limit (saturated).
__device__ __forceinline__ bool store_row_f16(uint8_t* tile, int row, const float (&v)[kD]) {
  bool hit = false;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint32_t u[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float a = v[8 * c + 2 * e], b = v[8 * c + 2 * e + 1];
      hit |= fabsf(a) >= 65504.f || fabsf(b) >= 65504.f;
      u[e] = ptx::pack_f16x2_sat(a, b);
    }
    *reinterpret_cast<uint4*>(tile + swz(row, c)) = make_uint4(u[0], u[1], u[2], u[3]);
  }
  return hit;
}

// A row as fp16 hi + lo parts (hi = the row rounded to fp16, lo = the rest
// rounded to fp16): two MMAs on hi and lo carry the row to about 22 bits.
__device__ __forceinline__ bool store_row_f16_split(uint8_t* hi_tile, uint8_t* lo_tile, int row,
                                                    const float (&v)[kD]) {
  float hi[kD], lo[kD];
#pragma unroll
  for (int e = 0; e < kD; ++e) {
    hi[e] = __half2float(__float2half_rn(v[e]));
    lo[e] = v[e] - hi[e];
  }
  const bool hit = store_row_f16(hi_tile, row, v);
  store_row_f16(lo_tile, row, lo);
  return hit;
}

__device__ __forceinline__ void zero_row(uint8_t* tile, int row) {
#pragma unroll
  for (int c = 0; c < 4; ++c) *reinterpret_cast<uint4*>(tile + swz(row, c)) = make_uint4(0, 0, 0, 0);
}

// x <- R(p) x (sign +1) or R(p)^T x (sign -1) on one half of the channels,
// from the CTA's cos / sin tables [axis][p][8].
__device__ __forceinline__ void rotate(float (&x)[kD], int half, int p, const float* rc, const float* rs,
                                       float sign) {
  const float* c = rc + (half * 64 + p) * 8;
  const float* s = rs + (half * 64 + p) * 8;
#pragma unroll
  for (int t = 0; t < 8; ++t) {
    const float a = x[half * 16 + 2 * t], b = x[half * 16 + 2 * t + 1], sn = sign * s[t];
    x[half * 16 + 2 * t] = a * c[t] - b * sn;
    x[half * 16 + 2 * t + 1] = a * sn + b * c[t];
  }
}

// p * (g . J x) on each rotated pair, added to acc[half * 8 + t].
__device__ __forceinline__ void rope_grad(const float (&x)[kD], const float (&g)[kD], int py, int px,
                                          float (&acc)[16]) {
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const float p = (float)(half ? px : py);
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      const int i0 = half * 16 + 2 * t;
      acc[half * 8 + t] += p * (g[i0 + 1] * x[i0] - g[i0] * x[i0 + 1]);
    }
  }
}

__device__ __forceinline__ float clamped_norm(const float (&v)[kD], bool& clamped) {
  float ss = 0.f;
#pragma unroll
  for (int e = 0; e < kD; ++e) ss = fmaf(v[e], v[e], ss);
  const float n = sqrtf(ss);
  clamped = !(n > kNormEps);
  return clamped ? kNormEps : n;
}

struct TcBwd {
  const __nv_bfloat16 *q, *k, *v, *dout;
  void *dq, *dk, *dv;
  void* out;  // the forward kernel's output
  int B, H, W, heads, M, shift, part;
  const float* tau;
  const float* table;
  const float* rope;
  double *acc_table, *acc_tau, *acc_rope;
  double2* stats;
  int* status;
  int nsx, tiles;  // rectangles per row of rectangles; tiles (of 128 tokens) per rectangle
};

struct Rect {
  SwinAxis ay, ax;
  int n;
  // iy (2M - 1) + ix of rectangle token t: the bias-table row of a pair is
  // off(query) - off(key) + (M - 1) 2M
  __device__ __forceinline__ int off(int t, int R) const { return (t / ax.len) * R + t % ax.len; }
  __device__ __forceinline__ int Y(int t) const { return ay.start + ay.stride * (t / ax.len); }
  __device__ __forceinline__ int X(int t) const { return ax.start + ax.stride * (t % ax.len); }
  __device__ __forceinline__ int PY(int t) const { return ay.base + t / ax.len; }
  __device__ __forceinline__ int PX(int t) const { return ax.base + t % ax.len; }
};

__device__ __forceinline__ Rect rect_of(const TcBwd& p, int rect) {
  Rect r;
  r.ay = swin_axis(p.part, rect / p.nsx, p.H, p.M, p.shift);
  r.ax = swin_axis(p.part, rect % p.nsx, p.W, p.M, p.shift);
  r.n = r.ay.len * r.ax.len;
  return r;
}

__device__ __forceinline__ size_t tok_off(const TcBwd& p, int b, int y, int x, int h) {
  SWIN_DCHECK(p.status, b >= 0 && b < p.B && y >= 0 && y < p.H && x >= 0 && x < p.W && h >= 0 && h < p.heads);
  return (((size_t)b * p.H + y) * p.W + x) * (size_t)p.heads * kD + (size_t)h * kD;
}

// Bounded wait on phase `parity` of the MMA barrier, by thread 0 alone (the
// issuer; it sleeps in hardware between probes) while the other threads wait
// at the CTA barrier that follows, issuing nothing; every thread then orders
// its TMEM reads after the MMAs with tcgen05.fence::after_thread_sync.  Returns
// false on every thread (and records the status) if the wait gave up.
__device__ __forceinline__ bool wait_mma(uint64_t* bar, uint32_t parity, int* status) {
  bool ok = true;
  if (threadIdx.x == 0 && !ptx::mbar_try_wait(bar, parity)) {
    const long long t0 = clock64();
    while (!ptx::mbar_try_wait_sleep(bar, parity, 20000u))
      if (clock64() - t0 > kWaitLimit) {
        atomicOr(status, (int)SWIN_ERR_TIMEOUT);
        ok = false;
        break;
      }
  }
  return __syncthreads_and(ok);
}

template <typename TG>
__device__ __forceinline__ void store_grad(TG* dst, const float (&g)[kD]);
template <>
__device__ __forceinline__ void store_grad<float>(float* dst, const float (&g)[kD]) {
  float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
  for (int c = 0; c < 8; ++c) d4[c] = make_float4(g[4 * c], g[4 * c + 1], g[4 * c + 2], g[4 * c + 3]);
}
template <>
__device__ __forceinline__ void store_grad<__nv_bfloat16>(__nv_bfloat16* dst, const float (&g)[kD]) {
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int c = 0; c < 4; ++c)
    d4[c] = make_uint4(ptx::pack_bf16x2(g[8 * c], g[8 * c + 1]), ptx::pack_bf16x2(g[8 * c + 2], g[8 * c + 3]),
                       ptx::pack_bf16x2(g[8 * c + 4], g[8 * c + 5]), ptx::pack_bf16x2(g[8 * c + 6], g[8 * c + 7]));
}

// Shared memory common to both kernels, after the operand tiles.
struct SmemCommon {
  float rc[2 * 64 * 8], rs[2 * 64 * 8];  // RoPE cos / sin [axis][p][t]
  // per block column, double-buffered with the operand blocks:
  float colf[2][kBlk];                   // 1/|k| (q kernel) or 1/(tau |q|) (kv kernel)
  int coff[2][kBlk];                     // iy (2M-1) + ix of its token in the rectangle
  float lse2[2][kBlk], dsum[2][kBlk];    // kv kernel: statistics of the block's queries
  double red[1 + 16];                    // CTA sums: d(tau), d(omega)
  uint64_t mma_bar;
  uint32_t tmem_base;
  int range_hit;
};

__device__ void build_rope(const float* freqs, int M, float* rc, float* rs) {
  for (int i = threadIdx.x; i < 2 * M * 8; i += kThreads) {
    const int axis = i / (M * 8), p = (i / 8) % M, t = i % 8;
    double sv, cv;
    sincos((double)p * (double)freqs[axis * 8 + t], &sv, &cv);
    rc[(axis * 64 + p) * 8 + t] = (float)cv;
    rs[(axis * 64 + p) * 8 + t] = (float)sv;
  }
}

// A row's raw head vector prepared as the MMA operand: mode 2 rotates it to
// window-local positions (py, px); the fp32 row is kept in `v`.
template <int MODE>
__device__ __forceinline__ void prep_row(float (&v)[kD], int py, int px, const float* rc, const float* rs) {
  if (MODE == 2) {
    rotate(v, 0, py, rc, rs, 1.f);
    rotate(v, 1, px, rc, rs, 1.f);
  }
}

// Warp sum of v added to a shared double.
__device__ __forceinline__ void warp_add(float v, double* slot) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if ((threadIdx.x & 31) == 0) atomicAdd(slot, (double)v);
}

// ============================================================== query kernel
template <int MODE, bool TABLE, typename TG>
__global__ void __launch_bounds__(kThreads) bwd_tc_q(const __grid_constant__ TcBwd p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* qs = smem;                  // Q tile, fp16 (128 rows)
  uint8_t* gs = qs + kTileB;           // dO tile, fp16
  uint8_t* qlo = gs + kTileB;          // mode 2: lo parts of the rotated Q tile
  uint8_t* kvb = qlo + kTileB;         // two buffers of [K block | V block | K lo parts] (64 rows each)
  SmemCommon* sc = reinterpret_cast<SmemCommon*>(kvb + 2 * 3 * kBlkB);
  float* tab = reinterpret_cast<float*>(sc + 1);  // (2M-1)^2 table entries x log2 e (TABLE)
  const int R = 2 * p.M - 1, RR = R * R;
  double* dtab = reinterpret_cast<double*>(tab + (TABLE ? ((RR + 1) & ~1) : 0));  // d(table) sums

  const int rect = blockIdx.x / p.tiles, tile = blockIdx.x % p.tiles;
  const int h = blockIdx.y, b = blockIdx.z;
  const Rect rc = rect_of(p, rect);
  const int t0 = tile * kRows;
  if (t0 >= rc.n) return;  // uniform
  const int tid = threadIdx.x, warp = tid >> 5;
  const int tq = t0 + tid;
  const bool row_ok = tq < rc.n;
  const bool want_T = TABLE && p.acc_table != nullptr;

  if (tid == 0) {
    ptx::mbar_init(&sc->mma_bar, 1);
    ptx::fence_mbar_init();
    sc->range_hit = 0;
  }
  if (warp == 0) {
    ptx::tmem_alloc(&sc->tmem_base, 256);
    ptx::tmem_relinquish();
  }
  for (int i = tid; i < 17; i += kThreads) sc->red[i] = 0.0;
  if (MODE == 2) build_rope(p.rope, p.M, sc->rc, sc->rs);
  if (TABLE)
    for (int i = tid; i < RR; i += kThreads) tab[i] = __ldg(p.table + (size_t)i * p.heads + h) * kLog2e;
  if (want_T)
    for (int i = tid; i < RR; i += kThreads) dtab[i] = 0.0;
  __syncthreads();

  // ---- this row: Q (prepared), dO, per-row factor
  const float t_eff = MODE == 1 ? fmaxf(__ldg(p.tau + h), kTauMin) : 1.f;
  float qrow[kD], grow[kD];
  bool qclamped = false;
  float qn = 1.f;
  const int pyq = row_ok ? rc.PY(tq) : 0, pxq = row_ok ? rc.PX(tq) : 0;
  {
    bool hit = false;
    if (row_ok) {
      const size_t off = tok_off(p, b, rc.Y(tq), rc.X(tq), h);
      load_row(p.q + off, qrow);
      load_row(p.dout + off, grow);
      if (MODE == 1) qn = clamped_norm(qrow, qclamped);
      prep_row<MODE>(qrow, pyq, pxq, sc->rc, sc->rs);
      hit |= MODE == 2 ? store_row_f16_split(qs, qlo, tid, qrow) : store_row_f16(qs, tid, qrow);
      hit |= store_row_f16(gs, tid, grow);
    } else {
#pragma unroll
      for (int e = 0; e < kD; ++e) qrow[e] = grow[e] = 0.f;
      zero_row(qs, tid);
      zero_row(gs, tid);
      if (MODE == 2) zero_row(qlo, tid);
    }
    if (hit) sc->range_hit = 1;
  }
  // per-row factor of the raw product in the log2 domain
  const float arow = MODE == 1 ? 1.f / (qn * t_eff) : 0.f;
  const float srow = MODE == 1 ? kLog2e * arow : kLog2e * rsqrtf((float)kD);
  const float dscale = MODE == 1 ? 1.f : rsqrtf((float)kD);  // dS = dl * dscale * colf(mode 1)
  // table row of the pair (this query, key j) = qbase - coff[j]
  const int qbase = rc.off(row_ok ? tq : t0, R) + (p.M - 1) * (R + 1);

  ptx::fence_proxy_async_smem();
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tbase = sc->tmem_base;
  const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
  const uint32_t tS = tbase, tP = tbase + 64, tDS = tbase + 128, tDQ = tbase + 160;  // column offsets
  constexpr uint32_t idS = ptx::idesc_f16(0, 0, 0, 0, kBlk, kRows);
  constexpr uint32_t idDQ = ptx::idesc_f16(0, 0, 0, 1, kD, kRows);
  const uint64_t qd = ptx::smem_desc(ptx::smem_addr(qs), 16, 512, ptx::kSwizzle64B);
  const uint64_t gd = ptx::smem_desc(ptx::smem_addr(gs), 16, 512, ptx::kSwizzle64B);
  const uint64_t qld = ptx::smem_desc(ptx::smem_addr(qlo), 16, 512, ptx::kSwizzle64B);
  // buffer x: K at kvb + 3 x kBlkB, V after it, K lo parts after that
  auto kbuf = [&](int x) { return kvb + 3 * x * kBlkB; };
  auto kdesc = [&](int x, int part) {
    return ptx::smem_desc(ptx::smem_addr(kbuf(x) + part * kBlkB), 16, 512, ptx::kSwizzle64B);
  };
  uint32_t phase = 0;
  bool ok = true;

  float m2 = -INFINITY, l = 0.f, u = 0.f;  // pass 1: running max (log2), sum, sum of p dP
  float lse2 = 0.f, Dv = 0.f;
  const int nkb = (rc.n + kBlk - 1) / kBlk;
  const int nsteps = 2 * nkb;  // pass 1 then pass 2 over the key blocks; step g uses buffer g & 1
  // Threads 0-63 carry K rows of a block, 64-127 V rows.  A step's rows are
  // fetched (registers) while the previous step computes, and stored once its
  // buffer is free: the wait on a step's S / dP commit also covers the dQ
  // MMAs issued before it, the last readers of the other buffer.
  const int lr = tid & (kBlk - 1);
  const bool isk = tid < kBlk;
  RawRow pre;
  auto fetch = [&](int g) {
    const int tk = (g % nkb) * kBlk + lr;
    if (tk < rc.n) fetch_row((isk ? p.k : p.v) + tok_off(p, b, rc.Y(tk), rc.X(tk), h), pre);
  };
  auto stash = [&](int g) {
    const int x = g & 1, tk = (g % nkb) * kBlk + lr;
    uint8_t* kt = kbuf(x);
    bool hit = false;
    if (isk) sc->coff[x][lr] = rc.off(min(tk, rc.n - 1), R);  // masked keys: a valid row, weight 0
    if (tk < rc.n) {
      float v[kD];
      unpack_row(pre, v);
      if (isk) {
        if (MODE == 1) {
          bool c;
          sc->colf[x][lr] = 1.f / clamped_norm(v, c);
        }
        prep_row<MODE>(v, rc.PY(tk), rc.PX(tk), sc->rc, sc->rs);
        hit = MODE == 2 ? store_row_f16_split(kt, kt + 2 * kBlkB, lr, v) : store_row_f16(kt, lr, v);
      } else {
        hit = store_row_f16(kt + kBlkB, lr, v);
      }
    } else {
      zero_row(isk ? kt : kt + kBlkB, lr);
      if (isk && MODE == 2) zero_row(kt + 2 * kBlkB, lr);
      if (isk && MODE == 1) sc->colf[x][lr] = 0.f;
    }
    if (hit) sc->range_hit = 1;
  };
  fetch(0);
  stash(0);
  ptx::fence_proxy_async_smem();
  ptx::tc_fence_before();
  __syncthreads();
  for (int g = 0; g < nsteps && ok; ++g) {
    const int x = g & 1, pass = g / nkb, kb = g % nkb;
    const int k0 = kb * kBlk, nk = min(kBlk, rc.n - k0);
    const uint64_t kd = kdesc(x, 0), vd = kdesc(x, 1), kld = kdesc(x, 2);
    // ---- S = Q K^T, dP = dO V^T (the commit also covers the previous dQ MMAs)
    if (tid == 0) {
      ptx::tc_fence_after();
      ptx::mma_ss(tS, qd, kd, idS, 0);
      ptx::mma_ss(tS, qd + 2, kd + 2, idS, 1);
      if (MODE == 2) {  // + Q_lo K_hi^T + Q_hi K_lo^T
        ptx::mma_ss(tS, qld, kd, idS, 1);
        ptx::mma_ss(tS, qld + 2, kd + 2, idS, 1);
        ptx::mma_ss(tS, qd, kld, idS, 1);
        ptx::mma_ss(tS, qd + 2, kld + 2, idS, 1);
      }
      ptx::mma_ss(tP, gd, vd, idS, 0);
      ptx::mma_ss(tP, gd + 2, vd + 2, idS, 1);
      ptx::mma_commit(&sc->mma_bar);
    }
    if (g + 1 < nsteps) fetch(g + 1);  // in flight during the MMAs and the softmax
    ok = wait_mma(&sc->mma_bar, phase, p.status);
    phase ^= 1;
    if (!ok) break;
    ptx::tc_fence_after();
    const float* colf = sc->colf[x];
    const int* coff = sc->coff[x];
    // the block's 64 keys in two halves of 32 (TMEM columns 32 hf ..)
    for (int hf = 0; hf < 2; ++hf) {
      uint32_t sr[32], dr[32];
      ptx::tmem_ld32(tS + 32 * hf + lane_off, sr);
      ptx::tmem_ld32(tP + 32 * hf + lane_off, dr);
      ptx::tmem_wait_ld();
      // logit of key j of this half in the log2 domain; masked keys -inf
      auto logit = [&](int j) {
        const int jj = 32 * hf + j;
        float xv = MODE == 1 ? __uint_as_float(sr[j]) * srow * colf[jj] : __uint_as_float(sr[j]) * srow;
        SWIN_DCHECK(p.status, !TABLE || (qbase - coff[jj] >= 0 && qbase - coff[jj] < RR));
        if (TABLE) xv += tab[qbase - coff[jj]];
        return jj < nk ? xv : -INFINITY;
      };
      if (pass == 0) {
        float mb = m2;
#pragma unroll
        for (int j = 0; j < 32; ++j) mb = fmaxf(mb, logit(j));
        const float c = ptx::ex2_approx(m2 - mb);  // 0 at the first half (m2 = -inf)
        l *= c;
        u *= c;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float pj = ptx::ex2_approx(logit(j) - mb);
          l += pj;
          u = fmaf(pj, __uint_as_float(dr[j]), u);
        }
        m2 = mb;
      } else {
        // dl = P (dP - D); dS = dl * (d logit / d raw product), fp16 into TMEM
        uint32_t pk[16];
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          float dl[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int jj = 32 * hf + j + e;
            const float pj = ptx::ex2_approx(logit(j + e) - lse2);  // 0 for masked keys
            dl[e] = row_ok ? pj * (__uint_as_float(dr[j + e]) - Dv) : 0.f;
            if (want_T && row_ok && jj < nk) atomicAdd(&dtab[qbase - coff[jj]], (double)dl[e]);
          }
          float a0 = dl[0] * dscale, a1 = dl[1] * dscale;
          if (MODE == 1) {
            a0 *= colf[32 * hf + j];
            a1 *= colf[32 * hf + j + 1];
          }
          if (fabsf(a0) >= 65504.f || fabsf(a1) >= 65504.f) sc->range_hit = 1;
          pk[j / 2] = ptx::pack_f16x2_sat(a0, a1);
        }
        ptx::tmem_st16(tDS + 16 * hf + lane_off, pk);
      }
    }
    if (pass == 0 && kb == nkb - 1) {
      lse2 = m2 + __log2f(l);
      Dv = u / l;
      if (row_ok)
        p.stats[(((size_t)b * p.H + rc.Y(tq)) * p.W + rc.X(tq)) * p.heads + h] = make_double2((double)lse2, (double)Dv);
    }
    if (pass == 1) {
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      __syncthreads();
      // ---- dQ += dS K (A = dS from TMEM, B = K as MN-major [keys x d]); not
      // waited for here: the next step's S / dP commit covers it
      if (tid == 0) {
        ptx::tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kBlk / 16; ++kk) {
          ptx::mma_ts(tDQ, tDS + kk * 8, kd + (uint64_t)(kk * 1024 >> 4), idDQ, (kb > 0 || kk > 0) ? 1u : 0u);
          if (MODE == 2) ptx::mma_ts(tDQ, tDS + kk * 8, kld + (uint64_t)(kk * 1024 >> 4), idDQ, 1u);
        }
      }
    }
    // the next step's buffer: its last readers (step g - 1's MMAs) are complete
    if (g + 1 < nsteps) stash(g + 1);
    ptx::fence_proxy_async_smem();
    ptx::tc_fence_before();
    __syncthreads();
  }
  // the last dQ MMAs
  if (ok) {
    if (tid == 0) {
      ptx::tc_fence_after();
      ptx::mma_commit(&sc->mma_bar);
    }
    ok = wait_mma(&sc->mma_bar, phase, p.status);
    phase ^= 1;
  }

  // ---- epilogue: dq from the accumulated gradient of the prepared q
  float dtau = 0.f, drope[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) drope[e] = 0.f;
  if (ok) {
    ptx::tc_fence_after();
    uint32_t acc[32];
    ptx::tmem_ld32(tDQ + lane_off, acc);
    ptx::tmem_wait_ld();
    float g[kD];
#pragma unroll
    for (int e = 0; e < kD; ++e) g[e] = __uint_as_float(acc[e]);
    if (MODE == 1) {
      // q~ = a q, dq~ = g; dq = (g - t^2 (q~ . g) q~) a, d(tau) = -(q~ . g) / t
      float qd2 = 0.f;
#pragma unroll
      for (int e = 0; e < kD; ++e) qd2 = fmaf(qrow[e] * arow, g[e], qd2);
      // the clamp passes the gradient where tau >= 0.01 as a real number
      if ((double)__ldg(p.tau + h) >= 0.01) dtau = row_ok ? -qd2 / t_eff : 0.f;
      const float tt = qclamped ? 0.f : t_eff * t_eff * qd2;
#pragma unroll
      for (int e = 0; e < kD; ++e) g[e] = (g[e] - tt * qrow[e] * arow) * arow;
    } else if (MODE == 2) {
      if (row_ok) rope_grad(qrow, g, pyq, pxq, drope);
      rotate(g, 0, pyq, sc->rc, sc->rs, -1.f);
      rotate(g, 1, pxq, sc->rc, sc->rs, -1.f);
    }
    if (row_ok) store_grad<TG>(static_cast<TG*>(p.dq) + tok_off(p, b, rc.Y(tq), rc.X(tq), h), g);
  }
  if (MODE == 1 && p.acc_tau) warp_add(dtau, &sc->red[0]);
  if (MODE == 2 && p.acc_rope)
#pragma unroll
    for (int e = 0; e < 16; ++e) warp_add(drope[e], &sc->red[1 + e]);
  ptx::tc_fence_before();
  __syncthreads();
  if (want_T)
    for (int i = tid; i < RR; i += kThreads)
      if (dtab[i] != 0.0) atomicAdd(p.acc_table + (size_t)i * p.heads + h, dtab[i]);
  if (MODE == 1 && p.acc_tau && tid == 0) atomicAdd(p.acc_tau + h, sc->red[0]);
  if (MODE == 2 && p.acc_rope && tid < 16) atomicAdd(p.acc_rope + tid, sc->red[1 + tid]);
  if (tid == 0 && sc->range_hit) atomicOr(p.status, (int)SWIN_ERR_UNSUPPORTED);
  if (warp == 0) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tbase, 256);
  }
}

// ============================================================== key kernel
template <int MODE, bool TABLE, typename TG>
__global__ void __launch_bounds__(kThreads) bwd_tc_kv(const __grid_constant__ TcBwd p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* ks = smem;          // K tile, fp16 (128 rows)
  uint8_t* vs = ks + kTileB;   // V tile, fp16
  uint8_t* klo = vs + kTileB;  // mode 2: lo parts of the rotated K tile
  uint8_t* qgb = klo + kTileB; // two buffers of [Q block | dO block | Q lo parts] (64 rows each)
  SmemCommon* sc = reinterpret_cast<SmemCommon*>(qgb + 2 * 3 * kBlkB);
  float* tab = reinterpret_cast<float*>(sc + 1);
  const int R = 2 * p.M - 1, RR = R * R;

  const int rect = blockIdx.x / p.tiles, tile = blockIdx.x % p.tiles;
  const int h = blockIdx.y, b = blockIdx.z;
  const Rect rc = rect_of(p, rect);
  const int t0 = tile * kRows;
  if (t0 >= rc.n) return;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int tk = t0 + tid;
  const bool row_ok = tk < rc.n;

  if (tid == 0) {
    ptx::mbar_init(&sc->mma_bar, 1);
    ptx::fence_mbar_init();
    sc->range_hit = 0;
  }
  if (warp == 0) {
    ptx::tmem_alloc(&sc->tmem_base, 256);
    ptx::tmem_relinquish();
  }
  for (int i = tid; i < 17; i += kThreads) sc->red[i] = 0.0;
  if (MODE == 2) build_rope(p.rope, p.M, sc->rc, sc->rs);
  if (TABLE)
    for (int i = tid; i < RR; i += kThreads) tab[i] = __ldg(p.table + (size_t)i * p.heads + h) * kLog2e;
  __syncthreads();

  const float t_eff = MODE == 1 ? fmaxf(__ldg(p.tau + h), kTauMin) : 1.f;
  float krow[kD];
  bool kclamped = false;
  float kn = 1.f;
  const int pyk = row_ok ? rc.PY(tk) : 0, pxk = row_ok ? rc.PX(tk) : 0;
  {
    bool hit = false;
    if (row_ok) {
      const size_t off = tok_off(p, b, rc.Y(tk), rc.X(tk), h);
      float vrow[kD];
      load_row(p.k + off, krow);
      load_row(p.v + off, vrow);
      if (MODE == 1) kn = clamped_norm(krow, kclamped);
      prep_row<MODE>(krow, pyk, pxk, sc->rc, sc->rs);
      hit |= MODE == 2 ? store_row_f16_split(ks, klo, tid, krow) : store_row_f16(ks, tid, krow);
      hit |= store_row_f16(vs, tid, vrow);
    } else {
#pragma unroll
      for (int e = 0; e < kD; ++e) krow[e] = 0.f;
      zero_row(ks, tid);
      zero_row(vs, tid);
      if (MODE == 2) zero_row(klo, tid);
    }
    if (hit) sc->range_hit = 1;
  }
  const float bcol = MODE == 1 ? 1.f / kn : 0.f;  // this key's 1/|k|
  const float srow = MODE == 1 ? kLog2e * bcol : kLog2e * rsqrtf((float)kD);
  const float dscale = MODE == 1 ? 1.f : rsqrtf((float)kD);
  // table row of the pair (query i, this key) = coff[i] - kbase
  const int kbase = rc.off(row_ok ? tk : t0, R) - (p.M - 1) * (R + 1);

  ptx::fence_proxy_async_smem();
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tbase = sc->tmem_base;
  const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
  const uint32_t tS = tbase, tP = tbase + 64, tPT = tbase + 128, tDS = tbase + 160, tDV = tbase + 192,
                 tDK = tbase + 224;
  constexpr uint32_t idS = ptx::idesc_f16(0, 0, 0, 0, kBlk, kRows);
  constexpr uint32_t idAcc = ptx::idesc_f16(0, 0, 0, 1, kD, kRows);
  const uint64_t kd = ptx::smem_desc(ptx::smem_addr(ks), 16, 512, ptx::kSwizzle64B);
  const uint64_t vd = ptx::smem_desc(ptx::smem_addr(vs), 16, 512, ptx::kSwizzle64B);
  const uint64_t kld = ptx::smem_desc(ptx::smem_addr(klo), 16, 512, ptx::kSwizzle64B);
  auto qbuf = [&](int x) { return qgb + 3 * x * kBlkB; };
  auto qdesc = [&](int x, int part) {
    return ptx::smem_desc(ptx::smem_addr(qbuf(x) + part * kBlkB), 16, 512, ptx::kSwizzle64B);
  };
  uint32_t phase = 0;
  bool ok = true;

  const int nqb = (rc.n + kBlk - 1) / kBlk;
  // Threads 0-63 carry Q rows (and their statistics) of a query block, 64-127
  // dO rows; block qb + 1 is fetched while qb computes and stored once its
  // buffer is free (the wait on S^T / dP^T of qb covers the dV / dK MMAs of
  // qb - 1, that buffer's last readers).
  const int lr = tid & (kBlk - 1);
  const bool isq = tid < kBlk;
  RawRow pre;
  double2 pst = make_double2(0.0, 0.0);
  auto fetch = [&](int qb) {
    const int tq = qb * kBlk + lr;
    if (tq < rc.n) {
      const size_t off = tok_off(p, b, rc.Y(tq), rc.X(tq), h);
      fetch_row((isq ? p.q : p.dout) + off, pre);
      if (isq) pst = p.stats[(((size_t)b * p.H + rc.Y(tq)) * p.W + rc.X(tq)) * p.heads + h];
    }
  };
  auto stash = [&](int qb) {
    const int x = qb & 1, tq = qb * kBlk + lr;
    uint8_t* qt = qbuf(x);
    bool hit = false;
    if (isq) sc->coff[x][lr] = rc.off(min(tq, rc.n - 1), R);
    if (tq < rc.n) {
      float v[kD];
      unpack_row(pre, v);
      if (isq) {
        if (MODE == 1) {
          bool c;
          sc->colf[x][lr] = 1.f / (clamped_norm(v, c) * t_eff);
        }
        prep_row<MODE>(v, rc.PY(tq), rc.PX(tq), sc->rc, sc->rs);
        hit = MODE == 2 ? store_row_f16_split(qt, qt + 2 * kBlkB, lr, v) : store_row_f16(qt, lr, v);
        sc->lse2[x][lr] = (float)pst.x;
        sc->dsum[x][lr] = (float)pst.y;
      } else {
        hit = store_row_f16(qt + kBlkB, lr, v);
      }
    } else {
      zero_row(isq ? qt : qt + kBlkB, lr);
      if (isq && MODE == 2) zero_row(qt + 2 * kBlkB, lr);
      if (isq) {
        sc->colf[x][lr] = 0.f;
        sc->lse2[x][lr] = INFINITY;  // exp2(x - inf) = 0: no weight for padding columns
        sc->dsum[x][lr] = 0.f;
      }
    }
    if (hit) sc->range_hit = 1;
  };
  fetch(0);
  stash(0);
  ptx::fence_proxy_async_smem();
  ptx::tc_fence_before();
  __syncthreads();
  for (int qb = 0; qb < nqb && ok; ++qb) {
    const int x = qb & 1;
    const uint64_t qd = qdesc(x, 0), gd = qdesc(x, 1), qld = qdesc(x, 2);
    // ---- S^T = K Q^T, dP^T = V dO^T (the commit also covers the previous dV / dK MMAs)
    if (tid == 0) {
      ptx::tc_fence_after();
      ptx::mma_ss(tS, kd, qd, idS, 0);
      ptx::mma_ss(tS, kd + 2, qd + 2, idS, 1);
      if (MODE == 2) {  // + K_lo Q_hi^T + K_hi Q_lo^T
        ptx::mma_ss(tS, kld, qd, idS, 1);
        ptx::mma_ss(tS, kld + 2, qd + 2, idS, 1);
        ptx::mma_ss(tS, kd, qld, idS, 1);
        ptx::mma_ss(tS, kd + 2, qld + 2, idS, 1);
      }
      ptx::mma_ss(tP, vd, gd, idS, 0);
      ptx::mma_ss(tP, vd + 2, gd + 2, idS, 1);
      ptx::mma_commit(&sc->mma_bar);
    }
    if (qb + 1 < nqb) fetch(qb + 1);  // in flight during the MMAs and the softmax
    ok = wait_mma(&sc->mma_bar, phase, p.status);
    phase ^= 1;
    if (!ok) break;
    ptx::tc_fence_after();
    const float* colf = sc->colf[x];
    const int* coff = sc->coff[x];
    const float* lse2 = sc->lse2[x];
    const float* dsum = sc->dsum[x];
    // the block's 64 queries in two halves of 32
    for (int hf = 0; hf < 2; ++hf) {
      uint32_t sr[32], dr[32];
      ptx::tmem_ld32(tS + 32 * hf + lane_off, sr);
      ptx::tmem_ld32(tP + 32 * hf + lane_off, dr);
      ptx::tmem_wait_ld();
      uint32_t pk[16], dk[16];
#pragma unroll
      for (int i = 0; i < 32; i += 2) {
        float pv[2], dsv[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int ii = 32 * hf + i + e;
          const float sv = __uint_as_float(sr[i + e]);
          float xv = MODE == 1 ? sv * srow * colf[ii] : sv * srow;
          SWIN_DCHECK(p.status, !TABLE || (coff[ii] - kbase >= 0 && coff[ii] - kbase < RR));
          if (TABLE) xv += tab[coff[ii] - kbase];
          const float pj = row_ok ? ptx::ex2_approx(xv - lse2[ii]) : 0.f;
          const float dl = pj * (__uint_as_float(dr[i + e]) - dsum[ii]);
          pv[e] = pj;
          dsv[e] = MODE == 1 ? dl * colf[ii] : dl * dscale;
        }
        if (fabsf(dsv[0]) >= 65504.f || fabsf(dsv[1]) >= 65504.f) sc->range_hit = 1;
        pk[i / 2] = ptx::pack_f16x2(pv[0], pv[1]);
        dk[i / 2] = ptx::pack_f16x2_sat(dsv[0], dsv[1]);
      }
      ptx::tmem_st16(tPT + 16 * hf + lane_off, pk);
      ptx::tmem_st16(tDS + 16 * hf + lane_off, dk);
    }
    ptx::tmem_wait_st();
    ptx::tc_fence_before();
    __syncthreads();
    // ---- dV += P^T dO, dK += dS^T Q (B operands MN-major [queries x d]); not
    // waited for here: the next block's S^T / dP^T commit covers them
    if (tid == 0) {
      ptx::tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < kBlk / 16; ++kk) {
        const uint32_t acc = (qb > 0 || kk > 0) ? 1u : 0u;
        ptx::mma_ts(tDV, tPT + kk * 8, gd + (uint64_t)(kk * 1024 >> 4), idAcc, acc);
        ptx::mma_ts(tDK, tDS + kk * 8, qd + (uint64_t)(kk * 1024 >> 4), idAcc, acc);
        if (MODE == 2) ptx::mma_ts(tDK, tDS + kk * 8, qld + (uint64_t)(kk * 1024 >> 4), idAcc, 1u);
      }
    }
    if (qb + 1 < nqb) stash(qb + 1);
    ptx::fence_proxy_async_smem();
    ptx::tc_fence_before();
    __syncthreads();
  }
  // the last dV / dK MMAs
  if (ok) {
    if (tid == 0) {
      ptx::tc_fence_after();
      ptx::mma_commit(&sc->mma_bar);
    }
    ok = wait_mma(&sc->mma_bar, phase, p.status);
    phase ^= 1;
  }

  float drope[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) drope[e] = 0.f;
  if (ok) {
    ptx::tc_fence_after();
    uint32_t av[32], ak[32];
    ptx::tmem_ld32(tDV + lane_off, av);
    ptx::tmem_ld32(tDK + lane_off, ak);
    ptx::tmem_wait_ld();
    float gv[kD], gk[kD];
#pragma unroll
    for (int e = 0; e < kD; ++e) {
      gv[e] = __uint_as_float(av[e]);
      gk[e] = __uint_as_float(ak[e]);
    }
    if (MODE == 1) {
      // k~ = b k, dk~ = gk; dk = (gk - (k~ . gk) k~) b
      float kd2 = 0.f;
#pragma unroll
      for (int e = 0; e < kD; ++e) kd2 = fmaf(krow[e] * bcol, gk[e], kd2);
      const float kk2 = kclamped ? 0.f : kd2;
#pragma unroll
      for (int e = 0; e < kD; ++e) gk[e] = (gk[e] - kk2 * krow[e] * bcol) * bcol;
    } else if (MODE == 2) {
      if (row_ok) rope_grad(krow, gk, pyk, pxk, drope);
      rotate(gk, 0, pyk, sc->rc, sc->rs, -1.f);
      rotate(gk, 1, pxk, sc->rc, sc->rs, -1.f);
    }
    if (row_ok) {
      const size_t off = tok_off(p, b, rc.Y(tk), rc.X(tk), h);
      store_grad<TG>(static_cast<TG*>(p.dk) + off, gk);
      store_grad<TG>(static_cast<TG*>(p.dv) + off, gv);
    }
  }
  if (MODE == 2 && p.acc_rope)
#pragma unroll
    for (int e = 0; e < 16; ++e) warp_add(drope[e], &sc->red[1 + e]);
  ptx::tc_fence_before();
  __syncthreads();
  if (MODE == 2 && p.acc_rope && tid < 16) atomicAdd(p.acc_rope + tid, sc->red[1 + tid]);
  if (tid == 0 && sc->range_hit) atomicOr(p.status, (int)SWIN_ERR_UNSUPPORTED);
  if (warp == 0) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tbase, 256);
  }
}

// ============================================================== forward
// The forward pass over arbitrary rectangles (interleaved windows, whose
// strided windows the TMA kernel does not gather, and windows of at most 64
// tokens): persistent CTAs, each walking work items (one query tile of one
// rectangle of one (image, head); heads outermost, so the bias table of a
// head is loaded once for several items).  Per item: the Q rows and the first
// K / V block's rows are loaded together, then S = Q K^T per 64-key block
// (RoPE operands split into fp16 hi + lo as in the backward), the softmax in
// fp32 with the running maximum kept until a block exceeds it by more than 8
// (log2 units; probabilities then <= 2^8, exact in fp16's range), P as fp16
// into TMEM and O += P V on the tensor cores.  The row sum is taken from the
// same fp16 probabilities that weight V, so O / l normalises exactly the
// weights applied.  128 TMEM columns (S 64, P 32, O 32) per CTA, allocated
// once.
template <int MODE, bool TABLE, typename TO>
__global__ void __launch_bounds__(kThreads, 4) fwd_tc_rect(const __grid_constant__ TcBwd p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* qs = smem;
  uint8_t* ks = qs + kTileB;
  uint8_t* vs = ks + kBlkB;
  uint8_t* qlo = vs + kBlkB;
  uint8_t* klo = qlo + kTileB;
  SmemCommon* sc = reinterpret_cast<SmemCommon*>(klo + kBlkB);
  float* tab = reinterpret_cast<float*>(sc + 1);
  const int R = 2 * p.M - 1, RR = R * R;
  const int tid = threadIdx.x, warp = tid >> 5;

  if (tid == 0) {
    ptx::mbar_init(&sc->mma_bar, 1);
    ptx::fence_mbar_init();
    sc->range_hit = 0;
  }
  if (warp == 0) {
    ptx::tmem_alloc(&sc->tmem_base, 128);
    ptx::tmem_relinquish();
  }
  if (MODE == 2) build_rope(p.rope, p.M, sc->rc, sc->rs);
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tbase = sc->tmem_base;
  const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
  const uint32_t tS = tbase, tP = tbase + 64, tO = tbase + 96;
  constexpr uint32_t idS = ptx::idesc_f16(0, 0, 0, 0, kBlk, kRows);
  constexpr uint32_t idO = ptx::idesc_f16(0, 0, 0, 1, kD, kRows);
  const uint64_t qd = ptx::smem_desc(ptx::smem_addr(qs), 16, 512, ptx::kSwizzle64B);
  const uint64_t kd = ptx::smem_desc(ptx::smem_addr(ks), 16, 512, ptx::kSwizzle64B);
  const uint64_t vd = ptx::smem_desc(ptx::smem_addr(vs), 16, 512, ptx::kSwizzle64B);
  const uint64_t qld = ptx::smem_desc(ptx::smem_addr(qlo), 16, 512, ptx::kSwizzle64B);
  const uint64_t kld = ptx::smem_desc(ptx::smem_addr(klo), 16, 512, ptx::kSwizzle64B);
  const int nrect = swin_nwin(p.part, p.H, p.M, p.shift) * p.nsx;
  const long long n_items = (long long)nrect * p.tiles * p.heads * p.B;
  uint32_t phase = 0;
  bool ok = true;
  int cur_h = -1;

  for (long long it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
    const int tile = (int)(it % p.tiles);
    long long rest = it / p.tiles;
    const int rect = (int)(rest % nrect);
    rest /= nrect;
    const int b = (int)(rest % p.B), h = (int)(rest / p.B);
    const Rect rc = rect_of(p, rect);
    const int t0 = tile * kRows;
    if (t0 >= rc.n) continue;  // uniform: the rectangle has fewer tiles
    const int tq = t0 + tid;
    const bool row_ok = tq < rc.n;
    // this thread's rows of the item, loaded together: its Q row and its K
    // (threads 0-63) or V (64-127) row of the first block
    const int kr = tid & (kBlk - 1);
    const bool isk = tid < kBlk;
    uint4 qraw[4], kvraw[4];
    if (row_ok) load_raw(p.q + tok_off(p, b, rc.Y(tq), rc.X(tq), h), qraw);
    if (kr < rc.n) load_raw((isk ? p.k : p.v) + tok_off(p, b, rc.Y(kr), rc.X(kr), h), kvraw);
    if (TABLE && h != cur_h) {  // uniform: every thread walks the same items
      for (int i = tid; i < RR; i += kThreads) tab[i] = __ldg(p.table + (size_t)i * p.heads + h) * kLog2e;
      cur_h = h;
      __syncthreads();
    }

    const float t_eff = MODE == 1 ? fmaxf(__ldg(p.tau + h), kTauMin) : 1.f;
    float qn = 1.f;
    {
      bool hit = false;
      if (row_ok) {
        float qrow[kD];
        unpack_row(qraw, qrow);
        bool c;
        if (MODE == 1) qn = clamped_norm(qrow, c);
        prep_row<MODE>(qrow, rc.PY(tq), rc.PX(tq), sc->rc, sc->rs);
        hit = MODE == 2 ? store_row_f16_split(qs, qlo, tid, qrow) : store_row_f16(qs, tid, qrow);
      } else {
        zero_row(qs, tid);
        if (MODE == 2) zero_row(qlo, tid);
      }
      if (hit) sc->range_hit = 1;
    }
    const float srow = MODE == 1 ? kLog2e / (qn * t_eff) : kLog2e * rsqrtf((float)kD);
    const int qbase = rc.off(row_ok ? tq : t0, R) + (p.M - 1) * (R + 1);

    float m2 = -INFINITY, l = 0.f;
    const int nkb = (rc.n + kBlk - 1) / kBlk;
    for (int kb = 0; kb < nkb && ok; ++kb) {
      const int k0 = kb * kBlk, nk = min(kBlk, rc.n - k0);
      {
        const int tk = k0 + kr;
        if (isk) sc->coff[0][kr] = rc.off(min(tk, rc.n - 1), R);
        bool hit = false;
        if (kr < nk) {
          float v[kD];
          if (kb == 0) {
            unpack_row(kvraw, v);
          } else {
            const size_t off = tok_off(p, b, rc.Y(tk), rc.X(tk), h);
            load_row((isk ? p.k : p.v) + off, v);
          }
          if (isk) {
            if (MODE == 1) {
              bool c;
              sc->colf[0][kr] = 1.f / clamped_norm(v, c);
            }
            prep_row<MODE>(v, rc.PY(tk), rc.PX(tk), sc->rc, sc->rs);
            hit = MODE == 2 ? store_row_f16_split(ks, klo, kr, v) : store_row_f16(ks, kr, v);
          } else {
            hit = store_row_f16(vs, kr, v);
          }
        } else {
          zero_row(isk ? ks : vs, kr);
          if (isk && MODE == 2) zero_row(klo, kr);
          if (isk && MODE == 1) sc->colf[0][kr] = 0.f;
        }
        if (hit) sc->range_hit = 1;
      }
      ptx::fence_proxy_async_smem();
      ptx::tc_fence_before();
      __syncthreads();
      if (tid == 0) {
        ptx::tc_fence_after();
        ptx::mma_ss(tS, qd, kd, idS, 0);
        ptx::mma_ss(tS, qd + 2, kd + 2, idS, 1);
        if (MODE == 2) {
          ptx::mma_ss(tS, qld, kd, idS, 1);
          ptx::mma_ss(tS, qld + 2, kd + 2, idS, 1);
          ptx::mma_ss(tS, qd, kld, idS, 1);
          ptx::mma_ss(tS, qd + 2, kld + 2, idS, 1);
        }
        ptx::mma_commit(&sc->mma_bar);
      }
      ok = wait_mma(&sc->mma_bar, phase, p.status);
      phase ^= 1;
      if (!ok) break;
      ptx::tc_fence_after();
      uint32_t sr[2][32];
      ptx::tmem_ld32(tS + lane_off, sr[0]);
      ptx::tmem_ld32(tS + 32 + lane_off, sr[1]);
      ptx::tmem_wait_ld();
      // log2-domain logits, formed once (the score registers are reused)
      float xl[kBlk];
      float mb = -INFINITY;
#pragma unroll
      for (int jj = 0; jj < kBlk; ++jj) {
        const float sv = __uint_as_float(sr[jj >> 5][jj & 31]);
        float xv = MODE == 1 ? sv * srow * sc->colf[0][jj] : sv * srow;
        if (TABLE) xv += tab[qbase - sc->coff[0][jj]];
        xl[jj] = jj < nk ? xv : -INFINITY;
        mb = fmaxf(mb, xl[jj]);
      }
      // lazy maximum: raised only when this block exceeds it by more than 8
      float c = 1.f;
      if (mb > m2 + 8.f) {
        c = ptx::ex2_approx(m2 - mb);  // 0 at the first block
        m2 = mb;
        l *= c;
      }
      if (kb > 0 && __any_sync(0xffffffffu, c != 1.f)) {  // rescale O (the previous PV has completed)
        uint32_t o[32];
        ptx::tmem_ld32(tO + lane_off, o);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * c);
        ptx::tmem_st32(tO + lane_off, o);
      }
      uint32_t pk[32];
#pragma unroll
      for (int jj = 0; jj < kBlk; jj += 2) {
        const uint32_t w2 = ptx::pack_f16x2(ptx::ex2_approx(xl[jj] - m2), ptx::ex2_approx(xl[jj + 1] - m2));
        const __half2 hp = *reinterpret_cast<const __half2*>(&w2);
        l += __low2float(hp) + __high2float(hp);  // the weights V receives
        pk[jj / 2] = w2;
      }
      ptx::tmem_st32(tP + lane_off, pk);
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      __syncthreads();
      if (tid == 0) {
        ptx::tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kBlk / 16; ++kk)
          ptx::mma_ts(tO, tP + kk * 8, vd + (uint64_t)(kk * 1024 >> 4), idO, (kb > 0 || kk > 0) ? 1u : 0u);
        ptx::mma_commit(&sc->mma_bar);
      }
      ok = wait_mma(&sc->mma_bar, phase, p.status);
      phase ^= 1;
      ptx::tc_fence_before();
      __syncthreads();
    }
    if (!ok) break;
    ptx::tc_fence_after();
    uint32_t o[32];
    ptx::tmem_ld32(tO + lane_off, o);
    ptx::tmem_wait_ld();
    const float inv = 1.f / l;
    float g[kD];
#pragma unroll
    for (int e = 0; e < kD; ++e) g[e] = __uint_as_float(o[e]) * inv;
    if (row_ok) store_grad<TO>(static_cast<TO*>(p.out) + tok_off(p, b, rc.Y(tq), rc.X(tq), h), g);
    // the next item's first PV overwrites O: every thread has read it
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (tid == 0 && sc->range_hit) atomicOr(p.status, (int)SWIN_ERR_UNSUPPORTED);
  if (warp == 0) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tbase, 128);
  }
}

size_t smem_q(int M, bool table) {
  const int RR = (2 * M - 1) * (2 * M - 1);
  size_t s = 3 * kTileB + 6 * kBlkB + sizeof(SmemCommon);
  if (table) s += sizeof(float) * ((RR + 1) & ~1) + sizeof(double) * RR;
  return s;
}

size_t smem_kv(int M, bool table) {
  const int RR = (2 * M - 1) * (2 * M - 1);
  return 3 * kTileB + 6 * kBlkB + sizeof(SmemCommon) + (table ? sizeof(float) * RR : 0);
}

template <int MODE, bool TABLE, typename TG>
swin_status launch_tc(const TcBwd& p, cudaStream_t stream) {
  const int nsy = swin_nwin(p.part, p.H, p.M, p.shift);
  const dim3 grid(nsy * p.nsx * p.tiles, p.heads, p.B);
  auto kq = bwd_tc_q<MODE, TABLE, TG>;
  auto kkv = bwd_tc_kv<MODE, TABLE, TG>;
  // each CTA holds 256 TMEM columns, so two fit on an SM: shared memory of at
  // least 80 KB keeps a third from becoming resident and waiting in its
  // allocation
  constexpr size_t kMinSmem = 80 * 1024;
  const size_t sq = std::max(smem_q(p.M, TABLE), kMinSmem), skv = std::max(smem_kv(p.M, TABLE), kMinSmem);
  cudaError_t e = cudaFuncSetAttribute(kq, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sq);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(kkv, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)skv);
  if (e != cudaSuccess) return fail(SWIN_ERR_CUDA, "attn_bwd_tc smem attribute: %s", cudaGetErrorString(e));
  kq<<<grid, kThreads, sq, stream>>>(p);
  kkv<<<grid, kThreads, skv, stream>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return fail(SWIN_ERR_CUDA, "attn_bwd_tc launch: %s", cudaGetErrorString(e));
  return SWIN_OK;
}

template <typename TG>
swin_status launch_tg(const TcBwd& p, int mode, bool table, cudaStream_t stream) {
  switch (mode) {
    case 0: return table ? launch_tc<0, true, TG>(p, stream) : launch_tc<0, false, TG>(p, stream);
    case 1: return table ? launch_tc<1, true, TG>(p, stream) : launch_tc<1, false, TG>(p, stream);
    default: return launch_tc<2, false, TG>(p, stream);
  }
}

template <int MODE, bool TABLE, typename TO>
swin_status launch_fwd_rect(const TcBwd& p, cudaStream_t stream) {
  const long long items = (long long)swin_nwin(p.part, p.H, p.M, p.shift) * p.nsx * p.tiles * p.heads * p.B;
  if (items == 0) return SWIN_OK;
  auto kf = fwd_tc_rect<MODE, TABLE, TO>;
  const int RR = (2 * p.M - 1) * (2 * p.M - 1);
  // 128 TMEM columns per CTA: at most four CTAs per SM, which 50 KB of shared
  // memory or more ensures (a fifth would wait in its TMEM allocation)
  const size_t sm = std::max<size_t>(2 * kTileB + 3 * kBlkB + sizeof(SmemCommon) + (TABLE ? sizeof(float) * RR : 0),
                                     50 * 1024);
  cudaError_t e = cudaFuncSetAttribute(kf, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  // the occupancy below (and at launch) assumes the largest shared-memory carveout
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(kf, cudaFuncAttributePreferredSharedMemoryCarveout, (int)cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return fail(SWIN_ERR_CUDA, "attn_fwd_rect smem attribute: %s", cudaGetErrorString(e));
  // persistent: four CTAs per SM, all resident at once (128 registers and at
  // most ~56 KB of shared memory each)
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = (int)std::min<long long>(items, 4LL * sms);
  kf<<<grid, kThreads, sm, stream>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return fail(SWIN_ERR_CUDA, "attn_fwd_rect launch: %s", cudaGetErrorString(e));
  return SWIN_OK;
}

template <typename TO>
swin_status launch_fwd_to(const TcBwd& p, int mode, bool table, cudaStream_t stream) {
  switch (mode) {
    case 0: return table ? launch_fwd_rect<0, true, TO>(p, stream) : launch_fwd_rect<0, false, TO>(p, stream);
    case 1: return table ? launch_fwd_rect<1, true, TO>(p, stream) : launch_fwd_rect<1, false, TO>(p, stream);
    default: return launch_fwd_rect<2, false, TO>(p, stream);
  }
}

}  // namespace

swin_status launch_attn_fwd_tc_rect(const AttnArgs& a, bool f32_out, cudaStream_t stream) {
  if (a.d != kD || a.M > 32) return fail(SWIN_ERR_UNSUPPORTED, "rectangle tensor-core path: d = 32, M <= 32");
  TcBwd p = {};
  p.q = static_cast<const __nv_bfloat16*>(a.q);
  p.k = static_cast<const __nv_bfloat16*>(a.k);
  p.v = static_cast<const __nv_bfloat16*>(a.v);
  p.out = a.out;
  p.B = a.B;
  p.H = a.H;
  p.W = a.W;
  p.heads = a.heads;
  p.M = a.M;
  p.shift = a.shift;
  p.part = a.part;
  p.tau = a.tau;
  p.table = a.mode == 2 ? nullptr : a.table;
  p.rope = a.rope;
  p.status = a.status;
  p.nsx = swin_nwin(a.part, a.W, a.M, a.shift);
  p.tiles = (a.M * a.M + kRows - 1) / kRows;
  const bool table = p.table != nullptr;
  return f32_out ? launch_fwd_to<float>(p, a.mode, table, stream)
                 : launch_fwd_to<__nv_bfloat16>(p, a.mode, table, stream);
}

bool attn_bwd_tc_supported(const BwdArgs& a, bool bf16_in) {
  return bf16_in && a.d == kD && a.M <= 32;
}

swin_status launch_attn_bwd_tc(const BwdArgs& a, bool f32_grad, cudaStream_t stream) {
  TcBwd p = {};
  p.q = static_cast<const __nv_bfloat16*>(a.q);
  p.k = static_cast<const __nv_bfloat16*>(a.k);
  p.v = static_cast<const __nv_bfloat16*>(a.v);
  p.dout = static_cast<const __nv_bfloat16*>(a.dout);
  p.dq = a.dq;
  p.dk = a.dk;
  p.dv = a.dv;
  p.B = a.B;
  p.H = a.H;
  p.W = a.W;
  p.heads = a.heads;
  p.M = a.M;
  p.shift = a.shift;
  p.part = a.part;
  p.tau = a.tau;
  p.table = a.mode == 2 ? nullptr : a.table;
  p.rope = a.rope;
  p.acc_table = a.acc_table;
  p.acc_tau = a.acc_tau;
  p.acc_rope = a.acc_rope;
  p.stats = a.stats;
  p.status = a.status;
  p.nsx = swin_nwin(a.part, a.W, a.M, a.shift);
  p.tiles = (a.M * a.M + kRows - 1) / kRows;
  const bool table = p.table != nullptr;
  return f32_grad ? launch_tg<float>(p, a.mode, table, stream) : launch_tg<__nv_bfloat16>(p, a.mode, table, stream);
}

}  // namespace swin
