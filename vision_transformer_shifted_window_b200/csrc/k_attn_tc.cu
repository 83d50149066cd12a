// Shifted-window attention on the Blackwell tensor cores (bf16 inputs, d = 32).
//
// What is computed: for every rectangle (one segment of the shifted partition
// per axis, see swin_index.cuh) of every (image, head), exact softmax attention
// over the rectangle's tokens with the score of the chosen mode —
//   mode 0  q.k/sqrt(d) + T[r][h]        "Swin Transformer V2" eq. 1
//   mode 1  cos(q,k)/max(tau,0.01) + T   same page, eq. 2 (§3.2, §3.3)
//   mode 2  RoPE(q).RoPE(k)/sqrt(d)      FlashSwin abstract (window-local 2-D RoPE)
// — without ever storing a score matrix: FlashSwin's point is that the
// per-window score matrix is the memory problem; here S lives only in TMEM.
//
// Work unit: two consecutive query tiles (tile = floor(128 / lx) whole
// rectangle rows) of one row of rectangles, one per softmax warpgroup.  Tiles
// of one rectangle share its K/V blocks of floor(96 / lx) rectangle rows (at
// most 96 keys); tiles of two rectangles stream both rectangles' blocks.
//
// Warp roles (512 threads, one persistent CTA per SM):
//   warp 0      TMA producer: Q tiles and K/V blocks, 5-D tensor maps over
//               [B][H][W][heads][d] with 64-byte swizzle, no multicast
//   warps 1, 2  tcgen05.mma issuers, one thread each: warp 1 + g issues the
//               MMAs of softmax warpgroup g; warp 1 owns TMEM
//   warps 3, 12-15  operand prep in shared memory, one row per thread: K
//               unit-normalisation (mode 1), RoPE rotation of Q and K
//               (mode 2), per-row 1/(tau |q|) (mode 1), V to fp16
//   warps 4-7   softmax of warpgroup 0 (one TMEM lane = one query row)
//   warps 8-11  softmax of warpgroup 1
// TMEM per softmax warpgroup g (128 lanes): two score buffers X0, X1 of 96
// fp32 columns and O (48 columns: 32 outputs and, in column 32, the row sum
// of P).  Block b's scores S = Q K^T land in X[b % 2]; the softmax turns them
// into fp16 probabilities P written over the same columns, and O += P [V | c]
// (6 MMAs, N = 48, A from TMEM) reads them there.  With two buffers the
// softmax never waits for the previous block's PV; a thread's MMAs execute
// in issue order, so S(b+2) cannot overwrite P(b) before PV(b) has read it.
//
// Softmax: online, with the running maximum kept until a block exceeds it by
// more than 8 (log2 units), so O is rescaled rarely; P in fp16 (values up to
// 2^8) keeps that accurate: bf16 P, which would spare the V conversion, leaves
// errors of 2.6 % of the output RMS on sharp cosine attention.  V is converted
// to fp16 by the prep warps; the constant column c = 1 of [V | c] makes the
// same MMAs accumulate the row sum of the fp16 P, so O / l uses exactly the
// probabilities that weighted V.  V entries of magnitude 65504 or more
// saturate and record SWIN_ERR_UNSUPPORTED in the status word.
//
// Precision of the score operands: mode 0 multiplies the bf16 inputs as they
// are; mode 1 also multiplies the raw inputs and applies 1/|q| (per row),
// 1/|k| (per column) and 1/tau in fp32 afterwards, so the cosine is not
// rounded; mode 2 rotates q and k in fp32 and stores them as fp16 (scaled by
// powers of two so that no finite input overflows), the largest error term.
//
// Every wait is bounded: on time-out the kernel records SWIN_ERR_TIMEOUT in
// the status word, every role leaves its loop, in-flight copies and MMAs are
// drained with bounded waits, TMEM is freed and the kernel returns.
#include <cuda.h>
#include <cuda_fp16.h>

#include <cstring>

#include "sm100_ptx.cuh"
#include "swin_common.cuh"
#include "tma_encode.cuh"

// Phase markers for external timing builds; they compile to nothing here.
#ifndef SWIN_TC_MARK
#define SWIN_TC_MARK(k)
#endif

namespace swin {

// Division by a launch constant with a multiply and a shift (Granlund and
// Montgomery's method): n / d = (umulhi(m, n) + n) >> l for n < 2^31, with
// l = ceil(log2 d) and m = floor(2^32 (2^l - d) / d) + 1.
struct FastDiv {
  uint32_t d, m, l;
};

inline FastDiv make_fastdiv(uint32_t d) {
  FastDiv f;
  f.d = d;
  f.l = 0;
  while ((1ull << f.l) < d) ++f.l;
  f.m = (uint32_t)(((1ull << 32) * ((1ull << f.l) - d)) / d + 1);
  return f;
}

__device__ __forceinline__ uint32_t fdiv(uint32_t n, const FastDiv& f) {
  return (__umulhi(f.m, n) + n) >> f.l;
}

struct TcParams {
  CUtensorMap tmap[3][3];  // [tensor q/k/v][x-class first/middle/last]
  FastDiv div_ipb, div_B, div_mid_items, div_mid_tiles[3];
  FastDiv div_hb;  // B * heads
  int pos_major;   // walk items position-major (see decode)
  int lx[3], R[3], Rk[3];  // per x-class: segment width, rows per query tile, rows per K/V block
  // per row class (first, middle, last row of rectangles): height, items,
  // and per x-class the query tiles and K/V blocks of one rectangle
  int row_ly[3], row_items[3], row_tiles[3][3], row_nb[3][3];
  void* out;
  int B, H, W, heads, M, s, nsy, nsx;
  int R2e;  // row stride of the bias slot (even, >= 2M - 1, chosen against bank conflicts)
  long long n_items;
  const float* tau;
  const float* table;
  const float* rope;
  int* status;
  long long wait_limit;  // clock64 cycles before a wait gives up
  int debug_flags;       // bit 0: force a time-out (test of the failure path)
};

namespace {

constexpr int kThreads = 512;
constexpr int kPrepThreads = 160;  // warps 3 and 12-15
constexpr int kStages = 6;                  // K/V ring
constexpr int kTileBytes = 128 * 64;        // 128 rows x 32 16-bit values
constexpr int kBlk = 96;                    // keys per K/V block (TMEM: 2 x 96 + 48 columns per warpgroup)
constexpr int kQOff = 0;                    // [2 wg][2 buf] Q tiles
constexpr int kKVOff = kQOff + 4 * kTileBytes;
constexpr int kOnesOff = kKVOff + kStages * 2 * kTileBytes;   // per stage: 16 rows of [c, 0...] (1 KB)
constexpr int kScaleOff = kOnesOff + kStages * 1024;         // [2][2][128] f32
constexpr int kRopeOff = kScaleOff + 2 * 2 * 128 * 4;        // cos,sin [2][64][8] f32
constexpr int kKofsOff = kRopeOff + 2 * 2 * 64 * 8 * 4;      // [3][128] int
constexpr int kRposOff = kKofsOff + 3 * 128 * 4;             // [3][128] int: (r / lx) | (r % lx) << 16
constexpr int kKcolOff = kRposOff + 3 * 128 * 4;             // [kStages][128] f32, 1/|k| (mode 1)
// Relative-bias table of the current head, one slot per softmax warpgroup:
// rows dy padded to an even stride 2M, stored twice (the second copy one
// float ahead) so that every pair of adjacent keys is one aligned 8-byte load.
constexpr int kSlotFloats = 8192;                            // two copies of (2M-1) rows fit for M <= 32
constexpr int kCopy1 = kSlotFloats / 2 + 16;
constexpr int kBiasOff = kKcolOff + kStages * 128 * 4;
constexpr int kBarOff = kBiasOff + 2 * kSlotFloats * 4;
constexpr int kNumBars = 12 + 3 * kStages + 12 + 3 + 4;
constexpr int kSmemBytes = kBarOff + kNumBars * 8 + 64;
constexpr int kSmemAlloc = kSmemBytes + 1024;  // slack for 1024-byte alignment
static_assert(kSmemAlloc <= 227 * 1024, "shared memory budget");

constexpr float kLog2eF = 1.4426950408889634f;

struct Bars {
  uint64_t q_full[2][2], q_ready[2][2], q_empty[2][2];
  uint64_t kv_full[kStages], kv_ready[kStages], kv_empty[kStages];
  // per warpgroup and score buffer: a barrier's next phase (block b + 2) can
  // only start after its current one was consumed, so parity tests never alias
  uint64_t s_full[2][2], p_full[2][2], o_done[2][2];
  uint64_t never, drain[2];
  uint64_t tab_free[2], tab_ready[2];  // bias-table slot handshake of each softmax warpgroup (4 warps)
};
static_assert(sizeof(Bars) == kNumBars * 8, "barrier block size");

// One warpgroup's query tile: its rectangle (a column segment of the item's
// row of rectangles) and the tile's index in it.
struct Rect {
  int cls, lx, R, Rk, x0, tile, nb;  // x-class, width, tile rows, K/V block rows, first column, tile, K/V blocks
};

// A work item: query tiles 2i and 2i + 1 of one row of rectangles of one
// (head, image), the row's tiles listed rectangle by rectangle.  Warpgroup 0
// takes the first; warpgroup 1 the second, if the row has it.  Two tiles of
// one rectangle share its K/V blocks; tiles of two rectangles stream both
// rectangles' blocks, alternating (A0, B0, A1, B1, ...), then the longer one's
// remainder, each block used by one warpgroup.
struct Task {
  int b, h, y0, ly;
  bool v1;      // warpgroup 1 has a tile
  bool shared;  // both tiles in one rectangle
  int nbt;      // K/V blocks the item loads
  Rect r0, r1;
  __device__ __forceinline__ bool valid(int g) const { return g == 0 || v1; }
  __device__ __forceinline__ Rect rect(int g) const { return g ? r1 : r0; }
  __device__ __forceinline__ int nq(int g) const {  // queries of warpgroup g's tile
    const Rect r = rect(g);
    const int rows = ly - r.tile * r.R;
    return (rows < r.R ? rows : r.R) * r.lx;
  }
  // position among the item's K/V loads of warpgroup g's block j
  __device__ __forceinline__ int kv_index(int g, int j) const {
    if (shared) return j;
    const int mn = r0.nb < r1.nb ? r0.nb : r1.nb;
    return j < mn ? 2 * j + g : mn + j;
  }
  // owner warpgroup (its rectangle) and block index of the item's K/V load jj
  __device__ __forceinline__ Rect kv_rect(int jj, int& j) const {
    const int mn = shared ? 0 : (r0.nb < r1.nb ? r0.nb : r1.nb);
    if (jj < 2 * mn) {
      j = jj >> 1;
      return (jj & 1) ? r1 : r0;
    }
    j = jj - mn;
    return (shared || r0.nb > r1.nb) ? r0 : r1;
  }
};

__device__ __forceinline__ Task decode(const TcParams& p, long long item) {
  Task t;
  uint32_t i = (uint32_t)item;
  if (p.pos_major) {
    // item i is position i / (B heads) of (head, image) i % (B heads): the
    // round-robin CTAs then see every position class evenly (tile pairs of
    // full and edge rectangles cost up to 3x apart) instead of a run of
    // consecutive positions; used without a bias table, whose per-head
    // reload favours heads outermost
    const uint32_t pos = fdiv(i, p.div_hb);
    i = (i - pos * p.div_hb.d) * p.div_ipb.d + pos;
  }
  uint32_t q = fdiv(i, p.div_ipb);
  uint32_t rem = i - q * p.div_ipb.d;  // item within (head, image)
  i = q;
  q = fdiv(i, p.div_B);
  t.b = (int)(i - q * p.div_B.d);
  t.h = (int)q;  // heads outermost: a CTA keeps one head's bias table for many items
  // row of rectangles: row 0, the nsy - 2 middle rows, the last row
  int rc, sy;
  uint32_t ii;
  if (rem < (uint32_t)p.row_items[0]) {
    rc = 0;
    sy = 0;
    ii = rem;
  } else {
    rem -= (uint32_t)p.row_items[0];
    const uint32_t mid = p.nsy > 2 ? (uint32_t)(p.nsy - 2) * (uint32_t)p.row_items[1] : 0u;
    if (rem < mid) {
      const uint32_t r = fdiv(rem, p.div_mid_items);
      rc = 1;
      sy = 1 + (int)r;
      ii = rem - r * (uint32_t)p.row_items[1];
    } else {
      rc = 2;
      sy = p.nsy - 1;
      ii = rem - mid;
    }
  }
  t.y0 = swin_seg_start(sy, p.M, p.s);
  t.ly = p.row_ly[rc];
  const int T = p.nsx == 1 ? p.row_tiles[rc][0]
                           : p.row_tiles[rc][0] + (p.nsx - 2) * p.row_tiles[rc][1] + p.row_tiles[rc][2];
  // tile k of the row -> (column segment, tile)
  auto tile_at = [&](int k, Rect& r) -> int {
    int sx = 0;
    const int t0 = p.row_tiles[rc][0];
    if (p.nsx > 1 && k >= t0) {
      k -= t0;
      const int mid = (p.nsx - 2) * p.row_tiles[rc][1];
      if (k < mid) {
        const int r2 = (int)fdiv((uint32_t)k, p.div_mid_tiles[rc]);
        sx = 1 + r2;
        k -= r2 * p.row_tiles[rc][1];
      } else {
        sx = p.nsx - 1;
        k -= mid;
      }
    }
    r.cls = sx == 0 ? 0 : (sx == p.nsx - 1 ? 2 : 1);
    r.lx = p.lx[r.cls];
    r.R = p.R[r.cls];
    r.Rk = p.Rk[r.cls];
    r.x0 = swin_seg_start(sx, p.M, p.s);
    r.tile = k;
    r.nb = p.row_nb[rc][r.cls];
    return sx;
  };
  const int sx0 = tile_at(2 * (int)ii, t.r0);
  t.v1 = 2 * (int)ii + 1 < T;
  int sx1 = -1;
  if (t.v1) {
    sx1 = tile_at(2 * (int)ii + 1, t.r1);
  } else {
    t.r1 = t.r0;
    t.r1.nb = 0;
  }
  t.shared = sx1 == sx0;
  t.nbt = t.shared ? t.r0.nb : t.r0.nb + t.r1.nb;
  return t;
}

struct Ctl {
  volatile int* abort;
  const TcParams* p;
};

// Bounded wait on an mbarrier phase; false if the wait ran out or another
// role aborted.
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, const Ctl& c) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (ptx::mbar_try_wait_sleep(bar, parity, 20000u)) return true;
    if (*c.abort) return false;
    if (clock64() - t0 > c.p->wait_limit) {
      atomicOr(c.p->status, (int)SWIN_ERR_TIMEOUT);
      *c.abort = 1;
      return false;
    }
  }
}

__device__ __forceinline__ uint32_t swz64(int row, int chunk) {
  // byte offset of 16-byte chunk `chunk` of 64-byte row `row` under 64B swizzle
  return (uint32_t)(row * 64 + ((chunk ^ ((row >> 1) & 3)) << 4));
}

__device__ __forceinline__ float bf_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// ------------------------------------------------------------------ prep
// Score-prep operands go to the tensor core as fp16 (both Q and K, so the MMA
// sees one type): fp16 keeps 3 more mantissa bits than bf16, and rounding the
// rotated operands is the largest error term of the path.  A rotated Q row is
// first scaled by an exact power of two that brings it below 2^15 (divided
// out in the softmax); rotated K rows and V are converted with saturation,
// and an entry at or beyond the fp16 range is reported as unsupported.

// Half rows: channels [16 h, 16 h + 16) = 16-byte chunks 2h and 2h + 1.
__device__ __forceinline__ void load_half_bf16(const uint8_t* tile, int row, int h, float (&v)[16]) {
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    const uint4 w = *reinterpret_cast<const uint4*>(tile + swz64(row, 2 * h + c));
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      v[8 * c + 2 * e] = bf_lo(u[e]);
      v[8 * c + 2 * e + 1] = bf_hi(u[e]);
    }
  }
}

__device__ __forceinline__ void store_half_f16(uint8_t* tile, int row, int h, const float (&v)[16], float sc) {
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    uint32_t u[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) u[e] = ptx::pack_f16x2_sat(v[8 * c + 2 * e] * sc, v[8 * c + 2 * e + 1] * sc);
    *reinterpret_cast<uint4*>(tile + swz64(row, 2 * h + c)) = make_uint4(u[0], u[1], u[2], u[3]);
  }
}

// Rotate the 8 channel pairs of one half by position pos of its axis (half 0:
// rows, half 1: columns).
__device__ __forceinline__ void rope_half(float (&v)[16], int h, int pos, const float* rc, const float* rs) {
  const float4* cs4 = reinterpret_cast<const float4*>(rc + (h * 64 + pos) * 8);
  const float4* sn4 = reinterpret_cast<const float4*>(rs + (h * 64 + pos) * 8);
  const float4 c0 = cs4[0], c1 = cs4[1], s0 = sn4[0], s1 = sn4[1];
  const float cs[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
  const float sn[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
  for (int t = 0; t < 8; ++t) {
    const float a = v[2 * t], b = v[2 * t + 1];
    // explicit roundings: every instantiation of the kernel computes the same bits
    v[2 * t] = __fmaf_rn(a, cs[t], -__fmul_rn(b, sn[t]));
    v[2 * t + 1] = __fmaf_rn(a, sn[t], __fmul_rn(b, cs[t]));
  }
}

// 2^e for a pair on the FMA pipe, so that part of the exponentials leave the
// MUFU: e = j + f with j = rint(e) read from the low mantissa bits of
// e + 1.5 * 2^23 and f in [-1/2, 1/2]; 2^f is a degree-3 polynomial fitted by
// the Remez exchange algorithm for minimax relative error on [-1/2, 1/2]
// (7.5e-5, below half an fp16 ulp), and j is added to its exponent field.
// Arguments below -125 are clamped (the result then rounds to 0 in fp16).
__device__ __forceinline__ float2 exp2_poly2(float2 e) {
  constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
  e.x = fmaxf(e.x, -125.0f);
  e.y = fmaxf(e.y, -125.0f);
  const float2 t = __fadd2_rn(e, make_float2(kRound, kRound));
  const float2 r = __fadd2_rn(t, make_float2(-kRound, -kRound));     // rint(e), exact
  const float2 f = __ffma2_rn(r, make_float2(-1.0f, -1.0f), e);      // e - rint(e), exact
  float2 q = __ffma2_rn(f, make_float2(0.0551716685f, 0.0551716685f), make_float2(0.2426111251f, 0.2426111251f));
  q = __ffma2_rn(q, f, make_float2(0.6932609677f, 0.6932609677f));
  q = __ffma2_rn(q, f, make_float2(0.9999280572f, 0.9999280572f));
  return make_float2(__uint_as_float(__float_as_uint(q.x) + (__float_as_uint(t.x) << 23)),
                     __uint_as_float(__float_as_uint(q.y) + (__float_as_uint(t.y) << 23)));
}

__device__ __forceinline__ float half_absmax(const float (&v)[16]) {
  float m = 0.f;
#pragma unroll
  for (int e = 0; e < 16; ++e) m = fmaxf(m, fabsf(v[e]));
  return m;
}

__device__ __forceinline__ float half_sumsq(const float (&v)[16]) {
  float ss = 0.f;
#pragma unroll
  for (int e = 0; e < 16; ++e) ss = fmaf(v[e], v[e], ss);
  return ss;
}


// Power of two that brings a row maximum m below 2^15 (fp16 max is 65504).
__device__ __forceinline__ float pow2_scale(float m) {
  if (!(m > 0.f)) return 1.f;
  int e;
  frexpf(m, &e);  // m < 2^e
  return ldexpf(1.0f, 15 - e);
}

// How a launch adds the relative bias (a template argument, so that each
// kernel carries only the code it runs): no table; pair loads (every
// rectangle width of the launch even); one load per key (some width odd).
enum BiasKind { kBiasNone = 0, kBiasPairs = 1, kBiasKeys = 2 };

// ------------------------------------------------------------------ kernel
template <int MODE, bool OUT_F32, int BIAS>
__global__ void __launch_bounds__(kThreads, 1) attn_tc_kernel(const __grid_constant__ TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment by pointer arithmetic on the shared array itself, so
  // that every access below stays a shared-space load or store
  uint8_t* smem = smem_raw + ((1024u - (static_cast<uint32_t>(__cvta_generic_to_shared(smem_raw)) & 1023u)) & 1023u);
  uint8_t* qbuf = smem + kQOff;
  uint8_t* kvbuf = smem + kKVOff;
  uint8_t* ones = smem + kOnesOff;
  float* qscale = reinterpret_cast<float*>(smem + kScaleOff);
  float* rcos = reinterpret_cast<float*>(smem + kRopeOff);
  float* rsin = rcos + 2 * 64 * 8;
  int* kofs = reinterpret_cast<int*>(smem + kKofsOff);
  int* rpos = reinterpret_cast<int*>(smem + kRposOff);
  float* kcol = reinterpret_cast<float*>(smem + kKcolOff);
  float* sbias = reinterpret_cast<float*>(smem + kBiasOff);  // [2 warpgroups][kSlotFloats]
  Bars* bars = reinterpret_cast<Bars*>(smem + kBarOff);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + kBarOff + kNumBars * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int M = p.M, s = p.s;

  // ---- set-up: barriers, RoPE tables, bias tables and column offsets, TMEM
  if (threadIdx.x == 0) {
    for (int g = 0; g < 2; ++g)
      for (int b = 0; b < 2; ++b) {
        ptx::mbar_init(&bars->q_full[g][b], 1);
        ptx::mbar_init(&bars->q_ready[g][b], kPrepThreads);
        ptx::mbar_init(&bars->q_empty[g][b], 1 + 4);
      }
    for (int i = 0; i < kStages; ++i) {
      ptx::mbar_init(&bars->kv_full[i], 1);
      ptx::mbar_init(&bars->kv_ready[i], kPrepThreads);
      ptx::mbar_init(&bars->kv_empty[i], 2);  // one release per softmax warpgroup
    }
    for (int g = 0; g < 2; ++g) {
      for (int b = 0; b < 2; ++b) {
        ptx::mbar_init(&bars->s_full[g][b], 1);
        ptx::mbar_init(&bars->p_full[g][b], 128);
        ptx::mbar_init(&bars->o_done[g][b], 1);
      }
    }
    ptx::mbar_init(&bars->never, 1);
    ptx::mbar_init(&bars->drain[0], 1);
    ptx::mbar_init(&bars->drain[1], 1);
    for (int g = 0; g < 2; ++g) {
      ptx::mbar_init(&bars->tab_free[g], 4);
      ptx::mbar_init(&bars->tab_ready[g], 4);
    }
    *abort_flag = 0;
    tmem_holder[2] = 0;  // abort flag of the drain waits (never set by a role)
    ptx::fence_mbar_init();
  }
  if (MODE == 2) {
    // all 64 positions (rows past a rectangle's end, which are masked, read up to 63)
    for (int i = threadIdx.x; i < 2 * 64 * 8; i += kThreads) {
      const int axis = i / (64 * 8), pos = (i / 8) % 64, t = i % 8;
      float sv = 0.f, cv = 1.f;
      if (pos < M) sincosf((float)pos * p.rope[axis * 8 + t], &sv, &cv);
      rcos[(axis * 64 + pos) * 8 + t] = cv;
      rsin[(axis * 64 + pos) * 8 + t] = sv;
    }
  }
  const int R2e = p.R2e;
  constexpr bool has_table = MODE != 2 && BIAS != kBiasNone;
  for (int i = threadIdx.x; i < 3 * 128; i += kThreads) {
    const int c = i / 128, col = i % 128, lx = p.lx[c];
    kofs[i] = (col / lx) * R2e + (col % lx);  // slot offset of key col
    rpos[i] = (col / lx) | ((col % lx) << 16);
  }
  // zero the K/V ring and the ones blocks once, so rows a tile never writes
  // hold finite values
  for (int i = threadIdx.x; i < (kStages * 2 * kTileBytes + kStages * 1024) / 16; i += kThreads)
    reinterpret_cast<uint4*>(kvbuf)[i] = make_uint4(0, 0, 0, 0);
  __syncthreads();
  // the constant column block of every stage: fp16 1.0 in the first column of 16 rows
  if (threadIdx.x < 16 * kStages)
    *reinterpret_cast<uint16_t*>(ones + (threadIdx.x / 16) * 1024 + swz64(threadIdx.x % 16, 0)) = 0x3C00;
  if (warp == 1) {
    ptx::tmem_alloc(tmem_holder, 512);
    ptx::tmem_relinquish();
  }
  if (warp == 0 && lane == 0)
    for (int t = 0; t < 3; ++t)
      for (int c = 0; c < 3; ++c) ptx::prefetch_tmap(&p.tmap[t][c]);
  ptx::fence_proxy_async_smem();
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  Ctl ctl{abort_flag, &p};
  const long long first = blockIdx.x, step = gridDim.x;

  // Register split: warpgroups 0 (producer, MMA, prep) and 3 (prep) give
  // registers to the two softmax warpgroups: 512 x 128 = 256 x 64 + 256 x 192.
  if (warp < 4 || warp >= 12) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 64;\n" ::: "memory");
    if (warp == 0) {
      // ============================================================== producer
      if (lane == 0) {
        uint32_t qu[2] = {0, 0};
        uint32_t ku = 0;
        bool ok = true;
        for (long long it = first; it < p.n_items && ok; it += step) {
          const Task t = decode(p, it);
          for (int g = 0; g < 2 && ok; ++g) {
            if (!t.valid(g)) continue;
            const Rect r = t.rect(g);
            const int qs = qu[g] & 1;
            if (qu[g] >= 2) ok = wait_bar(&bars->q_empty[g][qs], ((qu[g] >> 1) - 1) & 1, ctl);
            if (!ok) break;
            SWIN_DCHECK(p.status, t.h >= 0 && t.h < p.heads && r.x0 >= 0 && r.x0 + r.lx <= p.W && t.b >= 0 &&
                                      t.b < p.B && t.y0 + r.tile * r.R >= 0 && t.y0 + r.tile * r.R < p.H);
            ptx::mbar_arrive_expect_tx(&bars->q_full[g][qs], (uint32_t)(64 * r.lx * r.R));
            ptx::tma_load_5d(qbuf + (g * 2 + qs) * kTileBytes, &p.tmap[0][r.cls], &bars->q_full[g][qs], 0, t.h,
                             r.x0, t.y0 + r.tile * r.R, t.b);
            ++qu[g];
          }
          for (int jj = 0; jj < t.nbt && ok; ++jj) {
            int j;
            const Rect r = t.kv_rect(jj, j);
            const int st = ku % kStages;
            if (ku >= (uint32_t)kStages) ok = wait_bar(&bars->kv_empty[st], ((ku / kStages) - 1) & 1, ctl);
            if (!ok) break;
            uint8_t* kb = kvbuf + st * 2 * kTileBytes;
            SWIN_DCHECK(p.status, t.h >= 0 && t.h < p.heads && r.x0 >= 0 && r.x0 + r.lx <= p.W && t.b >= 0 &&
                                      t.b < p.B && t.y0 + j * r.Rk >= 0 && t.y0 + j * r.Rk < p.H);
            ptx::mbar_arrive_expect_tx(&bars->kv_full[st], (uint32_t)(2 * 64 * r.lx * r.Rk));
            ptx::tma_load_5d(kb, &p.tmap[1][r.cls], &bars->kv_full[st], 0, t.h, r.x0, t.y0 + j * r.Rk, t.b);
            ptx::tma_load_5d(kb + kTileBytes, &p.tmap[2][r.cls], &bars->kv_full[st], 0, t.h, r.x0,
                             t.y0 + j * r.Rk, t.b);
            ++ku;
          }
        }
        // drain copies that may still be landing in shared memory (after an
        // abort; in a normal exit every phase waited here has completed)
        Ctl drain{reinterpret_cast<volatile int*>(tmem_holder + 2), &p};
        for (uint32_t u = (ku > (uint32_t)kStages ? ku - kStages : 0); u < ku; ++u)
          wait_bar(&bars->kv_full[u % kStages], (u / kStages) & 1, drain);
        for (int g = 0; g < 2; ++g)
          for (uint32_t u = (qu[g] > 2 ? qu[g] - 2 : 0); u < qu[g]; ++u)
            wait_bar(&bars->q_full[g][u & 1], (u >> 1) & 1, drain);
      }
    } else if (warp == 1 || warp == 2) {
      // ============================================================== MMA issuers
      // One thread per softmax warpgroup g (warp 1 + g) issues that group's
      // MMAs in program order: S(0), S(1), then for every later block b first
      // PV(b - 2), as soon as P(b - 2) is in TMEM, and then S(b).  A thread's
      // MMAs execute in issue order, so S(b) cannot overwrite P(b - 2) before
      // PV(b - 2) has read it.
      if (lane == 0) {
        const int g = warp - 1;
        // mode 2 feeds fp16 score operands (see prep), modes 0 and 1 the bf16 inputs
        constexpr uint32_t fmtS = MODE == 2 ? 0u : 1u;
        constexpr uint32_t idS = ptx::idesc_f16(fmtS, fmtS, 0, 0, kBlk, 128);
        constexpr uint32_t idPV = ptx::idesc_f16(0, 0, 0, 1, 48, 128);  // fp16 P (TMEM) x fp16 [V | c]
        // Operand descriptors (64-byte swizzle) of Q buffer 0 and K/V stage 0;
        // the others differ only in the start-address field (16-byte units)
        // and, for [V | c], in the leading byte offset to the stage's constant
        // column block, which sits outside the ring (N columns 32-47).
        const uint64_t qd0 = ptx::smem_desc(ptx::smem_addr(qbuf + g * 2 * kTileBytes), 16, 512, ptx::kSwizzle64B);
        const uint64_t kd0 = ptx::smem_desc(ptx::smem_addr(kvbuf), 16, 512, ptx::kSwizzle64B);
        const uint32_t va0 = ptx::smem_addr(kvbuf + kTileBytes), oa0 = ptx::smem_addr(ones);
        const uint64_t vd0 = ptx::smem_desc(va0, oa0 - va0, 512, ptx::kSwizzle64B);
        constexpr uint64_t kQBuf = kTileBytes >> 4;
        constexpr uint64_t kStageK = (2 * kTileBytes) >> 4;
        constexpr uint64_t kStageV = kStageK - ((uint64_t)((2 * kTileBytes - 1024) >> 4) << 16);
        // k-step kk of PV: V rows 16 kk.. (+1024 bytes), constant block unchanged
        constexpr uint64_t kStepV = (uint64_t)(1024 >> 4) - ((uint64_t)(1024 >> 4) << 16);
        const uint32_t tg = tmem_base + g * 256;
        bool ok = true;
        if (p.debug_flags & 1) ok = wait_bar(&bars->never, 0, ctl);  // forced time-out
        // blocks whose PV is still to be issued, by b & 1: stage | accumulate << 8 | second release << 9
        uint32_t pend0 = 0, pend1 = 0;
        auto issue_pv = [&](uint32_t k) -> bool {
          if (!wait_bar(&bars->p_full[g][k & 1], (k >> 1) & 1, ctl)) return false;
          ptx::tc_fence_after();
          const uint32_t info = (k & 1) ? pend1 : pend0;
          const uint32_t st = info & 0xffu;
          const uint64_t vd = vd0 + st * kStageV;
          const uint32_t aP = tg + (k & 1) * kBlk;
          ptx::mma_ts(tg + 2 * kBlk, aP, vd, idPV, (info >> 8) & 1u);
#pragma unroll
          for (int kk = 1; kk < kBlk / 16; ++kk) ptx::mma_ts(tg + 2 * kBlk, aP + kk * 8, vd + kk * kStepV, idPV, 1u);
          ptx::mma_commit(&bars->o_done[g][k & 1]);
          ptx::mma_commit(&bars->kv_empty[st]);
          if (info >> 9) ptx::mma_commit(&bars->kv_empty[st]);  // the other warpgroup has no tile here
          return true;
        };
        // K/V uses (all items), Q tiles, S and PV issued by this group, K/V use of S(b - 1)
        uint32_t u = 0, qcnt = 0, b = 0, npv = 0, u_last = 0;
        for (long long it = first; it < p.n_items && ok; it += step) {
          const Task t = decode(p, it);
          const uint32_t u0 = u;
          u += t.nbt;
          if (!t.valid(g)) continue;
          const uint32_t qs = qcnt & 1, qpar = (qcnt >> 1) & 1;
          ++qcnt;
          const uint64_t ad = qd0 + qs * kQBuf;
          const int nb = t.rect(g).nb;
          // a block used by this warpgroup alone takes both releases of its stage
          const uint32_t rel2 = t.shared ? 0u : 512u;
          for (int j = 0; j < nb; ++j, ++b) {
            const uint32_t uu = u0 + t.kv_index(g, j), st = uu % kStages;
            // S(b) overwrites P(b - 2): PV(b - 2) first
            while (ok && npv + 2 <= b) ok = issue_pv(npv++);
            // A pending PV(b - 1) whose K/V use is a whole ring behind block
            // uu holds a slot the producer needs before it can load uu (or
            // the next Q tile): issue it before waiting for either.
            if (ok && npv < b && u_last + kStages <= uu) ok = issue_pv(npv++);
            ok = ok && (j > 0 || wait_bar(&bars->q_ready[g][qs], qpar, ctl)) &&
                 wait_bar(&bars->kv_ready[st], (uu / kStages) & 1, ctl);
            if (!ok) break;
            ptx::tc_fence_after();
            const uint64_t bd = kd0 + st * kStageK;
            const uint32_t dS = tg + (b & 1) * kBlk;
            ptx::mma_ss(dS, ad, bd, idS, 0);
            ptx::mma_ss(dS, ad + 2, bd + 2, idS, 1);  // second 16-wide K step: +32 bytes
            ptx::mma_commit(&bars->s_full[g][b & 1]);
            if (j == nb - 1) ptx::mma_commit(&bars->q_empty[g][qs]);
            const uint32_t info = st | (j > 0 ? 256u : 0u) | rel2;
            if (b & 1) pend1 = info; else pend0 = info;
            u_last = uu;
          }
        }
        while (ok && npv < b) ok = issue_pv(npv++);
        // drain: every MMA this thread issued has completed before TMEM is freed
        ptx::mma_commit(&bars->drain[g]);
        Ctl drain{reinterpret_cast<volatile int*>(tmem_holder + 2), &p};
        wait_bar(&bars->drain[g], 0, drain);
      }
    } else {
      // ============================================================== prep
      // 160 threads (warps 3 and 12-15); work in half rows (16 channels):
      // the two halves of a row sit in adjacent lanes, and each half of a
      // RoPE row rotates along one axis only.
      // Row work goes to warps 12-15, one per SM sub-partition, so that every
      // softmax warp shares its sub-partition with the same prep load (warp 3
      // only takes part in the arrivals): query row (warp - 12) * 32 + lane,
      // key row (warp - 12) * 24 + lane.
      const int prow_q = warp >= 12 ? (warp - 12) * 32 + lane : 1 << 20;
      const int prow_k = warp >= 12 && lane < 24 ? (warp - 12) * 24 + lane : 1 << 20;
      uint32_t qu[2] = {0, 0}, ku = 0;
      bool ok = true;
      bool range_hit = false;  // a rotated K or a V entry saturated the fp16 range
      for (long long it = first; it < p.n_items && ok; it += step) {
        const Task t = decode(p, it);
        // window-local coordinate of the row of rectangles' first row
        const int py0 = swin_local_coord(t.y0, M, s);
        for (int g = 0; g < 2 && ok; ++g) {
          if (!t.valid(g)) continue;
          const Rect rq = t.rect(g);
          const int qrows = rq.lx * rq.R;
          const int* rp = rpos + rq.cls * 128;
          const int px0 = swin_local_coord(rq.x0, M, s);
          const int qs = qu[g] & 1;
          // warp-uniform outcome (the shuffles below need every lane)
          ok = __all_sync(0xffffffffu, wait_bar(&bars->q_full[g][qs], (qu[g] >> 1) & 1, ctl));
          ++qu[g];
          if (!ok) break;
          uint8_t* tile = qbuf + (g * 2 + qs) * kTileBytes;
          const float te = MODE == 1 ? fmaxf(__ldg(p.tau + t.h), kTauMin) : 1.f;
          if (MODE != 0) {
            // one query row per thread (a tile has at most 128 rows)
            const int r = prow_q;
            if (r < qrows) {
              float v0[16], v1[16];
              load_half_bf16(tile, r, 0, v0);
              load_half_bf16(tile, r, 1, v1);
              if (MODE == 1) {
                const float ss = half_sumsq(v0) + half_sumsq(v1);
                qscale[(g * 2 + qs) * 128 + r] = kLog2eF / (fmaxf(sqrtf(ss), kNormEps) * te);
              } else {
                // the row's scale needs both halves rotated: the first half is
                // rotated again for the store (fewer live registers)
                const int pr = rp[r];
                const int pos0 = min(py0 + rq.tile * rq.R + (pr & 0xFFFF), 63), pos1 = px0 + (pr >> 16);
                rope_half(v0, 0, pos0, rcos, rsin);
                rope_half(v1, 1, pos1, rcos, rsin);
                const float sc = pow2_scale(fmaxf(half_absmax(v0), half_absmax(v1)));  // exact, undone in the softmax
                store_half_f16(tile, r, 1, v1, sc);
                load_half_bf16(tile, r, 0, v0);
                rope_half(v0, 0, pos0, rcos, rsin);
                store_half_f16(tile, r, 0, v0, sc);
                qscale[(g * 2 + qs) * 128 + r] = kLog2eF * rsqrtf(32.0f) / sc;
              }
            }
            ptx::fence_proxy_async_smem();
          }
          ptx::mbar_arrive(&bars->q_ready[g][qs]);
        }
        for (int jj = 0; jj < t.nbt && ok; ++jj) {
          int j;
          const Rect rk = t.kv_rect(jj, j);
          const int krows = rk.lx * rk.Rk;
          const int* rp = rpos + rk.cls * 128;
          const int px0 = swin_local_coord(rk.x0, M, s);
          const int st = ku % kStages;
          ok = __all_sync(0xffffffffu, wait_bar(&bars->kv_full[st], (ku / kStages) & 1, ctl));
          ++ku;
          if (!ok) break;
          uint8_t* ktile = kvbuf + st * 2 * kTileBytes;
          uint8_t* vtile = ktile + kTileBytes;
          // one key row per thread (a block has at most 96 rows)
          {
            const int r = prow_k;
            if (r < krows) {
#pragma unroll 1
              for (int h = 0; h < 2; ++h) {
                float v[16];
                load_half_bf16(vtile, r, h, v);
                range_hit |= half_absmax(v) >= 65504.0f;
                store_half_f16(vtile, r, h, v, 1.0f);
              }
            }
          }
          if (MODE != 0) {
            const int r = prow_k;
            if (r < krows) {
              if (MODE == 1) {
                float v0[16], v1[16];
                load_half_bf16(ktile, r, 0, v0);
                load_half_bf16(ktile, r, 1, v1);
                kcol[st * 128 + r] = 1.0f / fmaxf(sqrtf(half_sumsq(v0) + half_sumsq(v1)), kNormEps);
              } else {
                const int pr = rp[r];
#pragma unroll 1
                for (int h = 0; h < 2; ++h) {
                  float v[16];
                  load_half_bf16(ktile, r, h, v);
                  rope_half(v, h, h ? px0 + (pr >> 16) : min(py0 + j * rk.Rk + (pr & 0xFFFF), 63), rcos, rsin);
                  range_hit |= half_absmax(v) >= 65504.0f;
                  store_half_f16(ktile, r, h, v, 1.0f);
                }
              }
            }
          }
          ptx::fence_proxy_async_smem();
          ptx::mbar_arrive(&bars->kv_ready[st]);
        }
      }
      if (range_hit) atomicOr(p.status, (int)SWIN_ERR_UNSUPPORTED);
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 192;\n" ::: "memory");
    // ================================================================ softmax
    const int g = (warp - 4) >> 2;              // warpgroup 0 or 1
    const int t = threadIdx.x - 128 - g * 128;  // row of the tile = TMEM lane
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tX = tmem_base + g * 256 + lane_off;  // X0; X1 = tX + kBlk
    const uint32_t tO = tX + 2 * kBlk;
    const float cscale = kLog2eF * rsqrtf(32.0f);
    float* slot = sbias + g * kSlotFloats;
    // second copy: slot[kCopy1 + i] = slot[i + 1], 16 banks away from the first
    int cur_h = -1;
    uint32_t tabn = 0;  // table loads of this warpgroup
    uint32_t qu = 0, ku = 0, blk = 0;  // Q tiles, K/V uses, blocks of this warpgroup
    bool ok = true;
    bool pend = false, pend_ok = false;  // an item's O still waiting in TMEM
    size_t pend_off = 0;
    // O / l of one row to global memory (32 values; column 32 holds l)
    auto store_rows = [&](const uint32_t (&o)[32], uint32_t l, size_t off, bool row_valid) {
      if (!row_valid) return;
#if SWIN_DEBUG_BUILD
      if (off % 32 != 0 || off + 32 > (size_t)p.B * p.H * p.W * p.heads * 32) {
        atomicOr(p.status, kStatusRangeCheck);
        return;
      }
#endif
      const float inv = 1.0f / __uint_as_float(l);  // row sum of the fp16 P
      if (OUT_F32) {
        float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + off);
#pragma unroll
        for (int c = 0; c < 8; ++c)
          dst[c] = make_float4(__uint_as_float(o[4 * c]) * inv, __uint_as_float(o[4 * c + 1]) * inv,
                               __uint_as_float(o[4 * c + 2]) * inv, __uint_as_float(o[4 * c + 3]) * inv);
      } else {
        uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + off);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            w[e] = ptx::pack_bf16x2(__uint_as_float(o[8 * c + 2 * e]) * inv,
                                    __uint_as_float(o[8 * c + 2 * e + 1]) * inv);
          dst[c] = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
    };
    // PV completion: o_done[parity] completes once per PV of that parity.
    // The softmax waits on it only where O is read (rescale, deferred
    // epilogue); every other completion is inferred: S(b)'s commit follows
    // PV(b - 2)'s MMAs in the issuing thread, so s_full(b) implies that
    // PV(0..b-2) are complete.  A parity wait for PV(k) cannot alias:
    // PV(k + 2) needs P(k + 2), which this warpgroup has not written yet.
    uint32_t o_cons = 0;  // PVs of this warpgroup known complete
    auto consume_pv = [&](uint32_t upto) -> bool {  // PV(0..upto) complete
      bool r = true;
      while (r && o_cons <= upto) {
        r = wait_bar(&bars->o_done[g][o_cons & 1], (o_cons >> 1) & 1, ctl);
        r = __all_sync(0xffffffffu, r);
        ++o_cons;
      }
      ptx::tc_fence_after();
      return r;
    };
    for (long long it = first; it < p.n_items && ok; it += step) {
      const Task tk = decode(p, it);
      const uint32_t ku0 = ku;
      ku += tk.nbt;  // K/V loads of this item (both warpgroups)
      if (!tk.valid(g)) continue;
      const Rect rg = tk.rect(g);
      if (has_table && tk.h != cur_h) {
        // new head: once all four warps are done with the old table, each
        // loads a quarter of the new one (times log2 e, zero padding column)
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&bars->tab_free[g]);
        ok = __all_sync(0xffffffffu, wait_bar(&bars->tab_free[g], tabn & 1, ctl));
        if (!ok) break;
        const int n = (2 * M - 1) * R2e;
        for (int i = (warp & 3) * 32 + lane; i < n; i += 128) {
          const int dy = i / R2e, c = i - dy * R2e;
          const float v = c < 2 * M - 1 ? __ldg(p.table + (size_t)(dy * (2 * M - 1) + c) * p.heads + tk.h) * kLog2eF : 0.f;
          slot[i] = v;
          if (i > 0) slot[kCopy1 + i - 1] = v;
        }
        if (warp == 4 + 4 * g && lane == 0) slot[kCopy1 + n - 1] = 0.f;
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&bars->tab_ready[g]);
        ok = __all_sync(0xffffffffu, wait_bar(&bars->tab_ready[g], tabn & 1, ctl));
        ++tabn;
        if (!ok) break;
        cur_h = tk.h;
      }
      const int qs = qu & 1;
      ok = wait_bar(&bars->q_ready[g][qs], (qu >> 1) & 1, ctl);
      ok = __all_sync(0xffffffffu, ok);
      ++qu;
      if (!ok) break;
      // per-row score scale: mode 1 log2e / (tau |q|), mode 2 log2e / (sqrt(d) 2^e)
      const float alpha = MODE == 0 ? cscale : qscale[(g * 2 + qs) * 128 + t];
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&bars->q_empty[g][qs]);
      const bool row_ok = t < tk.nq(g);
      const int qy = rg.tile * rg.R + t / rg.lx, qx = t % rg.lx;
      // Slot index of this row's bias for key (0, 0) of the rectangle; the
      // pair load for keys (2c, 2c+1) of a row starts one float earlier, in
      // copy 0 when that index is even, else in copy 1 (the parity is fixed
      // per query: row stride and even key offsets do not change it).
      // Bias loads are unconditional: rows past the tile use row M - 1, and
      // keys past the block (masked below) read other slot entries, at
      // most 95 rows of 2M floats before slot 0, inside shared memory.
      const int bbase = (min(qy, M - 1) + M - 1) * R2e + (qx + M - 1);
      const float* pbase = slot + (((bbase - 1) & 1) ? kCopy1 - 1 : 0) + bbase - 1;
      const int* kof = kofs + rg.cls * 128;
      float m_run = -INFINITY;
      for (int j = 0; j < rg.nb; ++j, ++blk) {
        SWIN_TC_MARK(0);
        ok = wait_bar(&bars->s_full[g][blk & 1], (blk >> 1) & 1, ctl);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        SWIN_TC_MARK(1);
        ptx::tc_fence_after();
        const uint32_t tS = tX + (blk & 1) * kBlk, tP = tS;  // P written over the scores
        float2 x[kBlk / 2];  // scores as packed pairs (keys 2c, 2c+1)
        {
          uint32_t r0[32], r1[32], r2[32];
          ptx::tmem_ld32(tS, r0);
          ptx::tmem_ld32(tS + 32, r1);
          ptx::tmem_ld32(tS + 64, r2);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            x[e] = make_float2(__uint_as_float(r0[2 * e]), __uint_as_float(r0[2 * e + 1]));
            x[16 + e] = make_float2(__uint_as_float(r1[2 * e]), __uint_as_float(r1[2 * e + 1]));
            x[32 + e] = make_float2(__uint_as_float(r2[2 * e]), __uint_as_float(r2[2 * e + 1]));
          }
        }
        SWIN_TC_MARK(2);
        const uint32_t u = ku0 + tk.kv_index(g, j), ust = u % kStages;
        if (MODE == 1) {
          // 1/|k| of the block's keys was written by prep before it released kv_ready
          ok = wait_bar(&bars->kv_ready[ust], (u / kStages) & 1, ctl);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
        }
        SWIN_TC_MARK(11);
        const float ascale = alpha;
        const int nk_all = (tk.ly - j * rg.Rk) * rg.lx;
        const int nk = nk_all < rg.Rk * rg.lx ? nk_all : rg.Rk * rg.lx;
        // x = log2-domain logits.  Mode 2: the scale is applied inside the
        // exponent below (max over raw scores, scale > 0).  Modes 0/1:
        // x = S * scale + bias in one rounding; the bias slot already holds
        // T * log2(e), and mode 1's scale is log2e / (tau |q| |k|).
        if (MODE != 2) {
          const float4* kc4 = reinterpret_cast<const float4*>(kcol + ust * 128);
          const int4* kof4 = reinterpret_cast<const int4*>(kof);
          const int jo = j * rg.Rk * R2e;  // block j starts Rk rectangle rows further
          if (!has_table) {
            const float2 a2 = make_float2(ascale, ascale);
#pragma unroll
            for (int c4 = 0; c4 < kBlk / 4; ++c4) {
              float2 s0 = a2, s1 = a2;
              if (MODE == 1) {
                const float4 kc = kc4[c4];
                s0 = __fmul2_rn(make_float2(kc.x, kc.y), a2);
                s1 = __fmul2_rn(make_float2(kc.z, kc.w), a2);
              }
              x[2 * c4] = __fmul2_rn(x[2 * c4], s0);
              x[2 * c4 + 1] = __fmul2_rn(x[2 * c4 + 1], s1);
            }
          } else if (BIAS == kBiasPairs) {
            const float* pb = pbase - jo;
#pragma unroll
            for (int c4 = 0; c4 < kBlk / 4; ++c4) {
              float2 s0 = make_float2(ascale, ascale), s1 = s0;
              if (MODE == 1) {
                const float4 kc = kc4[c4];  // same address in every lane: broadcast
                s0 = __fmul2_rn(make_float2(kc.x, kc.y), s0);
                s1 = __fmul2_rn(make_float2(kc.z, kc.w), s1);
              }
              const int4 ko = kof4[c4];  // broadcast; keys 4 c4 .. 4 c4 + 3 share a row pairwise
#if SWIN_DEBUG_BUILD
              // unmasked keys of a valid row read inside this warpgroup's slot
              if (row_ok && 4 * c4 < nk) {
                const long long i0 = (long long)(pb - ko.x - slot);
                SWIN_DCHECK(p.status, i0 >= 0 && i0 + 1 < kSlotFloats);
              }
              if (row_ok && 4 * c4 + 2 < nk) {
                const long long i1 = (long long)(pb - ko.z - slot);
                SWIN_DCHECK(p.status, i1 >= 0 && i1 + 1 < kSlotFloats);
              }
#endif
              const float2 b0 = *reinterpret_cast<const float2*>(pb - ko.x);  // (bias key+1, bias key)
              const float2 b1 = *reinterpret_cast<const float2*>(pb - ko.z);
              x[2 * c4] = __ffma2_rn(x[2 * c4], s0, make_float2(b0.y, b0.x));
              x[2 * c4 + 1] = __ffma2_rn(x[2 * c4 + 1], s1, make_float2(b1.y, b1.x));
            }
          } else {
            // odd rectangle widths: one load per key
            const float* hb = slot + bbase - jo;
#pragma unroll
            for (int c4 = 0; c4 < kBlk / 4; ++c4) {
              float2 s0 = make_float2(ascale, ascale), s1 = s0;
              if (MODE == 1) {
                const float4 kc = kc4[c4];
                s0 = __fmul2_rn(make_float2(kc.x, kc.y), s0);
                s1 = __fmul2_rn(make_float2(kc.z, kc.w), s1);
              }
              const int4 ko = kof4[c4];
#if SWIN_DEBUG_BUILD
              {
                const int kk[4] = {ko.x, ko.y, ko.z, ko.w};
                for (int e = 0; e < 4; ++e)
                  if (row_ok && 4 * c4 + e < nk) {
                    const long long ii = (long long)(hb - kk[e] - slot);
                    SWIN_DCHECK(p.status, ii >= 0 && ii < kSlotFloats);
                  }
              }
#endif
              x[2 * c4] = __ffma2_rn(x[2 * c4], s0, make_float2(hb[-ko.x], hb[-ko.y]));
              x[2 * c4 + 1] = __ffma2_rn(x[2 * c4 + 1], s1, make_float2(hb[-ko.z], hb[-ko.w]));
            }
          }
        }
        SWIN_TC_MARK(12);
        if (nk < kBlk) {  // partial block (uniform across the warpgroup): mask the tail keys
#pragma unroll
          for (int c = 0; c < kBlk / 2; ++c) {
            if (2 * c >= nk) x[c].x = -INFINITY;
            if (2 * c + 1 >= nk) x[c].y = -INFINITY;
          }
        }
        // block maximum: four independent 3-input max chains, two pairs a step
        static_assert(kBlk % 4 == 0, "pairs are taken two at a time");
        float mq[4] = {x[0].x, x[0].y, x[1].x, x[1].y};
#pragma unroll
        for (int c = 2; c < kBlk / 2; c += 2) {
          const int ch = 2 * ((c >> 1) & 1);
          mq[ch] = ptx::max3(mq[ch], x[c].x, x[c + 1].x);
          mq[ch + 1] = ptx::max3(mq[ch + 1], x[c].y, x[c + 1].y);
        }
        float mb = fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3]));
        if (MODE == 2) mb *= ascale;
        SWIN_TC_MARK(3);
        // running maximum, kept unless this block exceeds it by more than 8
        float factor = 1.f;
        bool rescale = false;
        if (j == 0) {
          m_run = mb;
        } else if (mb > m_run + 8.0f) {
          factor = ptx::ex2_approx(m_run - mb);
          m_run = mb;
          rescale = true;
        }
        if (blk >= 2 && o_cons < blk - 1) o_cons = blk - 1;  // PV(0..blk-2) done: s_full(blk) seen
        SWIN_TC_MARK(4);
        // probabilities, fp16; written over the scores after O is brought up to
        // date, so the scores' registers are free by then.
        // exponent argument: mode 2  x * ascale - m,  modes 0/1  x - m
        const float ea = MODE == 2 ? ascale : 1.0f, eb = -m_run;
        // keys 0-63 on the MUFU, stored to TMEM while keys 64-95 are done;
        // mode 2 (no bias work, MUFU-bound) takes those through the
        // polynomial on the FMA pipe
        uint32_t pa[32], pb[16];
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const float2 e = __ffma2_rn(x[c], make_float2(ea, ea), make_float2(eb, eb));
          pa[c] = ptx::pack_f16x2(ptx::ex2_approx(e.x), ptx::ex2_approx(e.y));
        }
        ptx::tmem_st32(tP, pa);
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const float2 e = __ffma2_rn(x[32 + c], make_float2(ea, ea), make_float2(eb, eb));
          if (MODE == 2) {
            const float2 pe = exp2_poly2(e);
            pb[c] = ptx::pack_f16x2(pe.x, pe.y);
          } else {
            pb[c] = ptx::pack_f16x2(ptx::ex2_approx(e.x), ptx::ex2_approx(e.y));
          }
        }
        SWIN_TC_MARK(5);
        // O (32 columns) and its row sum (column 32): rescaled to the new
        // maximum, or, in an item's first block, the previous item's result
        // read for the deferred store.  Both need PV(blk - 1) complete.
        uint32_t po[32], pl = 0;
        const bool epi = j == 0 && pend;
        const bool resc = j > 0 && __any_sync(0xffffffffu, rescale);
        if (epi || resc) {
          ok = consume_pv(blk - 1);
          if (!ok) break;
          ptx::tmem_ld32(tO, po);
          pl = ptx::tmem_ld1(tO + 32);
          ptx::tmem_wait_ld();
          if (resc) {
#pragma unroll
            for (int e = 0; e < 32; ++e) po[e] = __float_as_uint(__uint_as_float(po[e]) * factor);
            ptx::tmem_st32(tO, po);
            ptx::tmem_st1(tO + 32, __float_as_uint(__uint_as_float(pl) * factor));
          }
        }
        ptx::tmem_st16(tP + 32, pb);
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        ptx::mbar_arrive(&bars->p_full[g][blk & 1]);
        SWIN_TC_MARK(6);
        if (epi) {
          store_rows(po, pl, pend_off, pend_ok);
          pend = false;
        }
        SWIN_TC_MARK(7);
      }
      if (!ok) break;
      // this item's O is read in the next item's first block (or after the loop)
      SWIN_TC_MARK(8);
      pend = true;
      pend_ok = row_ok;
      pend_off = (((size_t)tk.b * p.H + (tk.y0 + qy)) * p.W + (rg.x0 + qx)) * (size_t)(p.heads * 32) +
                 (size_t)tk.h * 32;
      SWIN_TC_MARK(10);
    }
    if (ok && pend) {
      ok = consume_pv(blk - 1);
      if (ok) {
        uint32_t po[32];
        ptx::tmem_ld32(tO, po);
        const uint32_t pl = ptx::tmem_ld1(tO + 32);
        ptx::tmem_wait_ld();
        store_rows(po, pl, pend_off, pend_ok);
      }
    }
  }

  // ---- teardown
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem_base, 512);
  }
}

// ------------------------------------------------------------------ host
bool encode_map(CUtensorMap* m, const void* base, const AttnArgs& a, int lx, int R) {
  EncodeTiledFn fn = tma_encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[5] = {32, (cuuint64_t)a.heads, (cuuint64_t)a.W, (cuuint64_t)a.H, (cuuint64_t)a.B};
  const cuuint64_t row = 64;  // bytes of one head
  const cuuint64_t strides[4] = {row, row * a.heads, row * a.heads * a.W, row * a.heads * a.W * a.H};
  const cuuint32_t box[5] = {32, 1, (cuuint32_t)lx, (cuuint32_t)R, 1};
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int MODE, bool F32, int BIAS>
swin_status launch_mode(const TcParams& p, int grid, cudaStream_t stream) {
  auto k = attn_tc_kernel<MODE, F32, BIAS>;
  cudaError_t ea = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemAlloc);
  if (ea != cudaSuccess) return fail(SWIN_ERR_CUDA, "attn_tc smem attribute: %s", cudaGetErrorString(ea));
  k<<<grid, kThreads, kSmemAlloc, stream>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(SWIN_ERR_CUDA, "attn_tc launch: %s", cudaGetErrorString(e));
  return SWIN_OK;
}

}  // namespace

// The driver entry point, looked up once; a function-local static with an
// initialiser is thread-safe in C++11 and later.
EncodeTiledFn tma_encode_fn() {
  static const EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<EncodeTiledFn>(p);
    return nullptr;
  }();
  return fn;
}

static long long g_tc_wait_limit = 4000000000ll;  // ~2 s at 2 GHz
static int g_tc_debug_flags = 0;

void tc_set_debug(int flags, long long wait_limit) {
  g_tc_debug_flags = flags;
  g_tc_wait_limit = wait_limit > 0 ? wait_limit : 4000000000ll;
}

swin_status launch_attn_tc(const AttnArgs& a, bool f32_out, cudaStream_t stream) {
  if (a.d != 32) return fail(SWIN_ERR_UNSUPPORTED, "tensor-core path needs d == 32, got %d", a.d);
  if (a.M > 64) return fail(SWIN_ERR_UNSUPPORTED, "tensor-core path needs M <= 64");
  if (a.mode != 2 && a.table && (2 * a.M - 1) * (2 * a.M) > kSlotFloats - kCopy1)
    return fail(SWIN_ERR_UNSUPPORTED, "tensor-core path keeps a bias table only for M <= 32");
  TcParams p;
  memset(&p, 0, sizeof(p));
  p.B = a.B; p.H = a.H; p.W = a.W; p.heads = a.heads; p.M = a.M; p.s = a.shift;
  p.nsy = swin_nseg(a.H, a.M, a.shift);
  p.nsx = swin_nseg(a.W, a.M, a.shift);
  const int lxs[3] = {swin_seg_len(0, a.W, a.M, a.shift),
                      p.nsx > 2 ? swin_seg_len(1, a.W, a.M, a.shift) : swin_seg_len(0, a.W, a.M, a.shift),
                      swin_seg_len(p.nsx - 1, a.W, a.M, a.shift)};
  for (int c = 0; c < 3; ++c) {
    p.lx[c] = lxs[c];
    p.R[c] = 128 / lxs[c];    // query tile: whole rectangle rows, at most 128 queries
    p.Rk[c] = kBlk / lxs[c];  // K/V block: whole rectangle rows, at most 96 keys
    if (!encode_map(&p.tmap[0][c], a.q, a, p.lx[c], p.R[c]) ||
        !encode_map(&p.tmap[1][c], a.k, a, p.lx[c], p.Rk[c]) ||
        !encode_map(&p.tmap[2][c], a.v, a, p.lx[c], p.Rk[c]))
      return fail(SWIN_ERR_CUDA, "cuTensorMapEncodeTiled failed (lx=%d, R=%d)", p.lx[c], p.R[c]);
  }
  // rows of rectangles by class: first, middle (if any), last
  const int lys[3] = {swin_seg_len(0, a.H, a.M, a.shift),
                      p.nsy > 2 ? swin_seg_len(1, a.H, a.M, a.shift) : swin_seg_len(0, a.H, a.M, a.shift),
                      swin_seg_len(p.nsy - 1, a.H, a.M, a.shift)};
  for (int rc = 0; rc < 3; ++rc) {
    p.row_ly[rc] = lys[rc];
    for (int c = 0; c < 3; ++c) {
      p.row_tiles[rc][c] = (lys[rc] + p.R[c] - 1) / p.R[c];
      p.row_nb[rc][c] = (lys[rc] + p.Rk[c] - 1) / p.Rk[c];
    }
    const int T = p.nsx == 1 ? p.row_tiles[rc][0]
                             : p.row_tiles[rc][0] + (p.nsx - 2) * p.row_tiles[rc][1] + p.row_tiles[rc][2];
    p.row_items[rc] = (T + 1) / 2;
    p.div_mid_tiles[rc] = make_fastdiv((uint32_t)p.row_tiles[rc][1]);
  }
  const long long ipb = (long long)p.row_items[0] + (p.nsy > 2 ? (long long)(p.nsy - 2) * p.row_items[1] : 0) +
                        (p.nsy > 1 ? p.row_items[2] : 0);
  // Bias-slot row stride: the even value in [2M, 2M + 14] (whose two copies fit
  // the slot) with the fewest shared-memory wavefronts for the paired bias
  // loads of this launch's rectangle widths.  A warp's 32 queries load 8
  // bytes each in two 16-lane phases; query (qy, qx) of a width-lx rectangle
  // reads floats qy R2e + qx - 1 (+ kCopy1 - 1 when that is odd) and on.
  p.R2e = 2 * a.M;
  if (a.mode != 2 && a.table) {
    long best = -1;
    for (int r2 = 2 * a.M; r2 <= 2 * a.M + 14; r2 += 2) {
      if ((2 * a.M - 1) * r2 > kSlotFloats - kCopy1) break;
      long cost = 0;
      for (int c = 0; c < 3; ++c) {
        const int lx = p.lx[c];
        if (lx & 1) continue;
        for (int w0 = 0; w0 < 128; w0 += 32)
          for (int ph = 0; ph < 2; ++ph) {
            int hits[16] = {0}, mx = 0;
            for (int l = 0; l < 16; ++l) {
              const int t = w0 + 16 * ph + l, qy = t / lx, qx = t % lx;
              int idx = qy * r2 + qx + a.M - 2;  // parity as in the kernel's bbase - 1
              if (idx & 1) idx += kCopy1 - 1;
              const int bank2 = (idx >> 1) & 15;
              mx = ++hits[bank2] > mx ? hits[bank2] : mx;
            }
            cost += mx;
          }
      }
      if (best < 0 || cost < best) {
        best = cost;
        p.R2e = r2;
      }
    }
  }
  p.n_items = (long long)a.B * a.heads * ipb;
  if (p.n_items >= (1ll << 31)) return fail(SWIN_ERR_UNSUPPORTED, "too many work items (%lld)", p.n_items);
  p.div_ipb = make_fastdiv((uint32_t)ipb);
  p.div_mid_items = make_fastdiv((uint32_t)p.row_items[1]);
  p.div_B = make_fastdiv((uint32_t)a.B);
  p.div_hb = make_fastdiv((uint32_t)(a.B * a.heads));
  p.pos_major = a.mode == 2 || a.table == nullptr;  // no per-head bias table to keep
  p.out = a.out;
  p.tau = a.tau;
  p.table = a.table;
  p.rope = a.rope;
  p.status = a.status;
  p.wait_limit = g_tc_wait_limit;
  p.debug_flags = g_tc_debug_flags;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = (int)(p.n_items < sms ? p.n_items : sms);
  switch (a.mode) {
    case 0:
    case 1: {
      const bool all_even = !(p.lx[0] & 1) && !(p.lx[1] & 1) && !(p.lx[2] & 1);
      const int kind = !a.table ? kBiasNone : (all_even ? kBiasPairs : kBiasKeys);
#define SWIN_TC_LAUNCH(MD)                                                                               \
  switch (kind) {                                                                                       \
    case kBiasNone:                                                                                     \
      return f32_out ? launch_mode<MD, true, kBiasNone>(p, grid, stream)                                \
                     : launch_mode<MD, false, kBiasNone>(p, grid, stream);                              \
    case kBiasPairs:                                                                                    \
      return f32_out ? launch_mode<MD, true, kBiasPairs>(p, grid, stream)                               \
                     : launch_mode<MD, false, kBiasPairs>(p, grid, stream);                             \
    default:                                                                                            \
      return f32_out ? launch_mode<MD, true, kBiasKeys>(p, grid, stream)                                \
                     : launch_mode<MD, false, kBiasKeys>(p, grid, stream);                              \
  }
      if (a.mode == 0) SWIN_TC_LAUNCH(0)
      SWIN_TC_LAUNCH(1)
#undef SWIN_TC_LAUNCH
    }
    default:
      return f32_out ? launch_mode<2, true, kBiasNone>(p, grid, stream) : launch_mode<2, false, kBiasNone>(p, grid, stream);
  }
}

}  // namespace swin
