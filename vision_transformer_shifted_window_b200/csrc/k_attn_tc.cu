// Shifted-window attention on the Blackwell tensor cores (bf16 inputs, d = 32).
//
// What is computed: for every rectangle (one segment of the shifted partition
// per axis, see swin_index.cuh) of every (image, head), exact softmax attention
// over the rectangle's tokens with the score of the chosen mode —
//   mode 0  q.k/sqrt(d) + T[r][h]        "Swin Transformer V2" eq. 1
//   mode 1  cos(q,k)/max(tau,0.01) + T   same page, eq. 2 (§3.2, §3.3)
//   mode 2  RoPE(q).RoPE(k)/sqrt(d)      FlashSwin abstract (window-local 2-D RoPE)
// — without ever storing a score matrix: FlashSwin's point is that the
// per-window score matrix is the memory problem; here S and P live only in
// TMEM and O in TMEM until it is normalised and stored to its own token.
//
// Work.  One rectangle of one (image, head) is a unit.  Its queries are cut
// into tiles of R = floor(128 / lx) whole rows (<= 128 queries, one TMEM lane
// each), its keys into blocks of Rk = floor(64 / lx) whole rows (<= 64 keys).
// The tiles of all units are listed heads outermost, then images, rows and
// columns of rectangles; each persistent CTA takes a contiguous range of the
// list (cut on the host so that the ranges carry equal work) and hands its
// tiles alternately to its two softmax warpgroups.  Consecutive tiles of one
// unit in a CTA's range form a pass: the unit's K/V blocks are loaded once per
// pass into a ring of shared-memory stages, and every tile of the pass reads
// them there.  When the ring holds all of a unit's blocks plus three, a pass
// is every tile of the unit (the window's K/V stays resident while all its
// query tiles go by); otherwise a pass is at most two tiles, one per
// warpgroup, that stream the blocks together.
//
// Warp roles (512 threads, one persistent CTA per SM):
//   warp 0       K/V producer: TMA 5-D tile loads over [B][H][W][heads][d]
//                (64-byte swizzle, no multicast) into the ring
//   warp 3       Q producer: one TMA load per query tile into that tile's
//                warpgroup's buffers (4, or 2 for long tiles)
//   warps 1, 2   tcgen05.mma S issuers, one thread each: warp 1 + g issues
//                the S = Q K^T MMAs of softmax warpgroup g; warp 1 owns TMEM
//   warps 13, 15 tcgen05.mma PV issuers: warp 13 + 2g issues the O += P V
//                MMAs of softmax warpgroup g
//   warp 12      Q prep: 1/(tau |q|) per row (mode 1), RoPE of q (mode 2)
//   warp 14      K prep: 1/|k| per key (mode 1), RoPE of k (mode 2), V to fp16
//   warps 4-7    softmax of warpgroup 0 (one TMEM lane = one query row)
//   warps 8-11   softmax of warpgroup 1
//
// TMEM per softmax warpgroup g (128 lanes, columns from 256 g): score buffers
// S0, S1 (64 fp32 columns each), probability buffers P0, P1 (64 fp16 keys =
// 32 columns each) and O (48 columns: 32 outputs and, in column 32, the row
// sum of P).  Block b's S = Q K^T lands in S[b % 2]; the softmax copies it to
// registers and frees the buffer at once, so the issuer computes S(b + 2)
// while the softmax works on block b.  P(b) goes to P[b % 2], and
// O += P(b) [V | c] reads it there (c = the constant column 1: the same MMAs
// accumulate the row sum of exactly the fp16 probabilities that weight V).
// The softmax waits for the tensor core only where a buffer comes back two
// blocks later (PV(b - 2) done before P(b) is written), where it rescales O,
// and where it reads a finished O.  S and PV MMAs of a warpgroup come from two
// threads, so an S never queues behind a PV that waits for its probabilities.
//
// A query tile of at most 64 rows is placed in TMEM lanes 64-127 when it
// belongs to warpgroup 1 (lanes 0-63 for warpgroup 0), so that small windows
// keep all four SM sub-partitions busy; warps of a warpgroup without rows in
// the tile follow the barrier protocol but skip the arithmetic.
//
// Softmax: online, with the running maximum kept until a block exceeds it by
// more than 8 (log2 units), so O is rescaled rarely; P in fp16 (values up to
// 2^8): fp16 keeps 3 more mantissa bits than bf16, which the output needs
// (rounding P to bf16 gave about 9 times the output error of fp16).
// Exponentials of the first keys of each block go through a polynomial on
// the FMA pipe and the rest through the MUFU, in a ratio set by
// the measured pipe rates (MUFU 16 exp2 per clock per SM, FMA pipe 128 lanes).
//
// Precision of the score operands: modes 0 and 1 multiply the bf16 inputs as
// they are (mode 1 applies 1/|q|, 1/|k| and 1/tau in fp32 afterwards, so the
// cosine is not rounded); mode 2 rotates q and k in fp32 and stores them as
// fp16 (q scaled by a per-row power of two so that no finite input
// overflows).  V is carried in fp16, the type of P.  A rotated k entry or a V
// entry at or beyond 65504 saturates and records SWIN_ERR_UNSUPPORTED.
//
// Every wait is bounded: on time-out the kernel records SWIN_ERR_TIMEOUT in
// the status word, every role leaves its loop, in-flight copies and MMAs are
// drained with bounded waits, TMEM is freed and the kernel returns.
#include <cuda.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <cstring>
#include <vector>

#include "sm100_ptx.cuh"
#include "swin_common.cuh"

namespace swin {

// Division by a launch constant with a multiply and a shift (Granlund and
// Montgomery's method): n / d = (umulhi(m, n) + n) >> l for n < 2^31, with
// l = ceil(log2 d) and m = floor(2^32 (2^l - d) / d) + 1.
struct FastDiv {
  uint32_t d, m, l;
};

inline FastDiv make_fastdiv(uint32_t d) {
  FastDiv f;
  if (d == 0) d = 1;
  f.d = d;
  f.l = 0;
  while ((1ull << f.l) < d) ++f.l;
  f.m = (uint32_t)(((1ull << 32) * ((1ull << f.l) - d)) / d + 1);
  return f;
}

__host__ __device__ __forceinline__ uint32_t fdiv(uint32_t n, const FastDiv& f) {
#ifdef __CUDA_ARCH__
  return (__umulhi(f.m, n) + n) >> f.l;
#else
  return (uint32_t)((((uint64_t)f.m * n) >> 32) + n) >> f.l;
#endif
}

namespace {

constexpr int kThreads = 512;
constexpr int kMaxCtas = 256;
constexpr int kMaxStages = 32;
constexpr int kMaxQBuf = 4;
constexpr int kTileBytes = 128 * 64;          // Q tile: 128 rows x 32 16-bit values
constexpr int kHalfStage = 64 * 64;           // K or V block: 64 rows x 32 16-bit values
constexpr int kStageBytes = 2 * kHalfStage;   // K then V
constexpr int kBlkKeys = 64;                  // keys per K/V block (TMEM: 2 x 64 + 2 x 32 + 48 columns)
constexpr int kPrepThreads = 32;              // Q prep: warp 12; K prep: warp 14
constexpr int kSmemMax = 227 * 1024;
constexpr int kSmemSlack = 1024;              // for the 1024-byte alignment of the base
constexpr int kRopeBytes = 2 * 2 * 64 * 8 * 4;  // cos, sin [2 axes][64 positions][8]
constexpr float kLog2eF = 1.4426950408889634f;

struct Bars {
  uint64_t q_full[2][kMaxQBuf], q_ready[2][kMaxQBuf], q_empty[2][kMaxQBuf];
  uint64_t kv_full[kMaxStages], kv_ready[kMaxStages], kv_empty[kMaxStages];
  // per warpgroup and buffer; a barrier's next phase needs a step its waiter
  // has not taken yet, so parity waits never alias (see the softmax)
  uint64_t s_full[2][2], s_free[2][2], p_full[2][2], p_free[2][2];
  uint64_t tab_free[2], tab_ready[2];  // bias-table slot handshake of each softmax warpgroup (4 warps)
  uint64_t never, drain[4];
};
constexpr int kNumBars = sizeof(Bars) / 8;

// Shared-memory layout (byte offsets from the 1024-byte aligned base); the
// same function sizes the launch on the host.
struct Layout {
  uint32_t q, kv, ones, rope, qscale, kcol, kofs, kpos, qpos, bias, bars, holder, total;
};

__host__ __device__ inline Layout tc_layout(int nqb, int nst, bool rope, int slot_floats) {
  Layout L;
  uint32_t o = 0;
  L.q = o;
  o += 2u * nqb * kTileBytes;
  L.kv = o;
  o += (uint32_t)nst * kStageBytes;
  L.ones = o;  // 16 rows of [1, 0, ...]: the constant column block of [V | c]
  o += 1024;
  L.rope = o;
  o += rope ? kRopeBytes : 0;
  L.qscale = o;  // [2 warpgroups][kMaxQBuf][128] f32
  o += 2 * kMaxQBuf * 128 * 4;
  L.kcol = o;  // [stage][64] f32: 1/|k| (mode 1)
  o += (uint32_t)nst * kBlkKeys * 4;
  L.kofs = o;  // [3 classes][64] int: bias-slot offset of key c of a block
  o += 3 * kBlkKeys * 4;
  L.kpos = o;  // [3][64] int: (c / lx) | (c % lx) << 16
  o += 3 * kBlkKeys * 4;
  L.qpos = o;  // [3][128] int: (r / lx) | (r % lx) << 16
  o += 3 * 128 * 4;
  // Bias slots come after at least three ring stages: the unconditional bias
  // loads of masked keys may read up to 64 slot rows before slot 0.
  L.bias = o;
  o += 2u * (uint32_t)slot_floats * 4;
  L.bars = (o + 7) & ~7u;
  o = L.bars + kNumBars * 8;
  L.holder = o;  // TMEM base, abort flag, drain flag
  o += 16;
  L.total = o;
  return L;
}

}  // namespace

struct TcParams {
  CUtensorMap tmq[3], tmqh[3], tmk[3], tmv[3];  // per x-class: Q (R rows), Q (Rh rows), K, V (Rk rows)
  FastDiv div_img, div_B, div_rowmid, div_colmid[3];
  int lx[3], R[3], Rh[3], Rk[3];    // per x-class: width, rows per Q tile / half tile / K-V block
  int row_ly[3], row_tiles[3];      // per row class: height, tiles in one row of rectangles
  int rect_tiles[3][3], rect_nb[3][3];
  int nsy, nsx;
  int B, H, W, heads, M, s;
  int R2e, copy1, slot_floats;      // bias slot: row stride, offset of the shifted copy, floats per slot
  int nst, nqb, max_pass_tiles;     // ring stages, Q buffers per warpgroup, tiles per pass
  int n_ctas;
  int cta_start[kMaxCtas + 1];      // CTA c takes tiles [cta_start[c], cta_start[c + 1])
  void* out;
  const float* tau;
  const float* table;
  const float* rope;
  int* status;
  long long wait_limit;  // clock64 cycles before a wait gives up
  int debug_flags;       // bit 0: force a time-out (test of the failure path)
};

namespace {

// One unit (rectangle of one (image, head)) and a pass over it.
struct Unit {
  int h, b, cls, y0, ly, x0, lx, R, Rh, Rk, ntile, nb;
};

struct Pass {
  Unit u;
  int k0, n;  // tiles k0 .. k0 + n - 1 of the unit
};

__host__ __device__ __forceinline__ Unit decode_tile(const TcParams& p, uint32_t t, int& k) {
  Unit u;
  const uint32_t ih = fdiv(t, p.div_img);  // h * B + b
  uint32_t rem = t - ih * p.div_img.d;
  const uint32_t hq = fdiv(ih, p.div_B);
  u.h = (int)hq;
  u.b = (int)(ih - hq * p.div_B.d);
  int sy, rc;
  if (rem < (uint32_t)p.row_tiles[0]) {
    sy = 0;
    rc = 0;
  } else {
    rem -= (uint32_t)p.row_tiles[0];
    const uint32_t mid = p.nsy > 2 ? (uint32_t)(p.nsy - 2) * (uint32_t)p.row_tiles[1] : 0u;
    if (rem < mid) {
      const uint32_t r = fdiv(rem, p.div_rowmid);
      sy = 1 + (int)r;
      rc = 1;
      rem -= r * (uint32_t)p.row_tiles[1];
    } else {
      sy = p.nsy - 1;
      rc = 2;
      rem -= mid;
    }
  }
  int sx, cls;
  if (p.nsx == 1 || rem < (uint32_t)p.rect_tiles[rc][0]) {
    sx = 0;
    cls = 0;
  } else {
    rem -= (uint32_t)p.rect_tiles[rc][0];
    const uint32_t mid = p.nsx > 2 ? (uint32_t)(p.nsx - 2) * (uint32_t)p.rect_tiles[rc][1] : 0u;
    if (rem < mid) {
      const uint32_t r = fdiv(rem, p.div_colmid[rc]);
      sx = 1 + (int)r;
      cls = 1;
      rem -= r * (uint32_t)p.rect_tiles[rc][1];
    } else {
      sx = p.nsx - 1;
      cls = 2;
      rem -= mid;
    }
  }
  k = (int)rem;
  u.cls = cls;
  u.y0 = swin_seg_start(sy, p.M, p.s);
  u.ly = p.row_ly[rc];
  u.x0 = swin_seg_start(sx, p.M, p.s);
  u.lx = p.lx[cls];
  u.R = p.R[cls];
  u.Rh = p.Rh[cls];
  u.Rk = p.Rk[cls];
  u.ntile = p.rect_tiles[rc][cls];
  u.nb = p.rect_nb[rc][cls];
  return u;
}

__device__ __forceinline__ Pass pass_at(const TcParams& p, uint32_t t, uint32_t t_end) {
  Pass ps;
  ps.u = decode_tile(p, t, ps.k0);
  int n = ps.u.ntile - ps.k0;
  n = min(n, (int)(t_end - t));
  ps.n = min(n, p.max_pass_tiles);
  return ps;
}

__device__ __forceinline__ int tile_rows(const Unit& u, int k) { return min(u.R, u.ly - k * u.R); }
__device__ __forceinline__ bool tile_half(const Unit& u, int k) { return tile_rows(u, k) <= u.Rh; }
__device__ __forceinline__ int block_rows(const Unit& u, int j) { return min(u.Rk, u.ly - j * u.Rk); }

// Position in a ring of n slots: slot and the parity of the round.
struct Ring {
  uint32_t slot, ph;
};
__device__ __forceinline__ void ring_next(Ring& r, uint32_t n) {
  if (++r.slot == n) {
    r.slot = 0;
    r.ph ^= 1u;
  }
}
__device__ __forceinline__ Ring ring_adv(Ring r, uint32_t k, uint32_t n) {
  const uint32_t s = r.slot + k, q = s / n;
  r.slot = s - q * n;
  r.ph ^= q & 1u;
  return r;
}

// A softmax warpgroup's walk over its blocks: passes in order, the
// warpgroup's tiles of each pass, the blocks of each tile.
struct Walk {
  uint32_t t;  // first tile of the current pass
  Pass ps;
  int i, j;    // tile of the pass, block of the tile
  Ring base;   // ring position of the pass's block 0
  bool valid;
};

// Move to the first tile of warpgroup g at or after tile i of the current pass.
__device__ __forceinline__ void walk_seek(Walk& w, const TcParams& p, uint32_t t_begin, uint32_t t_end, int g,
                                          uint32_t nst) {
  while (true) {
    while (w.i < w.ps.n && (int)((w.t + w.i - t_begin) & 1u) != g) ++w.i;
    if (w.i < w.ps.n) return;
    w.base = ring_adv(w.base, w.ps.u.nb, nst);
    w.t += w.ps.n;
    if (w.t >= t_end) {
      w.valid = false;
      return;
    }
    w.ps = pass_at(p, w.t, t_end);
    w.i = 0;
  }
}

__device__ __forceinline__ void walk_init(Walk& w, const TcParams& p, uint32_t t_begin, uint32_t t_end, int g,
                                          uint32_t nst) {
  w.t = t_begin;
  w.base = Ring{0, 0};
  w.i = w.j = 0;
  w.valid = t_begin < t_end;
  if (w.valid) {
    w.ps = pass_at(p, t_begin, t_end);
    walk_seek(w, p, t_begin, t_end, g, nst);
  }
}

__device__ __forceinline__ void walk_next(Walk& w, const TcParams& p, uint32_t t_begin, uint32_t t_end, int g,
                                          uint32_t nst) {
  if (++w.j < w.ps.u.nb) return;
  w.j = 0;
  ++w.i;
  walk_seek(w, p, t_begin, t_end, g, nst);
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

// Registers written by an asynchronous tcgen05.ld are only valid after
// tcgen05.wait::ld; this empty asm "rewrites" them after the wait, so that no
// use can be scheduled before it.
__device__ __forceinline__ void reg_fence32(uint32_t* r) {
  asm volatile(""
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                 "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]),
                 "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]),
                 "+r"(r[29]), "+r"(r[30]), "+r"(r[31]));
}

// ------------------------------------------------------------------ prep
// Mode 2 feeds the score MMA fp16 operands (both Q and K, one type): fp16
// keeps 3 more mantissa bits than bf16, and rounding the rotated operands is
// the largest error term of that mode.  A rotated Q row is first scaled by an
// exact power of two that brings it below 2^15 (divided out in the softmax);
// rotated K rows are converted with saturation, and an entry at or beyond the
// fp16 range is reported as unsupported.

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

// 2^e for a pair on the FMA pipe, so that part of the exponentials leave the
// MUFU: e = j + f with j = rint(e) read from the low mantissa bits of
// e + 1.5 * 2^23 and f in [-1/2, 1/2]; 2^f is a degree-3 polynomial fitted by
// the Remez exchange algorithm for minimax relative error on [-1/2, 1/2]
// (7.5e-5, below half an fp16 ulp), and j is added to its exponent field.
// Arguments below -125 are clamped (the result is then at most 2^-125).
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

// How a launch adds the relative bias (a template argument, so that each
// kernel carries only the code it runs): no table; pair loads (every
// rectangle width of the launch even); one load per key (some width odd).
enum BiasKind { kBiasNone = 0, kBiasPairs = 1, kBiasKeys = 2 };

// Keys of a 64-key block whose exponentials go through the FMA-pipe
// polynomial (the first ones; the rest, including any masked tail keys,
// through the MUFU).  Mode 2 has no per-element bias work, so the FMA pipe
// can take a larger share.
template <int MODE>
struct ExpSplit {
  static constexpr int kPoly = MODE == 2 ? 24 : 16;
};

// ------------------------------------------------------------------ kernel
template <int MODE, bool OUT_F32, int BIAS>
__global__ void __launch_bounds__(kThreads, 1) attn_tc_kernel(const __grid_constant__ TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment by pointer arithmetic on the shared array itself, so
  // that every access below stays a shared-space load or store
  uint8_t* smem = smem_raw + ((1024u - (static_cast<uint32_t>(__cvta_generic_to_shared(smem_raw)) & 1023u)) & 1023u);
  const int nst = p.nst, nqb = p.nqb;
  constexpr bool has_table = MODE != 2 && BIAS != kBiasNone;
  const Layout L = tc_layout(nqb, nst, MODE == 2, has_table ? p.slot_floats : 0);
  uint8_t* qbuf = smem + L.q;
  uint8_t* kvbuf = smem + L.kv;
  uint8_t* ones = smem + L.ones;
  float* rcos = reinterpret_cast<float*>(smem + L.rope);
  float* rsin = rcos + 2 * 64 * 8;
  float* qscale = reinterpret_cast<float*>(smem + L.qscale);
  float* kcol = reinterpret_cast<float*>(smem + L.kcol);
  int* kofs = reinterpret_cast<int*>(smem + L.kofs);
  int* kpos = reinterpret_cast<int*>(smem + L.kpos);
  int* qpos = reinterpret_cast<int*>(smem + L.qpos);
  float* sbias = reinterpret_cast<float*>(smem + L.bias);  // [2 warpgroups][slot_floats]
  Bars* bars = reinterpret_cast<Bars*>(smem + L.bars);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L.holder);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int M = p.M, s = p.s;
  const uint32_t t_begin = (uint32_t)p.cta_start[blockIdx.x], t_end = (uint32_t)p.cta_start[blockIdx.x + 1];

  // ---- set-up: barriers, RoPE tables, index tables, constant column, TMEM
  if (threadIdx.x == 0) {
    for (int g = 0; g < 2; ++g)
      for (int b = 0; b < kMaxQBuf; ++b) {
        ptx::mbar_init(&bars->q_full[g][b], 1);
        ptx::mbar_init(&bars->q_ready[g][b], kPrepThreads);
        ptx::mbar_init(&bars->q_empty[g][b], 1 + 4);  // last S MMA of the tile + 4 softmax warps
      }
    for (int i = 0; i < kMaxStages; ++i) {
      ptx::mbar_init(&bars->kv_full[i], 1);
      ptx::mbar_init(&bars->kv_ready[i], kPrepThreads);
      ptx::mbar_init(&bars->kv_empty[i], 2);  // one release per softmax warpgroup
    }
    for (int g = 0; g < 2; ++g) {
      for (int b = 0; b < 2; ++b) {
        ptx::mbar_init(&bars->s_full[g][b], 1);
        ptx::mbar_init(&bars->s_free[g][b], 4);
        ptx::mbar_init(&bars->p_full[g][b], 4);
        ptx::mbar_init(&bars->p_free[g][b], 1);
      }
      ptx::mbar_init(&bars->tab_free[g], 4);
      ptx::mbar_init(&bars->tab_ready[g], 4);
    }
    ptx::mbar_init(&bars->never, 1);
    for (int i = 0; i < 4; ++i) ptx::mbar_init(&bars->drain[i], 1);
    *abort_flag = 0;
    tmem_holder[2] = 0;  // abort flag of the drain waits (never set by a role)
    ptx::fence_mbar_init();
  }
  if (MODE == 2) {
    for (int i = threadIdx.x; i < 2 * 64 * 8; i += kThreads) {
      const int axis = i / (64 * 8), pos = (i / 8) % 64, t = i % 8;
      float sv = 0.f, cv = 1.f;
      if (pos < M) sincosf((float)pos * p.rope[axis * 8 + t], &sv, &cv);
      rcos[(axis * 64 + pos) * 8 + t] = cv;
      rsin[(axis * 64 + pos) * 8 + t] = sv;
    }
  }
  for (int i = threadIdx.x; i < 3 * 128; i += kThreads) {
    const int c = i / 128, r = i % 128, lx = p.lx[c];
    qpos[i] = (r / lx) | ((r % lx) << 16);
    if (r < kBlkKeys) {
      kofs[c * kBlkKeys + r] = (r / lx) * p.R2e + (r % lx);
      kpos[c * kBlkKeys + r] = (r / lx) | ((r % lx) << 16);
    }
  }
  // zero the K/V ring and the constant block once, so rows a block never
  // writes hold finite values
  for (int i = threadIdx.x; i < (nst * kStageBytes + 1024) / 16; i += kThreads)
    reinterpret_cast<uint4*>(kvbuf)[i] = make_uint4(0, 0, 0, 0);
  __syncthreads();
  // the constant column: fp16 1.0 in the first column of 16 rows
  if (threadIdx.x < 16) *reinterpret_cast<uint16_t*>(ones + swz64(threadIdx.x, 0)) = 0x3C00;
  if (warp == 1) {
    ptx::tmem_alloc(tmem_holder, 512);
    ptx::tmem_relinquish();
  }
  if (warp == 0 && lane == 0)
    for (int c = 0; c < 3; ++c) {
      ptx::prefetch_tmap(&p.tmq[c]);
      ptx::prefetch_tmap(&p.tmqh[c]);
      ptx::prefetch_tmap(&p.tmk[c]);
      ptx::prefetch_tmap(&p.tmv[c]);
    }
  ptx::fence_proxy_async_smem();
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  Ctl ctl{abort_flag, &p};
  Ctl drain{reinterpret_cast<volatile int*>(tmem_holder + 2), &p};

  // Register split: warpgroups 0 (producers, issuers) and 3 (prep) give
  // registers to the two softmax warpgroups: 512 x 128 = 256 x 64 + 256 x 192.
  if (warp < 4 || warp >= 12) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 64;\n" ::: "memory");
    if (warp == 0) {
      // ============================================================ K/V producer
      if (lane == 0) {
        Ring w{0, 0};
        uint32_t loads = 0;
        bool ok = true;
        for (uint32_t t = t_begin; t < t_end && ok;) {
          const Pass ps = pass_at(p, t, t_end);
          const Unit& u = ps.u;
          for (int j = 0; j < u.nb && ok; ++j) {
            if (loads >= (uint32_t)nst) ok = wait_bar(&bars->kv_empty[w.slot], w.ph ^ 1u, ctl);
            if (!ok) break;
            uint8_t* dst = kvbuf + w.slot * kStageBytes;
            ptx::mbar_arrive_expect_tx(&bars->kv_full[w.slot], (uint32_t)(2 * 64 * u.lx * u.Rk));
            ptx::tma_load_5d(dst, &p.tmk[u.cls], &bars->kv_full[w.slot], 0, u.h, u.x0, u.y0 + j * u.Rk, u.b);
            ptx::tma_load_5d(dst + kHalfStage, &p.tmv[u.cls], &bars->kv_full[w.slot], 0, u.h, u.x0,
                             u.y0 + j * u.Rk, u.b);
            ring_next(w, nst);
            ++loads;
          }
          t += ps.n;
        }
        // copies still landing in shared memory (after an abort; in a normal
        // exit every one of them has been waited for by the K prep)
        const uint32_t m = loads < (uint32_t)nst ? loads : (uint32_t)nst;
        Ring d = ring_adv(Ring{0, 0}, loads - m, nst);
        for (uint32_t i = 0; i < m; ++i, ring_next(d, nst)) wait_bar(&bars->kv_full[d.slot], d.ph, drain);
      }
    } else if (warp == 3) {
      // ============================================================ Q producer
      if (lane == 0) {
        Ring qr[2] = {{0, 0}, {0, 0}};
        uint32_t qn[2] = {0, 0};
        bool ok = true;
        for (uint32_t t = t_begin; t < t_end && ok;) {
          const Pass ps = pass_at(p, t, t_end);
          const Unit& u = ps.u;
          for (int i = 0; i < ps.n && ok; ++i) {
            const int g = (int)((t + i - t_begin) & 1u), k = ps.k0 + i;
            if (qn[g] >= (uint32_t)nqb) ok = wait_bar(&bars->q_empty[g][qr[g].slot], qr[g].ph ^ 1u, ctl);
            if (!ok) break;
            const bool half = tile_half(u, k);
            uint8_t* dst = qbuf + (g * nqb + qr[g].slot) * kTileBytes + (half ? g * 4096 : 0);
            ptx::mbar_arrive_expect_tx(&bars->q_full[g][qr[g].slot], (uint32_t)(64 * u.lx * (half ? u.Rh : u.R)));
            ptx::tma_load_5d(dst, half ? &p.tmqh[u.cls] : &p.tmq[u.cls], &bars->q_full[g][qr[g].slot], 0, u.h,
                             u.x0, u.y0 + k * u.R, u.b);
            ring_next(qr[g], nqb);
            ++qn[g];
          }
          t += ps.n;
        }
        for (int g = 0; g < 2; ++g) {
          const uint32_t m = qn[g] < (uint32_t)nqb ? qn[g] : (uint32_t)nqb;
          Ring d = ring_adv(Ring{0, 0}, qn[g] - m, nqb);
          for (uint32_t i = 0; i < m; ++i, ring_next(d, nqb)) wait_bar(&bars->q_full[g][d.slot], d.ph, drain);
        }
      }
    } else if (warp == 1 || warp == 2 || warp == 13 || warp == 15) {
      // ============================================================ MMA issuers
      // Two issuer threads per softmax warpgroup g: warp 1 + g issues its S
      // MMAs, warp 13 + 2g its PV MMAs.  S and PV never touch the same TMEM
      // columns, and every dependence between them goes through the softmax
      // (S(b) -> softmax -> P(b) -> PV(b)), so they need no common order: an
      // S MMA never waits behind a PV whose probabilities are not written yet.
      if (lane == 0) {
        const bool s_role = warp < 4;
        const int g = s_role ? warp - 1 : (warp - 13) >> 1;
        const uint32_t tg = tmem_base + g * 256;
        bool ok = true;
        if (s_role) {
          // mode 2 feeds fp16 score operands (see prep), modes 0 and 1 the bf16 inputs
          constexpr uint32_t fmtS = MODE == 2 ? 0u : 1u;
          constexpr uint32_t idS = ptx::idesc_f16(fmtS, fmtS, 0, 0, kBlkKeys, 128);
          // Operand descriptors (64-byte swizzle) of this warpgroup's Q buffer
          // 0 and of K stage 0; the others differ only in the start-address
          // field (16-byte units).
          const uint64_t qd0 =
              ptx::smem_desc(ptx::smem_addr(qbuf + g * nqb * kTileBytes), 16, 512, ptx::kSwizzle64B);
          const uint64_t kd0 = ptx::smem_desc(ptx::smem_addr(kvbuf), 16, 512, ptx::kSwizzle64B);
          constexpr uint64_t kQBuf = kTileBytes >> 4;
          constexpr uint64_t kStageK = kStageBytes >> 4;
          if (g == 0 && (p.debug_flags & 1)) ok = wait_bar(&bars->never, 0, ctl);  // forced time-out
          Ring qr{0, 0}, base{0, 0};
          uint32_t b = 0;
          for (uint32_t t = t_begin; t < t_end && ok;) {
            const Pass ps = pass_at(p, t, t_end);
            const Unit& u = ps.u;
            for (int i = 0; i < ps.n && ok; ++i) {
              if ((int)((t + i - t_begin) & 1u) != g) continue;
              Ring w = base;
              for (int j = 0; j < u.nb; ++j, ++b, ring_next(w, nst)) {
                // S(b) into S[b % 2]: the softmax has copied S(b - 2) out
                if (b >= 2) ok = wait_bar(&bars->s_free[g][b & 1], ((b - 2) >> 1) & 1, ctl);
                ok = ok && (j > 0 || wait_bar(&bars->q_ready[g][qr.slot], qr.ph, ctl)) &&
                     wait_bar(&bars->kv_ready[w.slot], w.ph, ctl);
                if (!ok) break;
                ptx::tc_fence_after();
                const uint64_t ad = qd0 + qr.slot * kQBuf, bd = kd0 + w.slot * kStageK;
                const uint32_t dS = tg + (b & 1) * 64;
                ptx::mma_ss(dS, ad, bd, idS, 0);
                ptx::mma_ss(dS, ad + 2, bd + 2, idS, 1);  // second 16-wide K step: +32 bytes
                ptx::mma_commit(&bars->s_full[g][b & 1]);
                if (j == u.nb - 1) {
                  ptx::mma_commit(&bars->q_empty[g][qr.slot]);
                  ring_next(qr, nqb);
                }
              }
            }
            base = ring_adv(base, u.nb, nst);
            t += ps.n;
          }
        } else {
          constexpr uint32_t idPV = ptx::idesc_f16(0, 0, 0, 1, 48, 128);  // fp16 P (TMEM) x fp16 [V | c]
          // [V | c] of V stage 0: the constant column block sits after the
          // ring (N columns 32-47), at the leading byte offset; other stages
          // and k-steps move the start address and shorten that offset.
          const uint32_t va0 = ptx::smem_addr(kvbuf + kHalfStage), oa0 = ptx::smem_addr(ones);
          const uint64_t vd0 = ptx::smem_desc(va0, oa0 - va0, 512, ptx::kSwizzle64B);
          constexpr uint64_t kStageK = kStageBytes >> 4;
          constexpr uint64_t kStageV = kStageK - (kStageK << 16);
          // k-step kk of PV: V rows 16 kk.. (+1024 bytes), constant block unchanged
          constexpr uint64_t kStepV = (uint64_t)(1024 >> 4) - ((uint64_t)(1024 >> 4) << 16);
          Ring base{0, 0};
          uint32_t b = 0;
          for (uint32_t t = t_begin; t < t_end && ok;) {
            const Pass ps = pass_at(p, t, t_end);
            const Unit& u = ps.u;
            int last_i = -1;  // this warpgroup's last tile in the pass
            for (int i = 0; i < ps.n; ++i)
              if ((int)((t + i - t_begin) & 1u) == g) last_i = i;
            for (int i = 0; i < ps.n && ok; ++i) {
              if ((int)((t + i - t_begin) & 1u) != g) continue;
              // a block used by this warpgroup's last tile of the pass is
              // released after its PV; by both releases when the other
              // warpgroup has no tile in the pass
              const uint32_t rel = i == last_i ? (ps.n == 1 ? 2u : 1u) : 0u;
              Ring w = base;
              for (int j = 0; j < u.nb; ++j, ++b, ring_next(w, nst)) {
                // PV(b): its P is written once the softmax has released it
                ok = wait_bar(&bars->p_full[g][b & 1], (b >> 1) & 1, ctl);
                if (!ok) break;
                ptx::tc_fence_after();
                const uint64_t vd = vd0 + w.slot * kStageV;
                const uint32_t aP = tg + 128 + (b & 1) * 32;
                const uint32_t nch = (uint32_t)(block_rows(u, j) * u.lx + 15) >> 4;
                for (uint32_t kk = 0; kk < nch; ++kk)
                  ptx::mma_ts(tg + 192, aP + kk * 8, vd + kk * kStepV, idPV, (kk > 0 || j > 0) ? 1u : 0u);
                ptx::mma_commit(&bars->p_free[g][b & 1]);
                for (uint32_t r = 0; r < rel; ++r) ptx::mma_commit(&bars->kv_empty[w.slot]);
              }
            }
            base = ring_adv(base, u.nb, nst);
            t += ps.n;
          }
        }
        // drain: every MMA this thread issued has completed before TMEM is freed
        const int di = s_role ? g : 2 + g;
        ptx::mma_commit(&bars->drain[di]);
        wait_bar(&bars->drain[di], 0, drain);
      }
    } else if (warp == 12) {
      // ============================================================ Q prep
      // 32 threads; work in half rows (16 channels): the two halves of a row
      // sit in adjacent lanes, and each half of a RoPE row rotates along one
      // axis only.  Trip counts are uniform per warp (shuffles need all lanes).
      const int pt = lane;
      Ring qr[2] = {{0, 0}, {0, 0}};
      bool ok = true;
      for (uint32_t t = t_begin; t < t_end && ok;) {
        const Pass ps = pass_at(p, t, t_end);
        const Unit& u = ps.u;
        const float te = MODE == 1 ? fmaxf(__ldg(p.tau + u.h), kTauMin) : 1.f;
        const int* qp = qpos + u.cls * 128;
        for (int i = 0; i < ps.n && ok; ++i) {
          const int g = (int)((t + i - t_begin) & 1u), k = ps.k0 + i;
          const uint32_t qs = qr[g].slot;
          ok = __all_sync(0xffffffffu, wait_bar(&bars->q_full[g][qs], qr[g].ph, ctl));
          ring_next(qr[g], nqb);
          if (!ok) break;
          if (MODE != 0) {
            const int loff = tile_half(u, k) ? 64 * g : 0, nq = tile_rows(u, k) * u.lx;
            uint8_t* tile = qbuf + (g * nqb + qs) * kTileBytes;
            float* qsc = qscale + (g * kMaxQBuf + qs) * 128;
#pragma unroll 1
            for (int un = pt; un < 2 * 128; un += kPrepThreads) {
              const int r = un >> 1, h = un & 1, row = loff + r;
              const bool act = r < nq;
              float v[16];
              if (act) load_half_bf16(tile, row, h, v);
              else for (int e = 0; e < 16; ++e) v[e] = 0.f;
              if (MODE == 1) {
                float ss = half_sumsq(v);
                ss += __shfl_xor_sync(0xffffffffu, ss, 1);
                if (act && h == 0) qsc[row] = kLog2eF / (fmaxf(sqrtf(ss), kNormEps) * te);
              } else {
                if (act) {
                  const int pr = qp[r];
                  const int pos = h ? swin_local_coord(u.x0 + (pr >> 16), M, s)
                                    : swin_local_coord(u.y0 + k * u.R + (pr & 0xFFFF), M, s);
                  rope_half(v, h, pos, rcos, rsin);
                }
                float mx = half_absmax(v);
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
                const float sc = pow2_scale(mx);  // exact per-row scale, undone in the softmax
                if (act) {
                  store_half_f16(tile, row, h, v, sc);
                  if (h == 0) qsc[row] = kLog2eF * rsqrtf(32.0f) / sc;
                }
              }
            }
            ptx::fence_proxy_async_smem();
          }
          ptx::mbar_arrive(&bars->q_ready[g][qs]);
        }
        t += ps.n;
      }
    } else {
      // ============================================================ K prep
      const int pk = lane;
      Ring w{0, 0};
      bool ok = true;
      bool range_hit = false;  // a rotated K or a V entry saturated the fp16 range
      for (uint32_t t = t_begin; t < t_end && ok;) {
        const Pass ps = pass_at(p, t, t_end);
        const Unit& u = ps.u;
        const int* kp = kpos + u.cls * kBlkKeys;
        for (int j = 0; j < u.nb && ok; ++j, ring_next(w, nst)) {
          ok = __all_sync(0xffffffffu, wait_bar(&bars->kv_full[w.slot], w.ph, ctl));
          if (!ok) break;
          {
            const int nk = block_rows(u, j) * u.lx;
            uint8_t* ktile = kvbuf + w.slot * kStageBytes;
            uint8_t* vtile = ktile + kHalfStage;
            // units: half h of K row r and half h of V row r (r < nk <= 64);
            // fp16 with saturation, a saturated entry is reported after the
            // loop.  Trip counts are uniform per warp (the shuffle needs all lanes).
#pragma unroll 1
            for (int un = pk; un < 2 * kBlkKeys; un += kPrepThreads) {
              const int r = un >> 1, h = un & 1;
              const bool act = r < nk;
              if (MODE != 0) {
                float v[16];
                if (act) load_half_bf16(ktile, r, h, v);
                else for (int e = 0; e < 16; ++e) v[e] = 0.f;
                if (MODE == 1) {
                  float ss = half_sumsq(v);
                  ss += __shfl_xor_sync(0xffffffffu, ss, 1);
                  if (act && h == 0) kcol[w.slot * kBlkKeys + r] = 1.0f / fmaxf(sqrtf(ss), kNormEps);
                } else if (act) {
                  const int pr = kp[r];
                  const int pos = h ? swin_local_coord(u.x0 + (pr >> 16), M, s)
                                    : swin_local_coord(u.y0 + j * u.Rk + (pr & 0xFFFF), M, s);
                  rope_half(v, h, pos, rcos, rsin);
                  range_hit |= half_absmax(v) >= 65504.0f;
                  store_half_f16(ktile, r, h, v, 1.0f);
                }
              }
              if (act) {
                float v[16];
                load_half_bf16(vtile, r, h, v);
                range_hit |= half_absmax(v) >= 65504.0f;
                store_half_f16(vtile, r, h, v, 1.0f);
              }
            }
            ptx::fence_proxy_async_smem();
          }
          ptx::mbar_arrive(&bars->kv_ready[w.slot]);
        }
        t += ps.n;
      }
      if (range_hit) atomicOr(p.status, (int)SWIN_ERR_UNSUPPORTED);
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 192;\n" ::: "memory");
    // ================================================================ softmax
    // Software-pipelined over this warpgroup's blocks: while block b is
    // computed from registers, S(b + 1) is already being copied out of TMEM
    // into the other register set, and P(b)'s store lands while the next
    // block starts (its p_full arrival is deferred to the top of block b + 1).
    // O is touched (rescale, deferred epilogue) at the end of a block, after
    // P(b) is stored, which leaves PV(b - 1) the most time to complete.  The
    // loop body alternates the two register sets.
    const int g = (warp - 4) >> 2;  // warpgroup 0 or 1
    const int wq = warp & 3;        // TMEM lanes 32 wq .. 32 wq + 31
    const uint32_t tX = tmem_base + g * 256 + ((uint32_t)(wq * 32) << 16);
    const uint32_t tO = tX + 192;
    const float cscale = kLog2eF * rsqrtf(32.0f);
    float* slot = sbias + g * p.slot_floats;
    const int R2e = p.R2e, copy1 = p.copy1;
    int cur_h = -1;
    uint32_t tabn = 0;  // table loads of this warpgroup
    Ring qr{0, 0};
    bool ok = true;
    bool pend = false, pend_ok = false;  // a tile's O still waiting in TMEM (this warp's rows)
    size_t pend_off = 0;
    // O / l of one row to global memory (32 values; column 32 holds l)
    auto store_rows = [&](const uint32_t (&o)[32], uint32_t l, size_t off, bool row_valid) {
      if (!row_valid) return;
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
    // PV completions: p_free[x] completes once per PV of a block b with
    // b % 2 == x.  A wait for PV(k), k < the current block, cannot alias a
    // later phase: PV(k + 2) needs P(k + 2), which this warp has not released.
    uint32_t pv_done = 0;  // PVs of this warpgroup known complete
    auto wait_pv = [&](uint32_t upto) -> bool {  // PV(0..upto) complete
      bool r = true;
      while (r && pv_done <= upto) {
        r = wait_bar(&bars->p_free[g][pv_done & 1], (pv_done >> 1) & 1, ctl);
        r = __all_sync(0xffffffffu, r);
        ++pv_done;
      }
      ptx::tc_fence_after();
      return r;
    };
    // tile state
    bool active = false, row_ok = false;
    int qy = 0, qx = 0, bbase = 0;
    float alpha = 0.f, m_run = -INFINITY;
    const float* pbase = slot;
    uint32_t b = 0;            // blocks of this warpgroup
    bool p_pending = false;    // P(b - 1) stored; its p_full arrival not made yet
    Walk wk;
    walk_init(wk, p, t_begin, t_end, g, nst);
    uint32_t n_blocks = 0;  // blocks of this warpgroup in the CTA's range
    for (uint32_t t = t_begin; t < t_end;) {
      const Pass ps = pass_at(p, t, t_end);
      int mine = 0;
      for (int i = 0; i < ps.n; ++i) mine += (int)((t + i - t_begin) & 1u) == g;
      n_blocks += (uint32_t)(mine * ps.u.nb);
      t += ps.n;
    }
    uint32_t xs[2][kBlkKeys];  // two register sets of scores (this block, the next)

    auto arrive_p = [&]() {  // the deferred p_full of block b - 1
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&bars->p_full[g][(b - 1) & 1]);
      p_pending = false;
    };

    if (wk.valid) {
      // prologue: S(0) into registers
      ok = __all_sync(0xffffffffu, wait_bar(&bars->s_full[g][0], 0, ctl));
      if (ok) {
        ptx::tc_fence_after();
        ptx::tmem_ld32(tX, *reinterpret_cast<uint32_t(*)[32]>(&xs[0][0]));
        ptx::tmem_ld32(tX + 32, *reinterpret_cast<uint32_t(*)[32]>(&xs[0][32]));
        ptx::tmem_wait_ld();
        reg_fence32(&xs[0][0]);
        reg_fence32(&xs[0][32]);
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&bars->s_free[g][0]);
      }
    }
#pragma unroll 1
    while (ok && wk.valid) {
      // two blocks per trip, so that the register sets alternate statically
#pragma unroll
      for (int pp = 0; pp < 2; ++pp) {
        if (ok && wk.valid) {
          uint32_t* xc = xs[pp];
          uint32_t* xn = xs[pp ^ 1];
          const bool has_next = b + 1 < n_blocks;
          if (has_next) {
            // S(b + 1) was issued while block b - 1 was computed
            ok = __all_sync(0xffffffffu, wait_bar(&bars->s_full[g][(b + 1) & 1], ((b + 1) >> 1) & 1, ctl));
            if (ok) {
              ptx::tc_fence_after();
              const uint32_t tSn = tX + ((b + 1) & 1) * 64;
              ptx::tmem_ld32(tSn, *reinterpret_cast<uint32_t(*)[32]>(xn));
              ptx::tmem_ld32(tSn + 32, *reinterpret_cast<uint32_t(*)[32]>(xn + 32));
            }
          }
          // the previous block's P store has had a block boundary to land:
          // release it to the issuer
          if (ok && p_pending) arrive_p();
          const Unit& u = wk.ps.u;
          const int j = wk.j;
          if (ok && j == 0) {
            // ---- new tile: bias table of its head, row scale, row position
            if (has_table && u.h != cur_h) {
              // new head: once all four warps are done with the old table,
              // each loads a quarter of the new one (times log2 e, zero
              // padding columns)
              __syncwarp();
              if (lane == 0) ptx::mbar_arrive(&bars->tab_free[g]);
              ok = __all_sync(0xffffffffu, wait_bar(&bars->tab_free[g], tabn & 1, ctl));
              if (ok) {
                const int n = (2 * M - 1) * R2e;
                for (int i = wq * 32 + lane; i < n; i += 128) {
                  const int dy = i / R2e, c = i - dy * R2e;
                  const float v = c < 2 * M - 1
                                      ? __ldg(p.table + (size_t)(dy * (2 * M - 1) + c) * p.heads + u.h) * kLog2eF
                                      : 0.f;
                  slot[i] = v;
                  if (i > 0) slot[copy1 + i - 1] = v;
                }
                if (wq == 0 && lane == 0) slot[copy1 + n - 1] = 0.f;
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&bars->tab_ready[g]);
                ok = __all_sync(0xffffffffu, wait_bar(&bars->tab_ready[g], tabn & 1, ctl));
                ++tabn;
                cur_h = u.h;
              }
            }
            const int k = wk.ps.k0 + wk.i;
            const int loff = tile_half(u, k) ? 64 * g : 0, nq = tile_rows(u, k) * u.lx;
            active = wq * 32 + 31 >= loff && wq * 32 < loff + nq;  // warp-uniform
            const int r = wq * 32 + lane - loff;                    // query row in the tile
            row_ok = r >= 0 && r < nq;
            const int rr = min(max(r, 0), 127);
            const int* qp = qpos + u.cls * 128;
            qy = k * u.R + (qp[rr] & 0xFFFF);  // position in the rectangle
            qx = qp[rr] >> 16;
            const uint32_t qs = qr.slot;
            if (ok && MODE != 0) ok = __all_sync(0xffffffffu, wait_bar(&bars->q_ready[g][qs], qr.ph, ctl));
            // per-row score scale: mode 1 log2e / (tau |q|), mode 2 log2e / (sqrt(d) 2^e)
            alpha = MODE == 0 ? cscale : qscale[(g * kMaxQBuf + qs) * 128 + wq * 32 + lane];
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&bars->q_empty[g][qs]);
            ring_next(qr, nqb);
            // Slot index of this row's bias for key (0, 0) of the rectangle;
            // the pair load for keys (2c, 2c+1) of a row starts one float
            // earlier, in copy 0 when that index is even, else in copy 1 (the
            // parity is fixed per query: row stride and even key offsets do
            // not change it).  Bias loads are unconditional: rows past the
            // tile use row M - 1, and keys past the block (masked below) read
            // other slot entries, at most 64 rows of R2e floats before slot 0,
            // inside shared memory.
            bbase = (min(qy, M - 1) + M - 1) * R2e + (qx + M - 1);
            pbase = slot + (((bbase - 1) & 1) ? copy1 - 1 : 0) + bbase - 1;
            m_run = -INFINITY;
          }
          const int nk = block_rows(u, j) * u.lx;
          const int nch = (nk + 15) >> 4;
          const uint32_t tP = tX + 128 + (b & 1) * 32;
          float factor = 1.f;
          bool rescale = false;
          constexpr bool scale_in_exp = MODE == 2 || (MODE == 0 && !has_table);
          const float ea = scale_in_exp ? alpha : 1.0f;
          if (ok && active) {
            const Ring w = ring_adv(wk.base, (uint32_t)j, nst);
            if (MODE == 1) {
              // 1/|k| of the block's keys was written by the K prep before kv_ready
              ok = __all_sync(0xffffffffu, wait_bar(&bars->kv_ready[w.slot], w.ph, ctl));
            }
            // x = log2-domain logits.  Mode 2 (and mode 0 without a table):
            // the scale is applied inside the exponent below (max over raw
            // scores, scale > 0).  Otherwise x = S * scale + bias in one
            // rounding; the bias slot holds T * log2(e), and mode 1's scale
            // is log2e / (tau |q| |k|).
            if (!scale_in_exp) {
              const float4* kc4 = reinterpret_cast<const float4*>(kcol + w.slot * kBlkKeys);
              const int4* kof4 = reinterpret_cast<const int4*>(kofs + u.cls * kBlkKeys);
              const int jo = j * u.Rk * R2e;  // block j starts Rk rectangle rows further
#pragma unroll
              for (int c4 = 0; c4 < kBlkKeys / 4; ++c4) {
                float2 s0 = make_float2(alpha, alpha), s1 = s0;
                if (MODE == 1) {
                  const float4 kc = kc4[c4];  // same address in every lane: broadcast
                  s0 = __fmul2_rn(make_float2(kc.x, kc.y), s0);
                  s1 = __fmul2_rn(make_float2(kc.z, kc.w), s1);
                }
                float2 b0 = make_float2(0.f, 0.f), b1 = b0;
                if (BIAS == kBiasPairs) {
                  const int4 ko = kof4[c4];  // broadcast; keys 4 c4 .. 4 c4 + 3 share a row pairwise
                  const float2 v0 = *reinterpret_cast<const float2*>(pbase - jo - ko.x);  // (bias key+1, key)
                  const float2 v1 = *reinterpret_cast<const float2*>(pbase - jo - ko.z);
                  b0 = make_float2(v0.y, v0.x);
                  b1 = make_float2(v1.y, v1.x);
                } else if (BIAS == kBiasKeys) {
                  // odd rectangle widths: one load per key
                  const int4 ko = kof4[c4];
                  const float* hb = slot + bbase - jo;
                  b0 = make_float2(hb[-ko.x], hb[-ko.y]);
                  b1 = make_float2(hb[-ko.z], hb[-ko.w]);
                }
                const float2 x0 = make_float2(__uint_as_float(xc[4 * c4]), __uint_as_float(xc[4 * c4 + 1]));
                const float2 x1 = make_float2(__uint_as_float(xc[4 * c4 + 2]), __uint_as_float(xc[4 * c4 + 3]));
                const float2 y0 = has_table ? __ffma2_rn(x0, s0, b0) : __fmul2_rn(x0, s0);
                const float2 y1 = has_table ? __ffma2_rn(x1, s1, b1) : __fmul2_rn(x1, s1);
                xc[4 * c4] = __float_as_uint(y0.x);
                xc[4 * c4 + 1] = __float_as_uint(y0.y);
                xc[4 * c4 + 2] = __float_as_uint(y1.x);
                xc[4 * c4 + 3] = __float_as_uint(y1.y);
              }
            }
            if (nk < kBlkKeys) {  // partial block (uniform across the warpgroup): mask the tail keys
#pragma unroll
              for (int c = 0; c < kBlkKeys; ++c)
                if (c >= nk) xc[c] = __float_as_uint(-INFINITY);
            }
            // block maximum: four independent 3-input max chains
            float mq[4] = {__uint_as_float(xc[0]), __uint_as_float(xc[1]), __uint_as_float(xc[2]),
                           __uint_as_float(xc[3])};
#pragma unroll
            for (int c = 4; c < kBlkKeys; c += 4) {
              const int chn = 2 * ((c >> 2) & 1);
              mq[chn] = ptx::max3(mq[chn], __uint_as_float(xc[c]), __uint_as_float(xc[c + 2]));
              mq[chn + 1] = ptx::max3(mq[chn + 1], __uint_as_float(xc[c + 1]), __uint_as_float(xc[c + 3]));
            }
            float mb = fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3]));
            if (scale_in_exp) mb *= ea;
            // running maximum, kept unless this block exceeds it by more than 8
            if (j == 0) {
              m_run = mb;
            } else if (mb > m_run + 8.0f) {
              factor = ptx::ex2_approx(m_run - mb);
              m_run = mb;
              rescale = true;
            }
          }
          // P[b % 2] is free once PV(b - 2) has read it
          if (ok && b >= 2) ok = wait_pv(b - 2);
          if (ok && active) {
            // probabilities, fp16, 16 keys (8 columns) at a time: exponent
            // argument x * ea - m
            const float eb = -m_run;
            constexpr int kPoly = ExpSplit<MODE>::kPoly;
#pragma unroll
            for (int ch = 0; ch < kBlkKeys / 16; ++ch) {
              if (ch == 0 || ch < nch) {  // chunks past the block: PV never reads them
                uint32_t pr[8];
#pragma unroll
                for (int e2 = 0; e2 < 8; ++e2) {
                  const int c = ch * 16 + 2 * e2;
                  const float2 e = __ffma2_rn(make_float2(__uint_as_float(xc[c]), __uint_as_float(xc[c + 1])),
                                              make_float2(ea, ea), make_float2(eb, eb));
                  if (c < kPoly) {
                    const float2 pe = exp2_poly2(e);
                    pr[e2] = ptx::pack_f16x2(pe.x, pe.y);
                  } else {
                    pr[e2] = ptx::pack_f16x2(ptx::ex2_approx(e.x), ptx::ex2_approx(e.y));
                  }
                }
                ptx::tmem_st8(tP + ch * 8, pr);
              }
            }
          }
          p_pending = true;
          // O (32 columns) and its row sum (column 32): rescaled to the new
          // maximum, or, in a tile's first block, the previous tile's result
          // read for the deferred store.  Both need PV(b - 1) complete, and
          // both come before PV(b) (issued once p_full(b) is arrived, at the
          // top of the next block).
          const bool epi = j == 0 && pend;
          const bool resc = j > 0 && __any_sync(0xffffffffu, rescale);
          if (ok && (epi || resc)) {
            ok = wait_pv(b - 1);
            if (ok) {
              uint32_t po[32];
              ptx::tmem_ld32(tO, po);
              uint32_t pl = ptx::tmem_ld1(tO + 32);
              ptx::tmem_wait_ld();
              reg_fence32(po);
              asm volatile("" : "+r"(pl));
              if (resc) {
#pragma unroll
                for (int e = 0; e < 32; ++e) po[e] = __float_as_uint(__uint_as_float(po[e]) * factor);
                ptx::tmem_st32(tO, po);
                ptx::tmem_st1(tO + 32, __float_as_uint(__uint_as_float(pl) * factor));
              } else {
                store_rows(po, pl, pend_off, pend_ok);
                pend = false;
              }
            }
          }
          if (ok && has_next) {
            // S(b + 1) is in registers: S[(b + 1) % 2] may take S(b + 3)
            ptx::tmem_wait_ld();
            reg_fence32(xn);
            reg_fence32(xn + 32);
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&bars->s_free[g][(b + 1) & 1]);
          }
          if (j == u.nb - 1) {
            // this tile's O is read in the next tile's first block (or after the loop)
            pend = active;
            pend_ok = row_ok;
            pend_off = (((size_t)u.b * p.H + (u.y0 + qy)) * p.W + (u.x0 + qx)) * (size_t)(p.heads * 32) +
                       (size_t)u.h * 32;
          }
          ++b;
          walk_next(wk, p, t_begin, t_end, g, nst);
        }
      }
    }
    if (ok && p_pending) arrive_p();
    if (ok && pend && b > 0) {
      ok = wait_pv(b - 1);
      if (ok) {
        uint32_t po[32];
        ptx::tmem_ld32(tO, po);
        uint32_t pl = ptx::tmem_ld1(tO + 32);
        ptx::tmem_wait_ld();
        reg_fence32(po);
        asm volatile("" : "+r"(pl));
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
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The driver entry point, looked up once; a function-local static with an
// initialiser is thread-safe in C++11 and later.
EncodeTiledFn encode_fn() {
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

// Box of lx tokens x rows rectangle rows of one head (32 channels, 64 bytes).
// A head's 64-byte chunks of neighbouring tokens are heads * 64 bytes apart,
// so no L2 promotion: a wider fetch would bring in other heads' channels that
// are used much later.
bool encode_map(CUtensorMap* m, const void* base, const AttnArgs& a, int lx, int rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[5] = {32, (cuuint64_t)a.heads, (cuuint64_t)a.W, (cuuint64_t)a.H, (cuuint64_t)a.B};
  const cuuint64_t row = 64;  // bytes of one head
  const cuuint64_t strides[4] = {row, row * a.heads, row * a.heads * a.W, row * a.heads * a.W * a.H};
  const cuuint32_t box[5] = {32, 1, (cuuint32_t)lx, (cuuint32_t)rows, 1};
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int MODE, bool F32, int BIAS>
swin_status launch_mode(const TcParams& p, int smem, cudaStream_t stream) {
  auto k = attn_tc_kernel<MODE, F32, BIAS>;
  cudaError_t ea = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (ea != cudaSuccess) return fail(SWIN_ERR_CUDA, "attn_tc smem attribute: %s", cudaGetErrorString(ea));
  k<<<p.n_ctas, kThreads, smem, stream>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(SWIN_ERR_CUDA, "attn_tc launch: %s", cudaGetErrorString(e));
  return SWIN_OK;
}

}  // namespace

static long long g_tc_wait_limit = 4000000000ll;  // ~2 s at 2 GHz
static int g_tc_debug_flags = 0;

void tc_set_debug(int flags, long long wait_limit) {
  g_tc_debug_flags = flags;
  g_tc_wait_limit = wait_limit > 0 ? wait_limit : 4000000000ll;
}

// Everything about a launch that does not need the device: geometry, tile
// list, ring and buffer counts, bias-slot layout, per-CTA ranges, shared
// memory.  Tensor maps and pointers are filled in by launch_attn_tc.
swin_status tc_plan(int B, int H, int W, int heads, int M, int shift, int mode, bool table, int sms, TcParams& p,
                    int& smem, long long& n_tiles) {
  if (M > 64) return fail(SWIN_ERR_UNSUPPORTED, "tensor-core path needs M <= 64");
  if (table && M > 32) return fail(SWIN_ERR_UNSUPPORTED, "tensor-core path keeps a bias table only for M <= 32");
  memset(&p, 0, sizeof(p));
  p.B = B; p.H = H; p.W = W; p.heads = heads; p.M = M; p.s = shift;
  p.nsy = swin_nseg(H, M, shift);
  p.nsx = swin_nseg(W, M, shift);
  // column classes: first, middle (if any), last segment
  const int lxs[3] = {swin_seg_len(0, W, M, shift),
                      p.nsx > 2 ? swin_seg_len(1, W, M, shift) : swin_seg_len(0, W, M, shift),
                      swin_seg_len(p.nsx - 1, W, M, shift)};
  for (int c = 0; c < 3; ++c) {
    p.lx[c] = lxs[c];
    p.R[c] = 128 / lxs[c];         // query tile: whole rectangle rows, at most 128 queries
    p.Rh[c] = 64 / lxs[c];         // a tile of at most 64 rows: the half-height box
    p.Rk[c] = kBlkKeys / lxs[c];   // K/V block: whole rectangle rows, at most 64 keys
  }
  // row classes: first, middle (if any), last row of rectangles
  const int lys[3] = {swin_seg_len(0, H, M, shift),
                      p.nsy > 2 ? swin_seg_len(1, H, M, shift) : swin_seg_len(0, H, M, shift),
                      swin_seg_len(p.nsy - 1, H, M, shift)};
  for (int rc = 0; rc < 3; ++rc) {
    p.row_ly[rc] = lys[rc];
    for (int c = 0; c < 3; ++c) {
      p.rect_tiles[rc][c] = (lys[rc] + p.R[c] - 1) / p.R[c];
      p.rect_nb[rc][c] = (lys[rc] + p.Rk[c] - 1) / p.Rk[c];
    }
    p.row_tiles[rc] = p.nsx == 1 ? p.rect_tiles[rc][0]
                                 : p.rect_tiles[rc][0] + (p.nsx - 2) * p.rect_tiles[rc][1] + p.rect_tiles[rc][2];
  }
  auto row_cls = [&](int sy) { return sy == 0 ? 0 : (sy == p.nsy - 1 ? 2 : 1); };
  auto col_cls = [&](int sx) { return sx == 0 ? 0 : (sx == p.nsx - 1 ? 2 : 1); };
  // one representative segment of each class present: first, a middle one, last
  const int rep_y[3] = {0, p.nsy > 2 ? 1 : 0, p.nsy - 1}, rep_x[3] = {0, p.nsx > 2 ? 1 : 0, p.nsx - 1};
  int nb_max = 0;
  for (int i = 0; i < 3; ++i)
    for (int j = 0; j < 3; ++j) nb_max = std::max(nb_max, p.rect_nb[row_cls(rep_y[i])][col_cls(rep_x[j])]);
  const long long t_img = (long long)p.row_tiles[0] + (p.nsy > 2 ? (long long)(p.nsy - 2) * p.row_tiles[1] : 0) +
                          (p.nsy > 1 ? p.row_tiles[2] : 0);
  n_tiles = t_img * B * heads;
  if (n_tiles >= (1ll << 31)) return fail(SWIN_ERR_UNSUPPORTED, "too many query tiles (%lld)", n_tiles);
  p.div_img = make_fastdiv((uint32_t)t_img);
  p.div_B = make_fastdiv((uint32_t)B);
  p.div_rowmid = make_fastdiv((uint32_t)p.row_tiles[1]);
  for (int rc = 0; rc < 3; ++rc) p.div_colmid[rc] = make_fastdiv((uint32_t)p.rect_tiles[rc][1]);

  // Bias slot: rows dy with an even stride R2e in [2M, 2M + 14], stored twice
  // (the second copy one float ahead, copy1 floats further), so that the two
  // keys of an even-width row pair are one aligned 8-byte load.  R2e is the
  // candidate with the fewest shared-memory wavefronts for the paired loads
  // of this launch's rectangle widths: a warp's 32 queries load 8 bytes each
  // in two 16-lane phases; query (qy, qx) of a width-lx rectangle reads
  // floats qy R2e + qx - 1 (+ copy1 - 1 when that is odd) and on.
  p.R2e = 2 * M;
  if (table) {
    long best = -1;
    for (int r2 = 2 * M; r2 <= 2 * M + 14; r2 += 2) {
      const int cp1 = (2 * M - 1) * r2 + 16;
      long cost = 0;
      for (int c = 0; c < 3; ++c) {
        const int lx = p.lx[c];
        if (lx & 1) continue;
        for (int w0 = 0; w0 < 128; w0 += 32)
          for (int ph = 0; ph < 2; ++ph) {
            int hits[16] = {0}, mx = 0;
            for (int l = 0; l < 16; ++l) {
              const int t = w0 + 16 * ph + l, qy = t / lx, qx = t % lx;
              int idx = qy * r2 + qx + M - 2;  // parity as in the kernel's bbase - 1
              if (idx & 1) idx += cp1 - 1;
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
    p.copy1 = (2 * M - 1) * p.R2e + 16;
    p.slot_floats = p.copy1 + (2 * M - 1) * p.R2e;
  }

  // Ring stages from the shared-memory budget; Q buffers: 4 per warpgroup
  // for short tiles (few blocks), where loads must run further ahead.
  p.nqb = nb_max <= 4 ? 4 : 2;
  const int slot_f = table ? p.slot_floats : 0;
  int nst = kMaxStages;
  while (nst > 3 && tc_layout(p.nqb, nst, mode == 2, slot_f).total + kSmemSlack > (uint32_t)kSmemMax) --nst;
  if (tc_layout(p.nqb, nst, mode == 2, slot_f).total + kSmemSlack > (uint32_t)kSmemMax)
    return fail(SWIN_ERR_UNSUPPORTED, "tensor-core path: shared memory does not fit (M=%d)", M);
  p.nst = nst;
  // a whole window resident per pass when the ring holds its blocks plus three
  p.max_pass_tiles = nst >= nb_max + 3 ? (1 << 30) : 2;
  smem = (int)tc_layout(p.nqb, nst, mode == 2, slot_f).total + kSmemSlack;

  // Per-CTA tile ranges of equal work.  Work of a tile ~ its K/V blocks x the
  // 16-key chunks the softmax evaluates x the warps with rows, plus a fixed
  // cost per block and per tile; the list repeats per (head, image).
  std::vector<double> pre(1, 0.0);
  pre.reserve((size_t)t_img + 1);
  for (int sy = 0; sy < p.nsy; ++sy) {
    const int rc = row_cls(sy), ly = p.row_ly[rc];
    for (int sx = 0; sx < p.nsx; ++sx) {
      const int c = col_cls(sx), lx = p.lx[c];
      for (int k = 0; k < p.rect_tiles[rc][c]; ++k) {
        const int rows = std::min(p.R[c], ly - k * p.R[c]), nq = rows * lx;
        double w = 60.0;
        for (int j = 0; j < p.rect_nb[rc][c]; ++j) {
          const int nk = std::min(p.Rk[c], ly - j * p.Rk[c]) * lx;
          w += 16.0 * ((nk + 15) / 16) * ((nq + 31) / 32) + 40.0;
        }
        pre.push_back(pre.back() + w);
      }
    }
  }
  const int G = (int)std::min<long long>(std::min(sms, kMaxCtas), n_tiles);
  const long long n_ih = (long long)B * heads;
  const double w_img = pre.back(), total = w_img * (double)n_ih;
  p.n_ctas = G;
  p.cta_start[0] = 0;
  for (int c = 1; c < G; ++c) {
    const double target = total * c / G;
    long long ih = (long long)(target / w_img);
    double rem = target - (double)ih * w_img;
    if (ih >= n_ih) {
      ih = n_ih - 1;
      rem = w_img;
    }
    const long long idx = std::lower_bound(pre.begin(), pre.end(), rem) - pre.begin();
    long long start = ih * t_img + std::min<long long>(idx, t_img);
    start = std::max<long long>(start, (long long)p.cta_start[c - 1] + 1);  // every CTA gets a tile
    start = std::min<long long>(start, n_tiles - (G - c));
    p.cta_start[c] = (int)start;
  }
  p.cta_start[G] = (int)n_tiles;
  return SWIN_OK;
}

swin_status launch_attn_tc(const AttnArgs& a, bool f32_out, cudaStream_t stream) {
  if (a.d != 32) return fail(SWIN_ERR_UNSUPPORTED, "tensor-core path needs d == 32, got %d", a.d);
  const bool table = a.mode != 2 && a.table != nullptr;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  TcParams p;
  int smem = 0;
  long long n_tiles = 0;
  swin_status st = tc_plan(a.B, a.H, a.W, a.heads, a.M, a.shift, a.mode, table, sms, p, smem, n_tiles);
  if (st != SWIN_OK) return st;
  for (int c = 0; c < 3; ++c)
    if (!encode_map(&p.tmq[c], a.q, a, p.lx[c], p.R[c]) || !encode_map(&p.tmqh[c], a.q, a, p.lx[c], p.Rh[c]) ||
        !encode_map(&p.tmk[c], a.k, a, p.lx[c], p.Rk[c]) || !encode_map(&p.tmv[c], a.v, a, p.lx[c], p.Rk[c]))
      return fail(SWIN_ERR_CUDA, "cuTensorMapEncodeTiled failed (lx=%d)", p.lx[c]);
  p.out = a.out;
  p.tau = a.tau;
  p.table = a.table;
  p.rope = a.rope;
  p.status = a.status;
  p.wait_limit = g_tc_wait_limit;
  p.debug_flags = g_tc_debug_flags;
  switch (a.mode) {
    case 0:
    case 1: {
      const bool all_even = !(p.lx[0] & 1) && !(p.lx[1] & 1) && !(p.lx[2] & 1);
      const int kind = !table ? kBiasNone : (all_even ? kBiasPairs : kBiasKeys);
#define SWIN_TC_LAUNCH(MD)                                                                               \
  switch (kind) {                                                                                       \
    case kBiasNone:                                                                                     \
      return f32_out ? launch_mode<MD, true, kBiasNone>(p, smem, stream)                                \
                     : launch_mode<MD, false, kBiasNone>(p, smem, stream);                              \
    case kBiasPairs:                                                                                    \
      return f32_out ? launch_mode<MD, true, kBiasPairs>(p, smem, stream)                               \
                     : launch_mode<MD, false, kBiasPairs>(p, smem, stream);                             \
    default:                                                                                            \
      return f32_out ? launch_mode<MD, true, kBiasKeys>(p, smem, stream)                                \
                     : launch_mode<MD, false, kBiasKeys>(p, smem, stream);                              \
  }
      if (a.mode == 0) SWIN_TC_LAUNCH(0)
      SWIN_TC_LAUNCH(1)
#undef SWIN_TC_LAUNCH
    }
    default:
      return f32_out ? launch_mode<2, true, kBiasNone>(p, smem, stream)
                     : launch_mode<2, false, kBiasNone>(p, smem, stream);
  }
}

}  // namespace swin

// Test hook: the launch plan of the tensor-core kernel, computed on the host
// only (no device needed).  plan[0..9] = nst, nqb, max_pass_tiles, n_ctas,
// smem bytes, tiles, R2e, copy1, slot_floats, 0; plan[10..10+n_ctas] =
// cta_start.  tiles (may be NULL) receives, per tile t < max_tiles, the
// decoded unit: h, b, cls, y0, ly, x0, lx, R, Rh, Rk, ntile, nb, k.
extern "C" swin_status swin_debug_tc_plan(int B, int H, int W, int heads, int M, int shift, int mode, int have_table,
                                          int sms, int32_t* plan, int32_t* tiles, long long max_tiles) {
  using namespace swin;
  if (!plan || B < 1 || H < 1 || W < 1 || heads < 1 || M < 1 || shift < 0 || shift >= M || sms < 1 || mode < 0 ||
      mode > 2)
    return fail(SWIN_ERR_INVALID_ARG, "swin_debug_tc_plan: bad arguments");
  TcParams p;
  int smem = 0;
  long long n_tiles = 0;
  swin_status st = tc_plan(B, H, W, heads, M, shift, mode, mode != 2 && have_table, sms, p, smem, n_tiles);
  if (st != SWIN_OK) return st;
  const int32_t head[10] = {p.nst, p.nqb, p.max_pass_tiles, p.n_ctas, smem, (int32_t)n_tiles, p.R2e, p.copy1,
                            p.slot_floats, 0};
  memcpy(plan, head, sizeof(head));
  for (int c = 0; c <= p.n_ctas; ++c) plan[10 + c] = p.cta_start[c];
  if (tiles)
    for (long long t = 0; t < n_tiles && t < max_tiles; ++t) {
      int k = 0;
      const Unit u = decode_tile(p, (uint32_t)t, k);
      const int32_t row[13] = {u.h, u.b, u.cls, u.y0, u.ly, u.x0, u.lx, u.R, u.Rh, u.Rk, u.ntile, u.nb, k};
      memcpy(tiles + 13 * t, row, sizeof(row));
    }
  return SWIN_OK;
}

