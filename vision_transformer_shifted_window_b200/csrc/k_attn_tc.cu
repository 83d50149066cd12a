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
// Work unit: a pair of 128-row query tiles of one rectangle (tile = R whole
// rectangle rows, R = floor(128 / lx)), one per softmax warpgroup; both
// warpgroups stream the same K/V blocks of R rectangle rows.
//
// Warp roles (384 threads, one persistent CTA per SM):
//   warp 0      TMA producer: Q tiles and K/V blocks, 5-D tensor maps over
//               [B][H][W][heads][d] with 64-byte swizzle, no multicast
//   warp 1      tcgen05.mma issuer (one thread) and TMEM owner
//   warps 2-3   operand prep in shared memory: K unit-normalisation (mode 1),
//               RoPE rotation of Q and K (mode 2), per-row 1/(tau |q|) (mode 1)
//   warps 4-7   softmax of warpgroup 0 (one TMEM lane = one query row)
//   warps 8-11  softmax of warpgroup 1
// TMEM per softmax warpgroup g (128 lanes): S [g*256, +128) fp32 scores,
// P [g*256+128, +64) bf16x2 probabilities, O [g*256+192, +48) fp32: 32 output
// columns and, in column 32, the row sum of P.
// Per K/V block: S = Q K^T (2 MMAs, K-dim 32); softmax on S with the exact
// running maximum (O is rescaled whenever it grows, so the largest weight of
// a row is exactly 1 in bf16); P written to TMEM; O += P [V | 1] (8 MMAs,
// N = 48, A from TMEM): a constant block with a one in the first column
// appended to V makes the tensor core add up the same bf16-rounded P that
// multiplies V, so the normalisation is consistent and costs no ALU work.
// S of the next block is issued as soon as the softmax has copied the
// current S to registers.
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

#include <cstring>

#include "sm100_ptx.cuh"
#include "swin_common.cuh"

namespace swin {

struct TcParams {
  CUtensorMap tmap[3][3];  // [tensor q/k/v][x-class first/middle/last]
  int lx[3], R[3];         // per x-class: segment width, rows per tile
  void* out;
  int B, H, W, heads, M, s, nsy, nsx, pmax;
  long long n_items;
  const float* tau;
  const float* table;
  const float* rope;
  int* status;
  long long wait_limit;  // clock64 cycles before a wait gives up
  int debug_flags;       // bit 0: force a time-out (test of the failure path)
};

namespace {

constexpr int kThreads = 384;
constexpr int kStages = 6;                  // K/V ring
constexpr int kTileBytes = 128 * 64;        // 128 rows x 32 bf16
constexpr int kQOff = 0;                    // [2 wg][2 buf] Q tiles
constexpr int kKVOff = kQOff + 4 * kTileBytes;
constexpr int kOnesOff = kKVOff + kStages * 2 * kTileBytes;    // 16 rows of [1, 0...] (1 KB)
constexpr int kScaleOff = kOnesOff + 1024;                      // [2][2][128] f32
constexpr int kRopeOff = kScaleOff + 2 * 2 * 128 * 4;         // cos,sin [2][64][8] f32
constexpr int kKofsOff = kRopeOff + 2 * 2 * 64 * 8 * 4;       // [3][128] int
constexpr int kKscOff = kKofsOff + 3 * 128 * 4;                 // [kStages] f32 + reduction [2][2]
constexpr int kKcolOff = kKscOff + 256;                          // [kStages][128] f32, 1/|k| (mode 1)
constexpr int kBarOff = kKcolOff + kStages * 128 * 4;
constexpr int kNumBars = 12 + 3 * kStages + 8 + 2;
constexpr int kSmemBytes = kBarOff + kNumBars * 8 + 64;
constexpr int kSmemAlloc = kSmemBytes + 1024;  // slack for 1024-byte alignment

constexpr float kLog2eF = 1.4426950408889634f;

struct Bars {
  uint64_t q_full[2][2], q_ready[2][2], q_empty[2][2];
  uint64_t kv_full[kStages], kv_ready[kStages], kv_empty[kStages];
  uint64_t s_full[2], s_free[2], p_full[2], o_done[2];
  uint64_t never, drain;
};
static_assert(sizeof(Bars) == kNumBars * 8, "barrier block size");

struct Task {
  bool any;       // item has work for warpgroup 0
  bool valid[2];  // per warpgroup
  int b, h, cls, lx, R, y0, x0, ly, n, nb;
  int tile[2], nq[2];
};

__device__ __forceinline__ Task decode(const TcParams& p, long long item) {
  Task t;
  long long i = item;
  const int pr = (int)(i % p.pmax);
  i /= p.pmax;
  const int sx = (int)(i % p.nsx);
  i /= p.nsx;
  const int sy = (int)(i % p.nsy);
  i /= p.nsy;
  t.h = (int)(i % p.heads);
  t.b = (int)(i / p.heads);
  t.cls = sx == 0 ? 0 : (sx == p.nsx - 1 ? 2 : 1);
  t.lx = p.lx[t.cls];
  t.R = p.R[t.cls];
  t.y0 = swin_seg_start(sy, p.M, p.s);
  t.ly = swin_seg_len(sy, p.H, p.M, p.s);
  t.x0 = swin_seg_start(sx, p.M, p.s);
  t.n = t.ly * t.lx;
  t.nb = (t.ly + t.R - 1) / t.R;
  for (int g = 0; g < 2; ++g) {
    t.tile[g] = 2 * pr + g;
    t.valid[g] = t.tile[g] < t.nb;
    int rows = t.ly - t.tile[g] * t.R;
    t.nq[g] = t.valid[g] ? (rows < t.R ? rows : t.R) * t.lx : 0;
  }
  t.any = t.valid[0];
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
    if (ptx::mbar_try_wait(bar, parity)) return true;
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
// rotated / normalised operands is the largest error term of the path.  Unit
// vectors cannot overflow fp16; rotated rows are first scaled by an exact power
// of two (per query row, per K block) that is divided out in the softmax.

// Load one 32-element bf16 row (64-byte swizzled tile row) as fp32.
__device__ __forceinline__ void load_row_bf16(const uint8_t* tile, int row, float (&v)[32]) {
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const uint4 w = *reinterpret_cast<const uint4*>(tile + swz64(row, c));
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      v[8 * c + 2 * e] = bf_lo(u[e]);
      v[8 * c + 2 * e + 1] = bf_hi(u[e]);
    }
  }
}

// Store v * sc as fp16 into the same row.
__device__ __forceinline__ void store_row_f16(uint8_t* tile, int row, const float (&v)[32], float sc) {
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint32_t u[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) u[e] = ptx::pack_f16x2(v[8 * c + 2 * e] * sc, v[8 * c + 2 * e + 1] * sc);
    *reinterpret_cast<uint4*>(tile + swz64(row, c)) = make_uint4(u[0], u[1], u[2], u[3]);
  }
}

__device__ __forceinline__ float inv_norm(const float (&v)[32]) {
  float ss = 0.f;
#pragma unroll
  for (int e = 0; e < 32; ++e) ss = fmaf(v[e], v[e], ss);
  return 1.0f / fmaxf(sqrtf(ss), kNormEps);
}

// Rotate channels [0,16) by py and [16,32) by px (pairs (2t, 2t+1), t < 8).
__device__ __forceinline__ void rope_rotate(float (&v)[32], int py, int px, const float* rc, const float* rs) {
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int pos = half ? px : py;
    const float* cs = rc + (half * 64 + pos) * 8;
    const float* sn = rs + (half * 64 + pos) * 8;
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      const float a = v[16 * half + 2 * t], b = v[16 * half + 2 * t + 1];
      const float co = cs[t], si = sn[t];
      v[16 * half + 2 * t] = a * co - b * si;
      v[16 * half + 2 * t + 1] = a * si + b * co;
    }
  }
}

__device__ __forceinline__ float absmax(const float (&v)[32]) {
  float m = 0.f;
#pragma unroll
  for (int e = 0; e < 32; ++e) m = fmaxf(m, fabsf(v[e]));
  return m;
}

// Power of two that brings a row maximum m below 2^15 (fp16 max is 65504).
__device__ __forceinline__ float pow2_scale(float m) {
  if (!(m > 0.f)) return 1.f;
  int e;
  frexpf(m, &e);  // m < 2^e
  return ldexpf(1.0f, 15 - e);
}

// ------------------------------------------------------------------ kernel
template <int MODE, bool OUT_F32>
__global__ void __launch_bounds__(kThreads, 1) attn_tc_kernel(const __grid_constant__ TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* qbuf = smem + kQOff;
  uint8_t* kvbuf = smem + kKVOff;
  float* qscale = reinterpret_cast<float*>(smem + kScaleOff);
  float* rcos = reinterpret_cast<float*>(smem + kRopeOff);
  float* rsin = rcos + 2 * 64 * 8;
  int* kofs = reinterpret_cast<int*>(smem + kKofsOff);
  float* kscale = reinterpret_cast<float*>(smem + kKscOff);          // per K/V stage
  float* kred = kscale + 32;                                         // [2 parity][2 warps]
  float* kcol = reinterpret_cast<float*>(smem + kKcolOff);
  uint8_t* ones = smem + kOnesOff;
  Bars* bars = reinterpret_cast<Bars*>(smem + kBarOff);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + kBarOff + kNumBars * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int M = p.M, s = p.s;

  // ---- set-up: barriers, RoPE tables, bias column offsets, TMEM
  if (threadIdx.x == 0) {
    for (int g = 0; g < 2; ++g)
      for (int b = 0; b < 2; ++b) {
        ptx::mbar_init(&bars->q_full[g][b], 1);
        ptx::mbar_init(&bars->q_ready[g][b], 64);
        ptx::mbar_init(&bars->q_empty[g][b], 1 + 4);
      }
    for (int i = 0; i < kStages; ++i) {
      ptx::mbar_init(&bars->kv_full[i], 1);
      ptx::mbar_init(&bars->kv_ready[i], 64);
      ptx::mbar_init(&bars->kv_empty[i], 1);
    }
    for (int g = 0; g < 2; ++g) {
      ptx::mbar_init(&bars->s_full[g], 1);
      ptx::mbar_init(&bars->s_free[g], 128);
      ptx::mbar_init(&bars->p_full[g], 128);
      ptx::mbar_init(&bars->o_done[g], 1);
    }
    ptx::mbar_init(&bars->never, 1);
    ptx::mbar_init(&bars->drain, 1);
    *abort_flag = 0;
    tmem_holder[2] = 0;  // abort flag of the drain waits (never set by a role)
    ptx::fence_mbar_init();
  }
  if (MODE == 2) {
    for (int i = threadIdx.x; i < 2 * M * 8; i += kThreads) {
      const int axis = i / (M * 8), pos = (i / 8) % M, t = i % 8;
      float sv, cv;
      sincosf((float)pos * p.rope[axis * 8 + t], &sv, &cv);
      rcos[(axis * 64 + pos) * 8 + t] = cv;
      rsin[(axis * 64 + pos) * 8 + t] = sv;
    }
  }
  if (MODE != 2) {
    for (int i = threadIdx.x; i < 3 * 128; i += kThreads) {
      const int c = i / 128, col = i % 128, lx = p.lx[c];
      kofs[i] = (col / lx) * (2 * M - 1) + (col % lx);
    }
  }
  // zero the K/V ring once so rows a tile never writes hold finite values;
  // the ones block: 16 rows of 64 bytes (64B swizzle), bf16 1.0 at element 0
  for (int i = threadIdx.x; i < (kStages * 2 * kTileBytes + 1024) / 16; i += kThreads)
    reinterpret_cast<uint4*>(kvbuf)[i] = make_uint4(0, 0, 0, 0);
  __syncthreads();
  if (threadIdx.x < 16) *reinterpret_cast<uint16_t*>(ones + swz64(threadIdx.x, 0)) = 0x3F80;
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
  // Register split: warps 0-3 (producer, MMA, prep) give registers to the two
  // softmax warpgroups: 384 x 168 = 128 x 72 + 256 x 216.

  const long long first = blockIdx.x, step = gridDim.x;

  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 72;\n" ::: "memory");
  if (warp == 0) {
    // ================================================================ producer
    if (lane == 0) {
      uint32_t qu[2] = {0, 0};
      uint32_t ku = 0;
      bool ok = true;
      for (long long it = first; it < p.n_items && ok; it += step) {
        const Task t = decode(p, it);
        if (!t.any) continue;
        const uint32_t box_bytes = (uint32_t)(64 * t.lx * t.R);
        for (int g = 0; g < 2 && ok; ++g) {
          if (!t.valid[g]) continue;
          const int qs = qu[g] & 1;
          if (qu[g] >= 2) ok = wait_bar(&bars->q_empty[g][qs], ((qu[g] >> 1) - 1) & 1, ctl);
          if (!ok) break;
          ptx::mbar_arrive_expect_tx(&bars->q_full[g][qs], box_bytes);
          ptx::tma_load_5d(qbuf + (g * 2 + qs) * kTileBytes, &p.tmap[0][t.cls], &bars->q_full[g][qs], 0, t.h,
                           t.x0, t.y0 + t.tile[g] * t.R, t.b);
          ++qu[g];
        }
        for (int j = 0; j < t.nb && ok; ++j) {
          const int st = ku % kStages;
          if (ku >= (uint32_t)kStages) ok = wait_bar(&bars->kv_empty[st], ((ku / kStages) - 1) & 1, ctl);
          if (!ok) break;
          uint8_t* kb = kvbuf + st * 2 * kTileBytes;
          ptx::mbar_arrive_expect_tx(&bars->kv_full[st], 2 * box_bytes);
          ptx::tma_load_5d(kb, &p.tmap[1][t.cls], &bars->kv_full[st], 0, t.h, t.x0, t.y0 + j * t.R, t.b);
          ptx::tma_load_5d(kb + kTileBytes, &p.tmap[2][t.cls], &bars->kv_full[st], 0, t.h, t.x0,
                           t.y0 + j * t.R, t.b);
          ++ku;
        }
      }
      {
        // drain copies that may still be landing in shared memory (after an
        // abort; in a normal exit every phase waited here has completed)
        Ctl drain{reinterpret_cast<volatile int*>(tmem_holder + 2), &p};
        for (uint32_t u = (ku > (uint32_t)kStages ? ku - kStages : 0); u < ku; ++u)
          wait_bar(&bars->kv_full[u % kStages], (u / kStages) & 1, drain);
        for (int g = 0; g < 2; ++g)
          for (uint32_t u = (qu[g] > 2 ? qu[g] - 2 : 0); u < qu[g]; ++u)
            wait_bar(&bars->q_full[g][u & 1], (u >> 1) & 1, drain);
      }
    }
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      // mode 2 feeds fp16 operands (see prep), modes 0 and 1 the bf16 inputs
      constexpr uint32_t fmtS = MODE == 2 ? 0u : 1u;
      constexpr uint32_t idS = ptx::idesc_f16(fmtS, fmtS, 0, 0, 128, 128);
      constexpr uint32_t idPV = ptx::idesc_f16(1, 1, 0, 1, 48, 128);
      const uint32_t ones_addr = ptx::smem_addr(ones);
      uint32_t qu[2] = {0, 0}, s_iss[2] = {0, 0}, pv_cnt[2] = {0, 0};
      uint32_t ku = 0;  // K/V block uses consumed
      bool ok = true;
      if (p.debug_flags & 1) ok = wait_bar(&bars->never, 0, ctl);  // forced time-out

      auto issue_S = [&](int g, int qs, int st) -> bool {
        if (s_iss[g] > 0 && !wait_bar(&bars->s_free[g], (s_iss[g] - 1) & 1, ctl)) return false;
        ptx::tc_fence_after();
        const uint32_t qa = ptx::smem_addr(qbuf + (g * 2 + qs) * kTileBytes);
        const uint32_t ka = ptx::smem_addr(kvbuf + st * 2 * kTileBytes);
        const uint64_t ad = ptx::smem_desc(qa, 16, 512, ptx::kSwizzle64B);
        const uint64_t bd = ptx::smem_desc(ka, 16, 512, ptx::kSwizzle64B);
        const uint32_t dS = tmem_base + g * 256;
        ptx::mma_ss(dS, ad, bd, idS, 0);
        ptx::mma_ss(dS, ad + 2, bd + 2, idS, 1);  // second 16-wide K step: +32 bytes
        ptx::mma_commit(&bars->s_full[g]);
        ++s_iss[g];
        return true;
      };

      // Find the first item with work.
      long long it = first;
      Task cur;
      cur.any = false;
      for (; it < p.n_items; it += step) {
        cur = decode(p, it);
        if (cur.any) break;
      }
      int cur_qs[2] = {0, 0};
      uint32_t cur_k0 = 0;
      if (ok && it < p.n_items) {
        // prologue: S of block 0 of the first item
        for (int g = 0; g < 2 && ok; ++g)
          if (cur.valid[g]) {
            cur_qs[g] = qu[g] & 1;
            ok = wait_bar(&bars->q_ready[g][cur_qs[g]], (qu[g] >> 1) & 1, ctl);
            ++qu[g];
          }
        cur_k0 = ku;
        if (ok) ok = wait_bar(&bars->kv_ready[ku % kStages], (ku / kStages) & 1, ctl);
        for (int g = 0; g < 2 && ok; ++g)
          if (cur.valid[g]) {
            ok = issue_S(g, cur_qs[g], ku % kStages);
            if (ok && cur.nb == 1) ptx::mma_commit(&bars->q_empty[g][cur_qs[g]]);
          }
        ++ku;
      }
      while (ok && it < p.n_items) {
        long long nit = it + step;
        Task nxt;
        nxt.any = false;
        int nxt_qs[2] = {0, 0};
        for (int j = 0; j < cur.nb && ok; ++j) {
          const int st = (cur_k0 + j) % kStages;
          if (j + 1 < cur.nb) {
            ok = wait_bar(&bars->kv_ready[ku % kStages], (ku / kStages) & 1, ctl);
            for (int g = 0; g < 2 && ok; ++g)
              if (cur.valid[g]) {
                ok = issue_S(g, cur_qs[g], ku % kStages);
                if (ok && j + 1 == cur.nb - 1) ptx::mma_commit(&bars->q_empty[g][cur_qs[g]]);
              }
            ++ku;
          } else {
            // look ahead into the next item with work
            for (; nit < p.n_items; nit += step) {
              nxt = decode(p, nit);
              if (nxt.any) break;
            }
            if (nit < p.n_items) {
              for (int g = 0; g < 2 && ok; ++g)
                if (nxt.valid[g]) {
                  nxt_qs[g] = qu[g] & 1;
                  ok = wait_bar(&bars->q_ready[g][nxt_qs[g]], (qu[g] >> 1) & 1, ctl);
                  ++qu[g];
                }
              if (ok) ok = wait_bar(&bars->kv_ready[ku % kStages], (ku / kStages) & 1, ctl);
              for (int g = 0; g < 2 && ok; ++g)
                if (nxt.valid[g]) {
                  ok = issue_S(g, nxt_qs[g], ku % kStages);
                  if (ok && nxt.nb == 1) ptx::mma_commit(&bars->q_empty[g][nxt_qs[g]]);
                }
              ++ku;
            }
          }
          // O += P V for block j
          const uint32_t va = ptx::smem_addr(kvbuf + st * 2 * kTileBytes + kTileBytes);
          for (int g = 0; g < 2 && ok; ++g) {
            if (!cur.valid[g]) continue;
            ok = wait_bar(&bars->p_full[g], pv_cnt[g] & 1, ctl);
            ++pv_cnt[g];
            if (!ok) break;
            ptx::tc_fence_after();
            const uint32_t dO = tmem_base + g * 256 + 192, aP = tmem_base + g * 256 + 128;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              // N columns 0-31: V rows; 32-47: the ones block (LBO = its distance)
              const uint32_t vk = va + kk * 1024;
              const uint64_t bd = ptx::smem_desc(vk, ones_addr - vk, 512, ptx::kSwizzle64B);
              ptx::mma_ts(dO, aP + kk * 8, bd, idPV, (j > 0 || kk > 0) ? 1u : 0u);
            }
            ptx::mma_commit(&bars->o_done[g]);
          }
          if (ok) ptx::mma_commit(&bars->kv_empty[st]);
        }
        cur = nxt;
        cur_qs[0] = nxt_qs[0];
        cur_qs[1] = nxt_qs[1];
        cur_k0 = ku - 1;
        it = nit;
      }
      // drain: every MMA this thread issued has completed before TMEM is freed
      ptx::mma_commit(&bars->drain);
      Ctl drain{reinterpret_cast<volatile int*>(tmem_holder + 2), &p};
      wait_bar(&bars->drain, 0, drain);
    }
  } else if (warp < 4) {
    // ================================================================ prep
    const int pt = threadIdx.x - 64;  // 0..63
    uint32_t qu[2] = {0, 0}, ku = 0;
    bool ok = true;
    for (long long it = first; it < p.n_items && ok; it += step) {
      const Task t = decode(p, it);
      if (!t.any) continue;
      const int rows = t.lx * t.R;
      for (int g = 0; g < 2 && ok; ++g) {
        if (!t.valid[g]) continue;
        const int qs = qu[g] & 1;
        ok = wait_bar(&bars->q_full[g][qs], (qu[g] >> 1) & 1, ctl);
        ++qu[g];
        if (!ok) break;
        uint8_t* tile = qbuf + (g * 2 + qs) * kTileBytes;
        const float te = MODE == 1 ? fmaxf(__ldg(p.tau + t.h), kTauMin) : 1.f;
        if (MODE != 0) {
          for (int r = pt; r < rows; r += 64) {
            float v[32];
            load_row_bf16(tile, r, v);
            if (MODE == 1) {
              qscale[(g * 2 + qs) * 128 + r] = kLog2eF * inv_norm(v) / te;
            } else {
              const int qy = t.tile[g] * t.R + r / t.lx, qx = r % t.lx;
              rope_rotate(v, swin_local_coord(t.y0 + qy, M, s), swin_local_coord(t.x0 + qx, M, s), rcos, rsin);
              const float sc = pow2_scale(absmax(v));
              store_row_f16(tile, r, v, sc);
              qscale[(g * 2 + qs) * 128 + r] = kLog2eF * rsqrtf(32.0f) / sc;
            }
          }
          ptx::fence_proxy_async_smem();
        }
        ptx::mbar_arrive(&bars->q_ready[g][qs]);
      }
      for (int j = 0; j < t.nb && ok; ++j) {
        const int st = ku % kStages;
        ok = wait_bar(&bars->kv_full[st], (ku / kStages) & 1, ctl);
        ++ku;
        if (!ok) break;
        uint8_t* ktile = kvbuf + st * 2 * kTileBytes;
        if (MODE == 1) {
          for (int r = pt; r < rows; r += 64) {
            float v[32];
            load_row_bf16(ktile, r, v);
            kcol[st * 128 + r] = inv_norm(v);
          }
        }
        if (MODE == 2) {
          // rotate this thread's rows (at most two), then one power-of-two
          // scale for the whole block from the block's largest component
          float v0[32], v1[32];
          float mx = 0.f;
          const int r0 = pt, r1 = pt + 64;
          if (r0 < rows) {
            load_row_bf16(ktile, r0, v0);
            rope_rotate(v0, swin_local_coord(t.y0 + j * t.R + r0 / t.lx, M, s),
                        swin_local_coord(t.x0 + r0 % t.lx, M, s), rcos, rsin);
            mx = absmax(v0);
          }
          if (r1 < rows) {
            load_row_bf16(ktile, r1, v1);
            rope_rotate(v1, swin_local_coord(t.y0 + j * t.R + r1 / t.lx, M, s),
                        swin_local_coord(t.x0 + r1 % t.lx, M, s), rcos, rsin);
            mx = fmaxf(mx, absmax(v1));
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
          const int par = (ku - 1) & 1;
          if (lane == 0) kred[par * 2 + (warp - 2)] = mx;
          ptx::named_bar_sync(1, 64);
          const float sc = pow2_scale(fmaxf(kred[par * 2], kred[par * 2 + 1]));
          if (r0 < rows) store_row_f16(ktile, r0, v0, sc);
          if (r1 < rows) store_row_f16(ktile, r1, v1, sc);
          if (pt == 0) kscale[st] = 1.0f / sc;
          ptx::fence_proxy_async_smem();
        }
        ptx::mbar_arrive(&bars->kv_ready[st]);
      }
    }
  }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 216;\n" ::: "memory");
    // ================================================================ softmax
    const int g = (warp - 4) >> 2;            // warpgroup 0 or 1
    const int t = threadIdx.x - 128 - g * 128;  // row of the tile = TMEM lane
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem_base + g * 256 + lane_off;
    const uint32_t tP = tS + 128, tO = tS + 192;
    const float cscale = kLog2eF * rsqrtf(32.0f);
    const int R2 = 2 * M - 1;
    uint32_t qu = 0, s_cnt = 0, o_cnt = 0, ku = 0;
    bool ok = true;
    for (long long it = first; it < p.n_items && ok; it += step) {
      const Task tk = decode(p, it);
      const uint32_t ku0 = ku;
      if (tk.any) ku += tk.nb;  // K/V block uses of this item (both warpgroups)
      if (!tk.valid[g]) continue;
      const int qs = qu & 1;
      ok = wait_bar(&bars->q_ready[g][qs], (qu >> 1) & 1, ctl);
      ok = __all_sync(0xffffffffu, ok);
      ++qu;
      if (!ok) break;
      // per-row score scale: mode 1 log2e / (tau |q|), mode 2 log2e / (sqrt(d) 2^e)
      const float alpha = MODE == 0 ? cscale : qscale[(g * 2 + qs) * 128 + t];
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&bars->q_empty[g][qs]);
      const bool row_ok = t < tk.nq[g];
      const int qy = tk.tile[g] * tk.R + t / tk.lx, qx = t % tk.lx;
      const int bbase = (qy + M - 1) * R2 + (qx + M - 1);
      const int* kof = kofs + tk.cls * 128;
      const float* tab = p.table;
      float m_run = -INFINITY;
      for (int j = 0; j < tk.nb; ++j) {
        ok = wait_bar(&bars->s_full[g], s_cnt & 1, ctl);
        ok = __all_sync(0xffffffffu, ok);
        ++s_cnt;
        if (!ok) break;
        ptx::tc_fence_after();
        float x[128];
        {
          uint32_t r0[32], r1[32], r2[32], r3[32];
          ptx::tmem_ld32(tS, r0);
          ptx::tmem_ld32(tS + 32, r1);
          ptx::tmem_ld32(tS + 64, r2);
          ptx::tmem_ld32(tS + 96, r3);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            x[e] = __uint_as_float(r0[e]);
            x[32 + e] = __uint_as_float(r1[e]);
            x[64 + e] = __uint_as_float(r2[e]);
            x[96 + e] = __uint_as_float(r3[e]);
          }
        }
        ptx::tc_fence_before();
        ptx::mbar_arrive(&bars->s_free[g]);
        float ascale = alpha;
        const uint32_t u = ku0 + j, ust = u % kStages;
        if (MODE != 0) {
          // the block's K scales (mode 2: one per block, mode 1: 1/|k| per
          // column) were written by prep before it released kv_ready
          ok = wait_bar(&bars->kv_ready[ust], (u / kStages) & 1, ctl);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          if (MODE == 2) ascale = alpha * kscale[ust];
        }
        const float4* kc4 = reinterpret_cast<const float4*>(kcol + ust * 128);
        const int nk_all = tk.n - j * tk.R * tk.lx;
        const int nk = nk_all < tk.R * tk.lx ? nk_all : tk.R * tk.lx;
        const int jb = bbase - j * tk.R * R2;
        float mb = -INFINITY;
#pragma unroll
        for (int c = 0; c < 128; ++c) {
          float v;
          if (MODE == 1) {
            const float4 kc = kc4[c >> 2];  // same address in every lane: broadcast
            const float kcv = (c & 3) == 0 ? kc.x : (c & 3) == 1 ? kc.y : (c & 3) == 2 ? kc.z : kc.w;
            v = (x[c] * kcv) * ascale;
          } else {
            v = x[c] * ascale;
          }
          if (MODE != 2) {
            if (tab != nullptr && row_ok && c < nk)
              v = fmaf(__ldg(tab + (size_t)(jb - kof[c]) * p.heads + tk.h), kLog2eF, v);
          }
          v = c < nk ? v : -INFINITY;
          x[c] = v;
          mb = fmaxf(mb, v);
        }
        float factor = 1.f;
        bool rescale = false;
        if (j == 0) {
          m_run = mb;
        } else if (mb > m_run) {
          factor = ptx::ex2_approx(m_run - mb);
          m_run = mb;
          rescale = true;
        }
        if (j > 0) {
          // PV of the previous block must be done: it reads P and writes O
          ok = wait_bar(&bars->o_done[g], o_cnt & 1, ctl);
          ok = __all_sync(0xffffffffu, ok);
          ++o_cnt;
          if (!ok) break;
          ptx::tc_fence_after();
          if (__any_sync(0xffffffffu, rescale)) {
            // O and its row-sum column follow the new maximum
            uint32_t o[32], o2[16];
            ptx::tmem_ld32(tO, o);
            ptx::tmem_ld16(tO + 32, o2);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * factor);
#pragma unroll
            for (int e = 0; e < 16; ++e) o2[e] = __float_as_uint(__uint_as_float(o2[e]) * factor);
            ptx::tmem_st32(tO, o);
            ptx::tmem_st16(tO + 32, o2);
          }
        }
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          uint32_t pk[32];
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const float p0 = ptx::ex2_approx(x[64 * hf + 2 * c] - m_run);
            const float p1 = ptx::ex2_approx(x[64 * hf + 2 * c + 1] - m_run);
            pk[c] = ptx::pack_bf16x2(p0, p1);
          }
          ptx::tmem_st32(tP + 32 * hf, pk);
        }
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        ptx::mbar_arrive(&bars->p_full[g]);
      }
      if (!ok) break;
      // epilogue: O / l to global memory
      ok = wait_bar(&bars->o_done[g], o_cnt & 1, ctl);
      ok = __all_sync(0xffffffffu, ok);
      ++o_cnt;
      if (!ok) break;
      ptx::tc_fence_after();
      uint32_t o[32], o2[16];
      ptx::tmem_ld32(tO, o);
      ptx::tmem_ld16(tO + 32, o2);
      ptx::tmem_wait_ld();
      if (row_ok) {
        const float inv = 1.0f / __uint_as_float(o2[0]);  // row sum of the bf16 P
        const size_t tok = ((size_t)tk.b * p.H + (tk.y0 + qy)) * p.W + (tk.x0 + qx);
        const size_t off = tok * (size_t)(p.heads * 32) + (size_t)tk.h * 32;
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
              w[e] = ptx::pack_bf16x2(__uint_as_float(o[8 * c + 2 * e]) * inv, __uint_as_float(o[8 * c + 2 * e + 1]) * inv);
            dst[c] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
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

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

bool encode_map(CUtensorMap* m, const void* base, const AttnArgs& a, int lx, int R) {
  EncodeTiledFn fn = encode_fn();
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

template <int MODE, bool F32>
swin_status launch_mode(const TcParams& p, int grid, cudaStream_t stream) {
  auto k = attn_tc_kernel<MODE, F32>;
  cudaError_t ea = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemAlloc);
  if (ea != cudaSuccess) return fail(SWIN_ERR_CUDA, "attn_tc smem attribute: %s", cudaGetErrorString(ea));
  k<<<grid, kThreads, kSmemAlloc, stream>>>(p);
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

swin_status launch_attn_tc(const AttnArgs& a, bool f32_out, cudaStream_t stream) {
  if (a.d != 32) return fail(SWIN_ERR_UNSUPPORTED, "tensor-core path needs d == 32, got %d", a.d);
  if (a.M > 64) return fail(SWIN_ERR_UNSUPPORTED, "tensor-core path needs M <= 64");
  TcParams p;
  memset(&p, 0, sizeof(p));
  p.B = a.B; p.H = a.H; p.W = a.W; p.heads = a.heads; p.M = a.M; p.s = a.shift;
  p.nsy = swin_nseg(a.H, a.M, a.shift);
  p.nsx = swin_nseg(a.W, a.M, a.shift);
  const int lxs[3] = {swin_seg_len(0, a.W, a.M, a.shift),
                      p.nsx > 2 ? swin_seg_len(1, a.W, a.M, a.shift) : swin_seg_len(0, a.W, a.M, a.shift),
                      swin_seg_len(p.nsx - 1, a.W, a.M, a.shift)};
  int tiles_max = 1;
  for (int c = 0; c < 3; ++c) {
    p.lx[c] = lxs[c];
    p.R[c] = 128 / lxs[c];
    if (p.R[c] > 256) p.R[c] = 256;
    const int tl = (a.M + p.R[c] - 1) / p.R[c];
    if (tl > tiles_max) tiles_max = tl;
    if (!encode_map(&p.tmap[0][c], a.q, a, p.lx[c], p.R[c]) || !encode_map(&p.tmap[1][c], a.k, a, p.lx[c], p.R[c]) ||
        !encode_map(&p.tmap[2][c], a.v, a, p.lx[c], p.R[c]))
      return fail(SWIN_ERR_CUDA, "cuTensorMapEncodeTiled failed (lx=%d, R=%d)", p.lx[c], p.R[c]);
  }
  p.pmax = (tiles_max + 1) / 2;
  p.n_items = (long long)a.B * a.heads * p.nsy * p.nsx * p.pmax;
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
    case 0: return f32_out ? launch_mode<0, true>(p, grid, stream) : launch_mode<0, false>(p, grid, stream);
    case 1: return f32_out ? launch_mode<1, true>(p, grid, stream) : launch_mode<1, false>(p, grid, stream);
    default: return f32_out ? launch_mode<2, true>(p, grid, stream) : launch_mode<2, false>(p, grid, stream);
  }
}

}  // namespace swin
