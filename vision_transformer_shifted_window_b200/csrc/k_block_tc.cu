// The block steps either side of the attention ("Swin Transformer V2" wiki
// card, Method item 1 "Residual post-norm", §3.2, fig. 1, swin_v2_block
// pseudocode) as fused tensor-core kernels, for bf16 inputs whose channel
// count C = heads * d is a multiple of 32 and at most 128 (the weights stay
// resident in shared memory):
//   qkv        q | k | v = x W_qkv^T + b_qkv
//   post-norm  out = x + LN(a W_o^T + b_o) * gamma + beta
// Work unit: one tile of 128 tokens (one TMEM lane per token).  Per tile the
// input rows arrive by TMA (64-byte swizzle, 32-channel column chunks), the
// products are tcgen05 MMAs (M = 128, N = C per output, K = 16 steps) into a
// ring of TMEM accumulator slots of C columns (so the MMAs of the next tile
// run while the epilogue reads this one), and the epilogue (bias, or bias + layer norm + residual, in fp32)
// reads one row per thread from TMEM, rounds each output once and writes it
// through a shared-memory staging tile and a TMA store.  The accumulation
// order does not depend on the output type, so a bf16 output is exactly the
// fp32 one rounded to nearest even.
//
// Warps: 0 TMA producer (weights once, then input tiles into a ring of
// stages), 1 MMA issuer (and TMEM owner), 2-5 and 6-9 two epilogue
// warpgroups taking alternate products (warp w reads TMEM lanes
// 32 (w % 4) ...; one warpgroup where shared memory holds a single set of
// staging tiles).  Every wait is bounded; on time-out the kernel
// records SWIN_ERR_TIMEOUT, drains what it issued and returns.
#include <cuda.h>
#include <cuda_bf16.h>

#include "sm100_ptx.cuh"
#include "swin_common.cuh"
#include "tma_encode.cuh"

namespace swin {
namespace {

constexpr int kTok = 128;                // tokens per tile
constexpr int kChunk = kTok * 64;        // one column chunk of a tile: 128 rows x 64 bytes
constexpr int kThreadsBlk = 320;
constexpr int kMaxSmem = 227 * 1024;
constexpr long long kWaitLimit = 4000000000ll;  // clock64 cycles (~2 s)
constexpr int kMaxSlots = 6;                    // TMEM accumulator slots

struct BlkParams {
  CUtensorMap map_in;      // [tokens][C] bf16: x (qkv) or the attention output a (post-norm)
  CUtensorMap map_w;       // [nparts C][C] bf16 weights
  CUtensorMap map_res;     // [tokens][C] bf16 residual x (post-norm)
  CUtensorMap map_out[3];  // [tokens][C] outputs (bf16 or fp32)
  const float* bias;       // [nparts C] or null
  const float* gamma;      // [C] or null (post-norm)
  const float* beta;       // [C] or null (post-norm)
  float eps;
  int C, nparts, ntiles, nstages, nout;  // nout: staging buffers per epilogue warpgroup (1 or 2)
  int nepi;                              // epilogue warpgroups (1 or 2)
  int nslots;                            // TMEM accumulator slots of C columns
  int off_w, off_in, off_res, off_out, off_vec, off_bar;
  uint32_t tmem_cols;
  int* status;
};

__device__ __forceinline__ uint32_t swz64(int row, int chunk) {
  // byte offset of 16-byte chunk `chunk` of 64-byte row `row` under 64B swizzle
  return (uint32_t)(row * 64 + ((chunk ^ ((row >> 1) & 3)) << 4));
}

__device__ __forceinline__ void tma_load_2d(void* dst, const void* tmap, uint64_t* bar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(ptx::smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(ptx::smem_addr(bar)), "r"(c0), "r"(c1)
      : "memory");
}

__device__ __forceinline__ void tma_store_2d(const void* tmap, const void* src, int c0, int c1) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(tmap)),
               "r"(ptx::smem_addr(src)), "r"(c0), "r"(c1)
               : "memory");
}

__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// at most 1 (0) committed store groups may still be reading shared memory
__device__ __forceinline__ void bulk_wait_read1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

struct Wait {
  volatile int* abort;
  int* status;
  // bounded wait on an mbarrier phase; false if it ran out or another role aborted
  __device__ __forceinline__ bool operator()(uint64_t* bar, uint32_t parity) const {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
      if (ptx::mbar_try_wait_sleep(bar, parity, 20000u)) return true;
      if (*abort) return false;
      if (clock64() - t0 > kWaitLimit) {
        atomicOr(status, (int)SWIN_ERR_TIMEOUT);
        *abort = 1;
        return false;
      }
    }
  }
};

template <bool F32>
__device__ __forceinline__ void store_val(uint8_t* stage, int r, int col, const float (&v)[32]);

// 32 consecutive columns (col = 32 cc) of row r into the staging tile:
// bf16: chunk cc (32 columns of 2 bytes); fp32: chunks 2 cc, 2 cc + 1 (16 columns of 4 bytes)
template <>
__device__ __forceinline__ void store_val<false>(uint8_t* stage, int r, int col, const float (&v)[32]) {
  uint8_t* ch = stage + (col / 32) * kChunk;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint4 w;
    w.x = ptx::pack_bf16x2(v[8 * c], v[8 * c + 1]);
    w.y = ptx::pack_bf16x2(v[8 * c + 2], v[8 * c + 3]);
    w.z = ptx::pack_bf16x2(v[8 * c + 4], v[8 * c + 5]);
    w.w = ptx::pack_bf16x2(v[8 * c + 6], v[8 * c + 7]);
    *reinterpret_cast<uint4*>(ch + swz64(r, c)) = w;
  }
}

template <>
__device__ __forceinline__ void store_val<true>(uint8_t* stage, int r, int col, const float (&v)[32]) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint8_t* ch = stage + (col / 16 + h) * kChunk;
#pragma unroll
    for (int c = 0; c < 4; ++c)
      *reinterpret_cast<float4*>(ch + swz64(r, c)) =
          make_float4(v[16 * h + 4 * c], v[16 * h + 4 * c + 1], v[16 * h + 4 * c + 2], v[16 * h + 4 * c + 3]);
  }
}

template <bool PN, bool F32>
__global__ void __launch_bounds__(kThreadsBlk, 1) block_tc_kernel(const __grid_constant__ BlkParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (static_cast<uint32_t>(__cvta_generic_to_shared(smem_raw)) & 1023u)) & 1023u);
  const int C = p.C, N = p.nparts * C, KC = C / 32, S = p.nstages;
  uint8_t* sw = smem + p.off_w;      // [KC][N rows][64 B]
  uint8_t* sin = smem + p.off_in;    // [S][KC][128 rows][64 B]
  uint8_t* sres = smem + p.off_res;  // [S][KC][128 rows][64 B]  (post-norm)
  uint8_t* sout = smem + p.off_out;  // [nepi][nout][C * out bytes / 64][128 rows][64 B]
  float* sbias = reinterpret_cast<float*>(smem + p.off_vec);  // [N]
  float* sgam = sbias + N;                                    // [C] (post-norm)
  float* sbet = sgam + C;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + p.off_bar);
  uint64_t* w_full = bars;
  uint64_t* in_full = bars + 1;
  uint64_t* in_empty = bars + 1 + S;
  const int NS = p.nslots;
  uint64_t* slot_full = bars + 1 + 2 * S;
  uint64_t* slot_empty = slot_full + NS;
  uint64_t* drain = slot_empty + NS;
  uint32_t* holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(holder + 1);
  volatile int* drain_flag = reinterpret_cast<volatile int*>(holder + 2);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int out_bytes = F32 ? 4 : 2;
  const int stage_bytes = C * out_bytes * kTok;  // one output tile

  if (threadIdx.x == 0) {
    ptx::mbar_init(w_full, 1);
    for (int s = 0; s < S; ++s) {
      ptx::mbar_init(in_full + s, 1);
      ptx::mbar_init(in_empty + s, PN ? 2 : 1);  // MMA done (and, post-norm, residual read)
    }
    for (int k = 0; k < NS; ++k) {
      ptx::mbar_init(slot_full + k, 1);
      ptx::mbar_init(slot_empty + k, 4);  // one arrival per epilogue warp
    }
    ptx::mbar_init(drain, 1);
    *abort_flag = 0;
    *drain_flag = 0;
    ptx::fence_mbar_init();
  }
  for (int i = threadIdx.x; i < N; i += kThreadsBlk) sbias[i] = p.bias ? __ldg(p.bias + i) : 0.f;
  if (PN)
    for (int i = threadIdx.x; i < C; i += kThreadsBlk) {
      sgam[i] = p.gamma ? __ldg(p.gamma + i) : 1.f;
      sbet[i] = p.beta ? __ldg(p.beta + i) : 0.f;
    }
  if (warp == 1) {
    ptx::tmem_alloc(holder, p.tmem_cols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = *holder;
  const Wait wait{abort_flag, p.status};
  const Wait wait_drain{drain_flag, p.status};

  if (warp == 0) {
    // ================================================================ producer
    if (lane == 0) {
      ptx::prefetch_tmap(&p.map_in);
      ptx::prefetch_tmap(&p.map_w);
      if (PN) ptx::prefetch_tmap(&p.map_res);
      ptx::mbar_arrive_expect_tx(w_full, (uint32_t)(N * C * 2));
      for (int kc = 0; kc < KC; ++kc)
        for (int part = 0; part < p.nparts; ++part)
          tma_load_2d(sw + (kc * N + part * C) * 64, &p.map_w, w_full, kc * 32, part * C);
      bool ok = true;
      int i = 0;
      for (int tile = blockIdx.x; tile < p.ntiles && ok; tile += gridDim.x, ++i) {
        const int s = i % S;
        if (i >= S) ok = wait(in_empty + s, ((i / S) - 1) & 1);
        if (!ok) break;
        ptx::mbar_arrive_expect_tx(in_full + s, (uint32_t)(KC * kChunk * (PN ? 2 : 1)));
        for (int kc = 0; kc < KC; ++kc) {
          tma_load_2d(sin + (s * KC + kc) * kChunk, &p.map_in, in_full + s, kc * 32, tile * kTok);
          if (PN) tma_load_2d(sres + (s * KC + kc) * kChunk, &p.map_res, in_full + s, kc * 32, tile * kTok);
        }
      }
      // copies still landing (after an abort) complete before the CTA exits
      wait_drain(w_full, 0);
      for (int u = i > S ? i - S : 0; u < i; ++u) wait_drain(in_full + u % S, (u / S) & 1);
    }
  } else if (warp == 1) {
    // ================================================================ MMA
    if (lane == 0) {
      constexpr uint32_t kIdescBase = ptx::idesc_f16(1, 1, 0, 0, 0, 128);  // bf16 x bf16, K-major, M = 128
      const uint32_t idesc = kIdescBase | (((uint32_t)C >> 3) << 17);       // N = C
      const uint64_t ad0 = ptx::smem_desc(ptx::smem_addr(sin), 16, 512, ptx::kSwizzle64B);
      const uint64_t bd0 = ptx::smem_desc(ptx::smem_addr(sw), 16, 512, ptx::kSwizzle64B);
      bool ok = wait(w_full, 0);
      int i = 0, u = 0;  // tiles, (tile, output) products issued
      for (int tile = blockIdx.x; tile < p.ntiles && ok; tile += gridDim.x, ++i) {
        const int s = i % S;
        ok = wait(in_full + s, (i / S) & 1);
        for (int part = 0; part < p.nparts && ok; ++part, ++u) {
          const int k = u % NS;
          if (u >= NS) ok = wait(slot_empty + k, ((u / NS) - 1) & 1);  // the epilogue has read the slot
          if (!ok) break;
          ptx::tc_fence_after();
          for (int kc = 0; kc < KC; ++kc)
            for (int ks = 0; ks < 2; ++ks) {
              const uint64_t a = ad0 + (uint64_t)(((s * KC + kc) * kChunk + ks * 32) >> 4);
              const uint64_t b = bd0 + (uint64_t)(((kc * N + part * C) * 64 + ks * 32) >> 4);
              ptx::mma_ss(tmem_base + k * C, a, b, idesc, (kc | ks) != 0 ? 1u : 0u);
            }
          ptx::mma_commit(slot_full + k);
        }
        if (!ok) break;
        ptx::mma_commit(in_empty + s);
      }
      ptx::mma_commit(drain);
      wait_drain(drain, 0);
    }
  } else if ((warp - 2) >> 2 < p.nepi) {
    // ================================================================ epilogue
    const int ew = (warp - 2) >> 2;             // epilogue warpgroup: products u with u % nepi == ew
    const int et = (threadIdx.x - 64) & 127;    // 0..127 within the warpgroup
    const int bar = 1 + ew;                     // its named barrier
    const int lg = warp & 3;                    // TMEM lane group of this warp
    const int r = lg * 32 + lane;               // row of the tile
    const uint32_t tl = tmem_base + ((uint32_t)(lg * 32) << 16);
    uint8_t* sout_w = sout + ew * p.nout * stage_bytes;
    int ob = 0;
    bool ok = true;
    int i = 0, u = 0;  // tiles, (tile, output) products
    for (int tile = blockIdx.x; tile < p.ntiles && ok; tile += gridDim.x, ++i) {
      const int s = i % S;
      bool mine_tile = false;  // this warpgroup read the tile's residual rows
      for (int part = 0; part < p.nparts; ++part, ++u) {
        if (u % p.nepi != ew) continue;
        mine_tile = true;
        const int k = u % NS;
        ok = __all_sync(0xffffffffu, wait(slot_full + k, (u / NS) & 1) && (!PN || wait(in_full + s, (i / S) & 1)));
        ok = ptx::named_bar_and(bar, 128, ok);
        if (!ok) break;
        ptx::tc_fence_after();
        const uint32_t ts = tl + k * C;  // this product's accumulator slot
        float mean = 0.f, rstd = 0.f;
        if (PN) {
          float sum = 0.f;
          for (int cc = 0; cc < KC; ++cc) {
            uint32_t v[32];
            ptx::tmem_ld32(ts + cc * 32, v);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) sum += __uint_as_float(v[j]) + sbias[cc * 32 + j];
          }
          mean = sum / (float)C;
          float ss = 0.f;
          for (int cc = 0; cc < KC; ++cc) {
            uint32_t v[32];
            ptx::tmem_ld32(ts + cc * 32, v);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const float dv = __uint_as_float(v[j]) + sbias[cc * 32 + j] - mean;
              ss += dv * dv;
            }
          }
          rstd = rsqrtf(ss / (float)C + p.eps);
        }
        uint8_t* stage = sout_w + ob * stage_bytes;
        // the store that last read this staging buffer has finished reading it
        if (et == 0) {
          if (p.nout == 2) bulk_wait_read1();
          else bulk_wait_read0();
        }
        ptx::named_bar_sync(bar, 128);
        for (int cc = 0; cc < KC; ++cc) {
          uint32_t v[32];
          ptx::tmem_ld32(ts + cc * 32, v);
          ptx::tmem_wait_ld();
          float o[32];
          if (PN) {
            const uint8_t* xr = sres + (s * KC + cc) * kChunk;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const uint4 xw = *reinterpret_cast<const uint4*>(xr + swz64(r, c));
              const uint32_t xs[4] = {xw.x, xw.y, xw.z, xw.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int j = 8 * c + 2 * e, col = cc * 32 + j;
                const float x0 = __uint_as_float(xs[e] << 16), x1 = __uint_as_float(xs[e] & 0xFFFF0000u);
                o[j] = x0 + (__uint_as_float(v[j]) + sbias[col] - mean) * rstd * sgam[col] + sbet[col];
                o[j + 1] =
                    x1 + (__uint_as_float(v[j + 1]) + sbias[col + 1] - mean) * rstd * sgam[col + 1] + sbet[col + 1];
              }
            }
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) o[j] = __uint_as_float(v[j]) + sbias[part * C + cc * 32 + j];
          }
          store_val<F32>(stage, r, cc * 32, o);
        }
        // every TMEM read of the slot is complete: the MMAs may reuse it
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(slot_empty + k);
        ptx::fence_proxy_async_smem();
        ptx::named_bar_sync(bar, 128);
        if (et == 0) {
          const int nbox = F32 ? C / 16 : C / 32, bw = F32 ? 16 : 32;
          for (int c = 0; c < nbox; ++c) tma_store_2d(&p.map_out[part], stage + c * kChunk, c * bw, tile * kTok);
          bulk_commit();
        }
        if (p.nout == 2) ob ^= 1;
      }
      if (!ok) break;
      if (PN && mine_tile && et == 0) ptx::mbar_arrive(in_empty + s);  // residual rows read (the barrier above)
    }
    if (et == 0) bulk_wait_all();
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem_base, p.tmem_cols);
  }
}

bool encode_2d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int esize, int cols, long long rows,
               int box_cols, int box_rows) {
  EncodeTiledFn fn = tma_encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * esize};
  const cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) !=
                                                 cudaSuccess)
    return 148;
  return n > 0 ? n : 148;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace

// Shared-memory plan: weights, `stages` input (and residual) tiles, `nout`
// staging tiles per epilogue warpgroup, the bias / gamma / beta vectors and
// the barriers; two epilogue warpgroups where they fit, then the deepest ring
// (3 stages at most) and staging (2 tiles at most).
static bool plan_smem(BlkParams& p, bool pn, bool f32_out) {
  const int C = p.C, N = p.nparts * C;
  for (int nepi = 2; nepi >= 1; --nepi)
  for (int S = 3; S >= 2; --S)
    for (int nout = 2; nout >= 1; --nout) {
      int off = 0;
      p.off_w = off;
      off += N * C * 2;
      p.off_in = off;
      off += S * C * kTok * 2;
      p.off_res = off;
      if (pn) off += S * C * kTok * 2;
      p.off_out = off;
      off += nepi * nout * C * kTok * (f32_out ? 4 : 2);
      p.off_vec = off;
      off += ((N + 2 * C) * 4 + 15) / 16 * 16;
      p.off_bar = off;
      off += (2 + 2 * S + 2 * kMaxSlots) * 8 + 16;
      if (off + 1024 <= kMaxSmem) {
        p.nstages = S;
        p.nout = nout;
        p.nepi = nepi;
        return true;
      }
    }
  return false;
}

// The fused kernels take bf16 inputs with C a multiple of 32 up to 128 whose
// shared-memory plan fits with fp32 outputs (the larger staging tile), so that
// both output types of one shape run the same kernel.
bool block_tc_supported(int C, bool bf16_in, bool postnorm) {
  if (!bf16_in || C % 32 != 0 || C < 32 || C > 128) return false;
  BlkParams p{};
  p.C = C;
  p.nparts = postnorm ? 1 : 3;
  return plan_smem(p, postnorm, true);
}

static swin_status launch_block_tc(BlkParams& p, bool pn, bool f32_out, cudaStream_t stream) {
  if (!plan_smem(p, pn, f32_out)) return fail(SWIN_ERR_UNSUPPORTED, "block kernel: C = %d does not fit", p.C);
  const int smem = p.off_bar + (2 + 2 * p.nstages + 2 * kMaxSlots) * 8 + 16 + 1024;
  p.nslots = 512 / p.C < kMaxSlots ? 512 / p.C : kMaxSlots;
  if (p.nslots < p.nparts) p.nslots = p.nparts;  // C <= 128: at least 4 slots
  p.tmem_cols = 32;
  while ((int)p.tmem_cols < p.nslots * p.C) p.tmem_cols *= 2;
  p.status = status_word();
  const int grid = p.ntiles < sm_count() ? p.ntiles : sm_count();
  if (grid == 0) return SWIN_OK;
  auto go = [&](auto kern) -> swin_status {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return fail(SWIN_ERR_CUDA, "block kernel smem attribute: %s", cudaGetErrorString(e));
    kern<<<grid, kThreadsBlk, smem, stream>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return fail(SWIN_ERR_CUDA, "block kernel launch: %s", cudaGetErrorString(e));
    return SWIN_OK;
  };
  if (pn) return f32_out ? go(block_tc_kernel<true, true>) : go(block_tc_kernel<true, false>);
  return f32_out ? go(block_tc_kernel<false, true>) : go(block_tc_kernel<false, false>);
}

swin_status launch_qkv_proj_tc(const void* x, const void* w_qkv, const float* b_qkv, void* q, void* k, void* v,
                               bool f32_out, int tokens, int C, cudaStream_t stream) {
  const void* ptrs[5] = {x, w_qkv, q, k, v};
  for (const void* ptr : ptrs)
    if (!aligned16(ptr)) return fail(SWIN_ERR_INVALID_ARG, "block kernel: operands must be 16-byte aligned");
  BlkParams p{};
  p.C = C;
  p.nparts = 3;
  p.ntiles = (tokens + kTok - 1) / kTok;
  p.bias = b_qkv;
  const CUtensorMapDataType odt = f32_out ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  void* outs[3] = {q, k, v};
  bool ok = encode_2d(&p.map_in, x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, C, tokens, 32, kTok) &&
            encode_2d(&p.map_w, w_qkv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, C, 3LL * C, 32, C);
  for (int i = 0; i < 3 && ok; ++i)
    ok = encode_2d(&p.map_out[i], outs[i], odt, f32_out ? 4 : 2, C, tokens, f32_out ? 16 : 32, kTok);
  if (!ok) return fail(SWIN_ERR_CUDA, "cuTensorMapEncodeTiled failed (block kernel)");
  return launch_block_tc(p, false, f32_out, stream);
}

swin_status launch_proj_postnorm_tc(const void* a, const void* w_o, const float* b_o, const void* x,
                                    const float* gamma, const float* beta, float eps, void* out, bool f32_out,
                                    int tokens, int C, cudaStream_t stream) {
  const void* ptrs[4] = {a, w_o, x, out};
  for (const void* ptr : ptrs)
    if (!aligned16(ptr)) return fail(SWIN_ERR_INVALID_ARG, "block kernel: operands must be 16-byte aligned");
  BlkParams p{};
  p.C = C;
  p.nparts = 1;
  p.ntiles = (tokens + kTok - 1) / kTok;
  p.bias = b_o;
  p.gamma = gamma;
  p.beta = beta;
  p.eps = eps;
  const CUtensorMapDataType odt = f32_out ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const bool ok = encode_2d(&p.map_in, a, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, C, tokens, 32, kTok) &&
                  encode_2d(&p.map_w, w_o, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, C, C, 32, C) &&
                  encode_2d(&p.map_res, x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, C, tokens, 32, kTok) &&
                  encode_2d(&p.map_out[0], out, odt, f32_out ? 4 : 2, C, tokens, f32_out ? 16 : 32, kTok);
  if (!ok) return fail(SWIN_ERR_CUDA, "cuTensorMapEncodeTiled failed (block kernel)");
  return launch_block_tc(p, true, f32_out, stream);
}

}  // namespace swin
