// Latencies of the tensor-core round trip the attention kernel is built from,
// on one SM: tcgen05.mma issue to its commit's mbarrier completion (for the
// MMA shapes of one 64-key block: S = Q K^T as two M128 N64 K16 MMAs, O += P V
// as four M128 N48 K16 MMAs with A in TMEM), tcgen05.ld / tcgen05.st of 32
// columns with their waits, and an mbarrier arrival seen by a waiting warp.
//
//   nvcc -gencode arch=compute_100a,code=sm_100a -O3 -std=c++17 -I<package>/csrc \
//        -o ubench_tcgen05 ubench_tcgen05.cu && ./ubench_tcgen05
//
// One CTA of 128 threads; shared-memory operands are zero (their values do
// not change the timing); every wait is bounded.
#include <cstdint>
#include <cstdio>

#include "sm100_ptx.cuh"

using namespace swin;

constexpr int kReps = 64;
constexpr long long kLimit = 100000000ll;  // cycles before a wait gives up

__device__ __forceinline__ bool wait_bounded(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!ptx::mbar_try_wait(bar, parity))
    if (clock64() - t0 > kLimit) return false;
  return true;
}

struct Result {
  long long mma_s[kReps], mma_s_pv[kReps], ld32[kReps], st32[kReps], wake[kReps];
  long long pp_spin[kReps], pp_sleep[kReps], pp_commit[kReps];
  int ok;
};

// A wait as the attention kernel does it: one try_wait, then try_wait with a
// suspend-time hint, bounded.
__device__ __forceinline__ bool wait_hinted(uint64_t* bar, uint32_t parity) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (ptx::mbar_try_wait_sleep(bar, parity, 20000u)) return true;
    if (clock64() - t0 > kLimit) return false;
  }
}

__global__ void __launch_bounds__(128, 1) bench(Result* res) {
  __shared__ __align__(1024) uint8_t a_tile[128 * 64];
  __shared__ __align__(1024) uint8_t b_tile[64 * 64];
  __shared__ __align__(1024) uint8_t v_tile[64 * 64 + 1024];
  __shared__ uint64_t bar[2];
  __shared__ uint32_t tmem_holder;
  __shared__ volatile long long stamp;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < 128 * 64 / 4; i += 128) reinterpret_cast<uint32_t*>(a_tile)[i] = 0;
  for (int i = threadIdx.x; i < 64 * 64 / 4; i += 128) reinterpret_cast<uint32_t*>(b_tile)[i] = 0;
  for (int i = threadIdx.x; i < (64 * 64 + 1024) / 4; i += 128) reinterpret_cast<uint32_t*>(v_tile)[i] = 0;
  if (threadIdx.x == 0) {
    ptx::mbar_init(&bar[0], 1);
    ptx::mbar_init(&bar[1], 1);
    ptx::fence_mbar_init();
    res->ok = 1;
  }
  if (warp == 0) {
    ptx::tmem_alloc(&tmem_holder, 256);
    ptx::tmem_relinquish();
  }
  ptx::fence_proxy_async_smem();
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tbase = tmem_holder;
  const uint64_t ad = ptx::smem_desc(ptx::smem_addr(a_tile), 16, 512, ptx::kSwizzle64B);
  const uint64_t bd = ptx::smem_desc(ptx::smem_addr(b_tile), 16, 512, ptx::kSwizzle64B);
  const uint32_t va = ptx::smem_addr(v_tile);
  const uint64_t vd = ptx::smem_desc(va, 64 * 64, 512, ptx::kSwizzle64B);
  constexpr uint32_t idS = ptx::idesc_f16(0, 0, 0, 0, 64, 128);
  constexpr uint32_t idPV = ptx::idesc_f16(0, 0, 0, 1, 48, 128);
  constexpr uint64_t kStepV = (uint64_t)(1024 >> 4) - ((uint64_t)(1024 >> 4) << 16);
  uint32_t phase = 0;
  // 1) S: two M128 N64 K16 MMAs, commit, wait (issuing thread)
  if (threadIdx.x == 0) {
    for (int r = 0; r < kReps && res->ok; ++r) {
      const long long t0 = clock64();
      ptx::mma_ss(tbase, ad, bd, idS, 0);
      ptx::mma_ss(tbase, ad + 2, bd + 2, idS, 1);
      ptx::mma_commit(&bar[0]);
      if (!wait_bounded(&bar[0], phase)) res->ok = 0;
      phase ^= 1;
      res->mma_s[r] = clock64() - t0;
    }
    // 2) S then PV (4 MMAs, A = P from TMEM columns 128..) as one block's work
    for (int r = 0; r < kReps && res->ok; ++r) {
      const long long t0 = clock64();
      ptx::mma_ss(tbase, ad, bd, idS, 0);
      ptx::mma_ss(tbase, ad + 2, bd + 2, idS, 1);
      for (int kk = 0; kk < 4; ++kk)
        ptx::mma_ts(tbase + 192, tbase + 128 + kk * 8, vd + kk * kStepV, idPV, kk > 0 ? 1u : 0u);
      ptx::mma_commit(&bar[0]);
      if (!wait_bounded(&bar[0], phase)) res->ok = 0;
      phase ^= 1;
      res->mma_s_pv[r] = clock64() - t0;
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  // 3) tcgen05.ld / st of 32 columns, each followed by its wait (warp 0)
  if (warp == 0) {
    uint32_t v[32];
    for (int r = 0; r < kReps; ++r) {
      const long long t0 = clock64();
      ptx::tmem_ld32(tbase, v);
      ptx::tmem_wait_ld();
      const long long t1 = clock64();
      for (int e = 0; e < 32; ++e) v[e] += (uint32_t)r;
      const long long t2 = clock64();
      ptx::tmem_st32(tbase + 64, v);
      ptx::tmem_wait_st();
      const long long t3 = clock64();
      if (lane == 0) {
        res->ld32[r] = t1 - t0;
        res->st32[r] = t3 - t2;
      }
    }
  }
  __syncthreads();
  // 4) an arrival seen by a waiting warp (warp 1 waits, warp 0 arrives); the
  // trip count is fixed so that every thread reaches every __syncthreads
  for (int r = 0; r < kReps; ++r) {
    if (warp == 1 && lane == 0) {
      const bool okw = wait_bounded(&bar[1], (uint32_t)(r & 1));
      const long long t1 = clock64();
      res->wake[r] = t1 - stamp;
      if (!okw) res->ok = 0;
    } else if (warp == 0 && lane == 0) {
      const long long t0 = clock64();
      while (clock64() - t0 < 2000) {
      }
      stamp = clock64();
      __threadfence_block();
      ptx::mbar_arrive(&bar[1]);
    }
    __syncthreads();
  }
  // 5) ping-pong between lane 0 of warp 0 and lane 0 of warp 1 through two
  // mbarriers: per round trip, A arrives on p0 and waits p1; B waits p0 and
  // arrives on p1 (plain arrive, or tcgen05.commit with no MMA pending).
  // Three flavours: spinning try_wait; the hinted wait; commit as B's arrive.
  __shared__ uint64_t pb[6];
  if (threadIdx.x == 0) {
    for (int i = 0; i < 6; ++i) ptx::mbar_init(&pb[i], 1);
    ptx::fence_mbar_init();
  }
  __syncthreads();
  for (int fl = 0; fl < 3; ++fl) {
    uint64_t* p0 = &pb[2 * fl];
    uint64_t* p1 = &pb[2 * fl + 1];
    long long* out = fl == 0 ? res->pp_spin : (fl == 1 ? res->pp_sleep : res->pp_commit);
    if (warp == 0 && lane == 0) {
      for (int r = 0; r < kReps; ++r) {
        const long long t0 = clock64();
        ptx::mbar_arrive(p0);
        const bool okw = fl == 0 ? wait_bounded(p1, (uint32_t)(r & 1)) : wait_hinted(p1, (uint32_t)(r & 1));
        out[r] = clock64() - t0;
        if (!okw) res->ok = 0;
      }
    } else if (warp == 1 && lane == 0) {
      for (int r = 0; r < kReps; ++r) {
        const bool okw = fl == 0 ? wait_bounded(p0, (uint32_t)(r & 1)) : wait_hinted(p0, (uint32_t)(r & 1));
        if (!okw) res->ok = 0;
        if (fl == 2) {
          ptx::tc_fence_after();
          ptx::mma_commit(p1);
        } else {
          ptx::mbar_arrive(p1);
        }
      }
    }
    __syncthreads();
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tbase, 256);
  }
}

static void summary(const char* name, const long long* v) {
  long long s[kReps];
  for (int i = 0; i < kReps; ++i) s[i] = v[i];
  for (int i = 0; i < kReps; ++i)
    for (int j = i + 1; j < kReps; ++j)
      if (s[j] < s[i]) {
        long long t = s[i];
        s[i] = s[j];
        s[j] = t;
      }
  printf("%-58s min %6lld  median %6lld  max %6lld cycles\n", name, s[0], s[kReps / 2], s[kReps - 1]);
}

int main() {
  Result* d = nullptr;
  if (cudaMalloc(&d, sizeof(Result)) != cudaSuccess) return 1;
  bench<<<1, 128>>>(d);
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) {
    printf("error %s\n", cudaGetErrorString(e));
    return 1;
  }
  Result h;
  cudaMemcpy(&h, d, sizeof(Result), cudaMemcpyDeviceToHost);
  printf("# one SM, %d repetitions; ok=%d\n", kReps, h.ok);
  summary("S: 2x mma M128 N64 K16 (smem A, B) -> commit -> wait", h.mma_s);
  summary("S + PV: 2x above + 4x mma M128 N48 K16 (A in TMEM)", h.mma_s_pv);
  summary("tcgen05.ld 32x32b.x32 + wait::ld", h.ld32);
  summary("tcgen05.st 32x32b.x32 + wait::st", h.st32);
  summary("mbarrier arrive (warp 0) -> try_wait succeeds (warp 1)", h.wake);
  summary("ping-pong round trip, spinning try_wait", h.pp_spin);
  summary("ping-pong round trip, try_wait + suspend hint", h.pp_sleep);
  summary("ping-pong round trip, hinted waits, B arrives by commit", h.pp_commit);
  cudaFree(d);
  return h.ok ? 0 : 1;
}
