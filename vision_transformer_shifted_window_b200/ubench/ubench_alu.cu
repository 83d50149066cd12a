// Per-SM throughput of the instructions the tensor-core softmax is built from
// (one attended pair = one exponential plus a few FMA-pipe and ALU ops), so
// that the split of the exponentials between the MUFU and an FMA-pipe
// polynomial can be chosen from measured rates instead of guesses.
//
//   nvcc -gencode arch=compute_100a,code=sm_100a -O3 -o ubench_alu ubench_alu.cu && ./ubench_alu
//
// Every test runs 16 warps per SM (4 per scheduler), each thread a loop of 8
// independent dependency chains, and reports element operations per clock per
// SM (a packed pair instruction counts two).  The grid is one CTA per SM;
// clock64 brackets the loop in each CTA and the slowest CTA is taken.
#include <cstdio>
#include <cstdint>

#define CK(x)                                                                   \
  do {                                                                          \
    cudaError_t e_ = (x);                                                       \
    if (e_ != cudaSuccess) {                                                    \
      printf("CUDA error %s at %s:%d\n", cudaGetErrorString(e_), __FILE__, __LINE__); \
      return 1;                                                                 \
    }                                                                           \
  } while (0)

constexpr int kIters = 4096;
constexpr int kChains = 8;
constexpr int kThreads = 512;

enum Op {
  kEx2F32, kEx2Bf16x2, kFfma, kFfma2, kFadd2, kMax3, kCvtBf16x2, kLea, kMixEx2Ffma2, kMixEx2Ffma2x3, kNumOps
};
static const char* kNames[kNumOps] = {
    "ex2.approx.ftz.f32", "ex2.approx.ftz.bf16x2", "fma.rn.f32", "fma.rn.f32x2", "add.rn.f32x2",
    "max.f32 (3 inputs)", "cvt.rn.bf16x2.f32", "shl.b32 + add.u32 (lea)",
    "1 ex2.f32 + 1 fma.f32x2 (elements of both)", "1 ex2.f32 + 3 fma.f32x2 (elements of both)"};
// elements per instruction group of each test
static const double kElems[kNumOps] = {1, 2, 1, 2, 2, 2, 2, 1, 3, 7};

template <int OP>
__global__ void __launch_bounds__(kThreads, 1) bench(float seed, long long* cycles, float* sink) {
  float a[kChains], b[kChains];
  uint32_t u[kChains];
#pragma unroll
  for (int c = 0; c < kChains; ++c) {
    a[c] = seed * (threadIdx.x + c) * 1e-7f - 0.5f;
    b[c] = seed * (c + 1) * 1e-3f;
    u[c] = threadIdx.x * 7 + c;
  }
  __syncthreads();
  const long long t0 = clock64();
  for (int it = 0; it < kIters; ++it) {
#pragma unroll
    for (int c = 0; c < kChains; ++c) {
      if (OP == kEx2F32) {
        asm volatile("ex2.approx.ftz.f32 %0, %0;" : "+f"(a[c]));
      } else if (OP == kEx2Bf16x2) {
        asm volatile("ex2.approx.ftz.bf16x2 %0, %0;" : "+r"(u[c]));
      } else if (OP == kFfma) {
        asm volatile("fma.rn.f32 %0, %0, %1, %1;" : "+f"(a[c]) : "f"(b[c]));
      } else if (OP == kFfma2) {
        asm volatile("{\n .reg .b64 x, y;\n mov.b64 x, {%0, %1};\n mov.b64 y, {%2, %2};\n"
                     " fma.rn.f32x2 x, x, y, y;\n mov.b64 {%0, %1}, x;\n}"
                     : "+f"(a[c]), "+f"(b[c]) : "f"(seed));
      } else if (OP == kFadd2) {
        asm volatile("{\n .reg .b64 x, y;\n mov.b64 x, {%0, %1};\n mov.b64 y, {%2, %2};\n"
                     " add.rn.f32x2 x, x, y;\n mov.b64 {%0, %1}, x;\n}"
                     : "+f"(a[c]), "+f"(b[c]) : "f"(seed));
      } else if (OP == kMax3) {
        asm volatile("max.f32 %0, %0, %1, %2;" : "+f"(a[c]) : "f"(b[c]), "f"(seed));
      } else if (OP == kCvtBf16x2) {
        asm volatile("{\n cvt.rn.bf16x2.f32 %0, %1, %2;\n mov.b32 %1, %0;\n}" : "+r"(u[c]), "+f"(a[c]) : "f"(b[c]));
      } else if (OP == kLea) {
        asm volatile("{\n .reg .b32 t;\n shl.b32 t, %0, 23;\n add.u32 %0, t, %1;\n}" : "+r"(u[c]) : "r"(u[c ^ 1]));
      } else if (OP == kMixEx2Ffma2) {
        asm volatile("ex2.approx.ftz.f32 %0, %0;" : "+f"(a[c]));
        asm volatile("{\n .reg .b64 x, y;\n mov.b64 x, {%0, %1};\n mov.b64 y, {%2, %2};\n"
                     " fma.rn.f32x2 x, x, y, y;\n mov.b64 {%0, %1}, x;\n}"
                     : "+f"(b[c]), "+f"(b[c ^ 1]) : "f"(seed));
      } else if (OP == kMixEx2Ffma2x3) {
        asm volatile("ex2.approx.ftz.f32 %0, %0;" : "+f"(a[c]));
#pragma unroll
        for (int r = 0; r < 3; ++r)
          asm volatile("{\n .reg .b64 x, y;\n mov.b64 x, {%0, %1};\n mov.b64 y, {%2, %2};\n"
                       " fma.rn.f32x2 x, x, y, y;\n mov.b64 {%0, %1}, x;\n}"
                       : "+f"(b[c]), "+f"(b[c ^ 1]) : "f"(seed));
      }
    }
  }
  const long long t1 = clock64();
  float acc = 0.f;
#pragma unroll
  for (int c = 0; c < kChains; ++c) acc += a[c] + b[c] + (float)u[c];
  sink[blockIdx.x * kThreads + threadIdx.x] = acc;
  if (threadIdx.x == 0) cycles[blockIdx.x] = t1 - t0;
}

template <int OP>
int run(int sms, long long* d_cyc, float* d_sink, long long* h_cyc) {
  bench<OP><<<sms, kThreads>>>(1.0f, d_cyc, d_sink);
  CK(cudaGetLastError());
  CK(cudaDeviceSynchronize());
  bench<OP><<<sms, kThreads>>>(1.0f, d_cyc, d_sink);
  CK(cudaGetLastError());
  CK(cudaMemcpy(h_cyc, d_cyc, sizeof(long long) * sms, cudaMemcpyDeviceToHost));
  long long mx = 0;
  for (int i = 0; i < sms; ++i) mx = h_cyc[i] > mx ? h_cyc[i] : mx;
  const double groups = (double)kThreads * kIters * kChains;
  printf("%-44s %8.1f element ops / clk / SM\n", kNames[OP], groups * kElems[OP] / (double)mx);
  return 0;
}

int main() {
  int dev = 0, sms = 0;
  CK(cudaGetDevice(&dev));
  CK(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  cudaDeviceProp prop;
  CK(cudaGetDeviceProperties(&prop, dev));
  printf("# %s, %d SMs, %d threads per SM, %d independent chains per thread\n", prop.name, sms, kThreads,
         kChains);
  long long* d_cyc = nullptr;
  float* d_sink = nullptr;
  CK(cudaMalloc(&d_cyc, sizeof(long long) * sms));
  CK(cudaMalloc(&d_sink, sizeof(float) * sms * kThreads));
  long long* h_cyc = new long long[sms];
  int rc = 0;
  rc |= run<kEx2F32>(sms, d_cyc, d_sink, h_cyc);
  rc |= run<kEx2Bf16x2>(sms, d_cyc, d_sink, h_cyc);
  rc |= run<kFfma>(sms, d_cyc, d_sink, h_cyc);
  rc |= run<kFfma2>(sms, d_cyc, d_sink, h_cyc);
  rc |= run<kFadd2>(sms, d_cyc, d_sink, h_cyc);
  rc |= run<kMax3>(sms, d_cyc, d_sink, h_cyc);
  rc |= run<kCvtBf16x2>(sms, d_cyc, d_sink, h_cyc);
  rc |= run<kLea>(sms, d_cyc, d_sink, h_cyc);
  rc |= run<kMixEx2Ffma2>(sms, d_cyc, d_sink, h_cyc);
  rc |= run<kMixEx2Ffma2x3>(sms, d_cyc, d_sink, h_cyc);
  delete[] h_cyc;
  CK(cudaFree(d_cyc));
  CK(cudaFree(d_sink));
  return rc;
}
