// Shared declarations of libswinattn's translation units (not part of the ABI).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

#include "../../include/swin_attn.h"
#include "swin_index.cuh"

namespace swin {

// Records a failure message for swin_last_error() and returns st.
swin_status fail(swin_status st, const char* fmt, ...);

// Device address of this device's status word (set up once per device).
int* status_word();

// Every argument check of swin_window_attn_fwd that does not depend on the
// workspace; SWIN_OK or the failure (message recorded), nothing launched.
swin_status check_fwd_args(const void* q, const void* k, const void* v, const void* out, swin_dtype dt,
                           swin_dtype out_dt, int B, int H, int W, int heads, int d, int M, int shift,
                           swin_mode mode, const float* tau, const float* bias_table,
                           const swin_cpb_weights* cpb, const float* rope_freqs);

// Status bit a SWIN_DEBUG build's kernels OR into the status word when an
// index check fails (the access is then skipped where skipping is safe);
// swin_stream_status reports it.  Release builds compile the checks away.
constexpr int kStatusRangeCheck = 0x100;
#ifdef SWIN_DEBUG
#define SWIN_DCHECK(status_ptr, cond)                                  \
  do {                                                                 \
    if (!(cond)) atomicOr((status_ptr), ::swin::kStatusRangeCheck);    \
  } while (0)
#define SWIN_DEBUG_BUILD 1
#else
#define SWIN_DCHECK(status_ptr, cond) \
  do {                                \
  } while (0)
#define SWIN_DEBUG_BUILD 0
#endif

// fp32 RoPE tables are built in the kernels from the caller's frequencies.
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kTauMin = 0.01f;
constexpr float kNormEps = 1e-12f;

struct AttnArgs {
  const void* q;
  const void* k;
  const void* v;
  void* out;
  int B, H, W, heads, d, M, shift, mode;
  int part;  // SwinPartition (the tensor-core path takes kPartShifted only)
  const float* tau;
  const float* table;  // [(2M-1)^2][heads] or nullptr
  const float* rope;   // [2][d/4] or nullptr
  int* status;
};

// Arguments of the backward kernels.  The double accumulators of the
// parameter gradients lie contiguously at acc_base: table, then tau, then
// rope; a gradient not asked for has a NULL pointer and no slot.
struct BwdArgs {
  const void* q;
  const void* k;
  const void* v;
  const void* dout;
  void* dq;
  void* dk;
  void* dv;
  int B, H, W, heads, d, M, shift, mode;
  int part;  // SwinPartition
  const float* tau;
  const float* table;  // [(2M-1)^2][heads] or nullptr
  const float* rope;   // [2][d/4] or nullptr
  double* acc_base;
  double* acc_table;
  double* acc_tau;
  double* acc_rope;
  double2* stats;  // [B][H][W][heads]: (log-sum-exp, D) of each query row
  int* status;     // device status word (range checks of a SWIN_DEBUG build)
};

// Launchers (one per translation unit).
swin_status launch_cpb_eval(int M, int heads, const swin_cpb_weights& g, float* table,
                            cudaStream_t stream, int form = SWIN_CPB_PAPER, int pretrained_M = 0);
swin_status launch_index_tables(int H, int W, int M, int shift, int32_t* tw, int32_t* tr,
                                int32_t* tl, int32_t* ri, cudaStream_t stream);
swin_status launch_attn_tc(const AttnArgs& a, bool f32_out, cudaStream_t stream);
void tc_set_debug(int flags, long long wait_limit);
swin_status launch_attn_simt(const AttnArgs& a, bool bf16_in, bool f32_out, cudaStream_t stream);
// y: fp32 scratch of tokens x 3C (qkv) or tokens x C (post-norm) floats.
swin_status launch_qkv_proj(const void* x, const void* w_qkv, const float* b_qkv, void* q, void* k, void* v,
                            bool bf16, bool f32_out, int tokens, int C, float* y, cudaStream_t stream);
swin_status launch_proj_postnorm(const void* a, const void* w_o, const float* b_o, const void* x,
                                 const float* gamma, const float* beta, float eps, void* out, bool bf16, bool f32_out,
                                 int tokens, int C, float* y, cudaStream_t stream);
swin_status launch_attn_bwd(const BwdArgs& a, bool bf16_in, bool f32_grad, float* dtable, float* dtau,
                            float* drope, cudaStream_t stream);
// The tensor-core backward (bf16, d = 32, M <= 32): dq, dk, dv and the
// parameter-gradient accumulators, with the statistics in a.stats.
bool attn_bwd_tc_supported(const BwdArgs& a, bool bf16_in);
// The tensor-core forward over arbitrary rectangles (bf16, d = 32, M <= 32),
// used for the interleaved partition.
swin_status launch_attn_fwd_tc_rect(const AttnArgs& a, bool f32_out, cudaStream_t stream);
// Fused tensor-core block steps (k_block_tc.cu): bf16 inputs, C % 32 == 0,
// C <= 128, weights and tiles within shared memory.
bool block_tc_supported(int C, bool bf16_in, bool postnorm);
swin_status launch_qkv_proj_tc(const void* x, const void* w_qkv, const float* b_qkv, void* q, void* k, void* v,
                               bool f32_out, int tokens, int C, cudaStream_t stream);
swin_status launch_proj_postnorm_tc(const void* a, const void* w_o, const float* b_o, const void* x,
                                    const float* gamma, const float* beta, float eps, void* out, bool f32_out,
                                    int tokens, int C, cudaStream_t stream);
swin_status launch_attn_bwd_tc(const BwdArgs& a, bool f32_grad, cudaStream_t stream);

}  // namespace swin
