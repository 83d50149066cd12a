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
};

// Launchers (one per translation unit).
swin_status launch_cpb_eval(int M, int heads, const swin_cpb_weights& g, float* table,
                            cudaStream_t stream, int form = SWIN_CPB_PAPER, int pretrained_M = 0);
swin_status launch_index_tables(int H, int W, int M, int shift, int32_t* tw, int32_t* tr,
                                int32_t* tl, int32_t* ri, cudaStream_t stream);
swin_status launch_attn_tc(const AttnArgs& a, bool f32_out, cudaStream_t stream);
void tc_set_debug(int flags, long long wait_limit);
swin_status launch_attn_simt(const AttnArgs& a, bool bf16_in, bool f32_out, cudaStream_t stream);
swin_status launch_attn_bwd(const BwdArgs& a, bool bf16_in, bool f32_grad, float* dtable, float* dtau,
                            float* drope, cudaStream_t stream);

}  // namespace swin
