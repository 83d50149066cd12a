// Host side of the C ABI declared in include/swin_attn.h: argument checks,
// workspace layout, kernel selection and the device status word.
#include <cstdarg>
#include <cstdio>
#include <mutex>
#include <string>

#include "swin_common.cuh"

namespace swin {

namespace {
thread_local std::string g_last_error;

// One status word per device; kernels OR error codes into it, never trap.  Its
// address is cached per device ordinal for the life of the process: the
// library must not be used across a cudaDeviceReset.
__device__ int g_status_word;

constexpr int kMaxDevices = 64;
int* g_status_ptr[kMaxDevices] = {};
std::mutex g_status_mu;

}  // namespace

swin_status fail(swin_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

int* status_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_status_mu);
  if (!g_status_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return nullptr;
    g_status_ptr[dev] = static_cast<int*>(p);
  }
  return g_status_ptr[dev];
}

}  // namespace swin

using swin::fail;

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static bool overlaps(const void* a, size_t an, const void* b, size_t bn) {
  uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
  return a0 < b0 + bn && b0 < a0 + an;
}

namespace swin {

swin_status check_fwd_args(const void* q, const void* k, const void* v, const void* out, swin_dtype dt,
                           swin_dtype out_dt, int B, int H, int W, int heads, int d, int M, int shift,
                           swin_mode mode, const float* tau, const float* bias_table,
                           const swin_cpb_weights* cpb, const float* rope_freqs) {
  if (!q || !k || !v || !out) return fail(SWIN_ERR_INVALID_ARG, "q, k, v and out must be non-NULL");
  if (dt != SWIN_F32 && dt != SWIN_BF16) return fail(SWIN_ERR_INVALID_ARG, "unknown dtype %d", (int)dt);
  if (out_dt != dt && !(dt == SWIN_BF16 && out_dt == SWIN_F32))
    return fail(SWIN_ERR_INVALID_ARG, "output dtype %d not allowed for input dtype %d", (int)out_dt, (int)dt);
  if (B < 1 || H < 1 || W < 1 || heads < 1 || d < 1)
    return fail(SWIN_ERR_INVALID_ARG, "B, H, W, heads and d must be >= 1");
  if (M < 1 || M > 64) return fail(SWIN_ERR_INVALID_ARG, "M=%d outside [1, 64]", M);
  if (shift < 0 || shift >= M) return fail(SWIN_ERR_INVALID_ARG, "shift=%d outside [0, M)", shift);
  if (mode != SWIN_MODE_DOT_BIAS && mode != SWIN_MODE_COSINE_CPB && mode != SWIN_MODE_ROPE)
    return fail(SWIN_ERR_INVALID_ARG, "unknown mode %d", (int)mode);
  const long long elems = (long long)B * H * W * heads * d;
  if (elems >= (1ll << 31)) return fail(SWIN_ERR_UNSUPPORTED, "B*H*W*heads*d must be < 2^31");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
    return fail(SWIN_ERR_INVALID_ARG, "q, k, v and out must be 16-byte aligned");
  const size_t bytes = (size_t)elems * (dt == SWIN_F32 ? 4 : 2);
  const size_t obytes = (size_t)elems * (out_dt == SWIN_F32 ? 4 : 2);
  if (overlaps(out, obytes, q, bytes) || overlaps(out, obytes, k, bytes) || overlaps(out, obytes, v, bytes))
    return fail(SWIN_ERR_INVALID_ARG, "out overlaps q, k or v");
  if (mode == SWIN_MODE_COSINE_CPB && !tau) return fail(SWIN_ERR_INVALID_ARG, "cosine mode needs tau");
  if (mode == SWIN_MODE_ROPE) {
    if (!rope_freqs) return fail(SWIN_ERR_INVALID_ARG, "RoPE mode needs rope_freqs");
    if (d % 4 != 0) return fail(SWIN_ERR_INVALID_ARG, "RoPE mode needs d %% 4 == 0, got %d", d);
    if (bias_table) return fail(SWIN_ERR_INVALID_ARG, "RoPE mode takes no bias table");
  }
  if (cpb && (cpb->hidden < 1 || cpb->hidden > 4096 || !cpb->w1 || !cpb->w2))
    return fail(SWIN_ERR_INVALID_ARG, "cpb weights incomplete or hidden outside [1, 4096]");
  if (heads > 64 && mode == SWIN_MODE_COSINE_CPB && !bias_table && cpb)
    return fail(SWIN_ERR_INVALID_ARG, "cpb evaluation supports heads <= 64");
  return SWIN_OK;
}

}  // namespace swin

extern "C" {

const char* swin_last_error(void) { return swin::g_last_error.c_str(); }

int swin_version(void) { return 100; }

swin_status swin_cpb_eval(int M, int heads, const swin_cpb_weights* g, float* table_out,
                          swin_stream_t stream) {
  return swin_cpb_eval_form(M, heads, g, SWIN_CPB_PAPER, 0, table_out, stream);
}

swin_status swin_cpb_eval_form(int M, int heads, const swin_cpb_weights* g, swin_cpb_form form,
                               int pretrained_M, float* table_out, swin_stream_t stream) {
  if (form != SWIN_CPB_PAPER && form != SWIN_CPB_CODE) return fail(SWIN_ERR_INVALID_ARG, "form=%d", (int)form);
  if (pretrained_M < 0 || pretrained_M > 64)
    return fail(SWIN_ERR_INVALID_ARG, "pretrained_M=%d outside [0, 64]", pretrained_M);
  if (form == SWIN_CPB_PAPER && pretrained_M != 0)
    return fail(SWIN_ERR_INVALID_ARG, "pretrained_M applies to SWIN_CPB_CODE only");
  if (M < 1 || M > 64) return fail(SWIN_ERR_INVALID_ARG, "M=%d outside [1, 64]", M);
  if (heads < 1 || heads > 64) return fail(SWIN_ERR_INVALID_ARG, "heads=%d outside [1, 64]", heads);
  if (!g) return fail(SWIN_ERR_INVALID_ARG, "cpb weights struct is NULL");
  if (g->hidden < 1 || g->hidden > 4096)
    return fail(SWIN_ERR_INVALID_ARG, "hidden=%d outside [1, 4096]", g->hidden);
  if (!g->w1 || !g->w2 || !table_out)
    return fail(SWIN_ERR_INVALID_ARG, "w1, w2 and table_out must be non-NULL");
  return swin::launch_cpb_eval(M, heads, *g, table_out, reinterpret_cast<cudaStream_t>(stream), (int)form,
                               pretrained_M);
}

size_t swin_window_attn_workspace_size(int M, int heads, swin_mode mode, int have_table) {
  if (mode != SWIN_MODE_COSINE_CPB || have_table || M < 1 || heads < 1) return 0;
  size_t bytes = sizeof(float) * (size_t)(2 * M - 1) * (2 * M - 1) * heads;
  return (bytes + 255) & ~size_t(255);
}

swin_status swin_window_attn_fwd(const void* q, const void* k, const void* v, void* out,
                                 swin_dtype dt, swin_dtype out_dt, int B, int H, int W, int heads,
                                 int d, int M,
                                 int shift, swin_mode mode, const float* tau,
                                 const float* bias_table, const swin_cpb_weights* cpb,
                                 const float* rope_freqs, void* workspace,
                                 size_t workspace_bytes, swin_stream_t stream) {
  return swin_window_attn_fwd_ex(q, k, v, out, dt, out_dt, B, H, W, heads, d, M, shift, SWIN_PARTITION_SHIFTED,
                                 mode, tau, bias_table, cpb, rope_freqs, workspace, workspace_bytes, stream);
}

static swin_status check_partition(swin_partition partition, int shift) {
  if (partition != SWIN_PARTITION_SHIFTED && partition != SWIN_PARTITION_INTERLEAVED)
    return fail(SWIN_ERR_INVALID_ARG, "unknown partition %d", (int)partition);
  if (partition == SWIN_PARTITION_INTERLEAVED && shift != 0)
    return fail(SWIN_ERR_INVALID_ARG, "interleaved windows take no shift (got %d)", shift);
  return SWIN_OK;
}

swin_status swin_window_attn_fwd_ex(const void* q, const void* k, const void* v, void* out, swin_dtype dt,
                                    swin_dtype out_dt, int B, int H, int W, int heads, int d, int M, int shift,
                                    swin_partition partition, swin_mode mode, const float* tau,
                                    const float* bias_table, const swin_cpb_weights* cpb, const float* rope_freqs,
                                    void* workspace, size_t workspace_bytes, swin_stream_t stream) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  swin_status vs = swin::check_fwd_args(q, k, v, out, dt, out_dt, B, H, W, heads, d, M, shift, mode, tau,
                                        bias_table, cpb, rope_freqs);
  if (vs != SWIN_OK) return vs;
  vs = check_partition(partition, shift);
  if (vs != SWIN_OK) return vs;

  const float* table = bias_table;
  if (mode == SWIN_MODE_COSINE_CPB && !bias_table && cpb) {
    size_t need = swin_window_attn_workspace_size(M, heads, mode, 0);
    if (!workspace || workspace_bytes < need)
      return fail(SWIN_ERR_INVALID_ARG, "workspace of %zu bytes needed, got %zu", need, workspace_bytes);
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
      return fail(SWIN_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    float* ws_table = static_cast<float*>(workspace);
    swin_status s = swin::launch_cpb_eval(M, heads, *cpb, ws_table, st);
    if (s != SWIN_OK) return s;
    table = ws_table;
  }
  if (mode == SWIN_MODE_ROPE) table = nullptr;

  swin::AttnArgs a;
  a.q = q; a.k = k; a.v = v; a.out = out;
  a.B = B; a.H = H; a.W = W; a.heads = heads; a.d = d; a.M = M; a.shift = shift; a.mode = (int)mode;
  a.part = (int)partition;
  a.tau = tau; a.table = table; a.rope = rope_freqs;
  a.status = swin::status_word();
  if (!a.status) return fail(SWIN_ERR_CUDA, "could not resolve the device status word");
  // tensor cores, bf16 and d = 32.  Interleaved windows, and windows of at most
  // 64 tokens (M <= 8: one query tile and one key block each, where the
  // rectangle kernel measured faster, 0.134 against 0.145 ms on Swin-T stage 1),
  // take the kernel over row-loaded rectangles; other shifted windows the TMA
  // kernel, whose bias-table slot holds M <= 32.
  if (dt == SWIN_BF16 && d == 32 && M <= 32 && (partition == SWIN_PARTITION_INTERLEAVED || M <= 8))
    return swin::launch_attn_fwd_tc_rect(a, out_dt == SWIN_F32, st);
  if (dt == SWIN_BF16 && d == 32 && partition == SWIN_PARTITION_SHIFTED && (table == nullptr || M <= 32))
    return swin::launch_attn_tc(a, out_dt == SWIN_F32, st);
  return swin::launch_attn_simt(a, dt == SWIN_BF16, out_dt == SWIN_F32, st);
}

static size_t bwd_acc_doubles(int heads, int d, int M) {
  return (size_t)(2 * M - 1) * (2 * M - 1) * heads + (size_t)heads + 2 * (size_t)(d / 4);
}

size_t swin_window_attn_bwd_workspace_size(int B, int H, int W, int heads, int d, int M) {
  if (B < 1 || H < 1 || W < 1 || heads < 1 || d < 1 || M < 1 || M > 64) return 0;
  const size_t acc = (sizeof(double) * bwd_acc_doubles(heads, d, M) + 255) & ~size_t(255);
  const size_t stats = sizeof(double) * 2 * (size_t)B * H * W * heads;
  return acc + ((stats + 255) & ~size_t(255));
}

swin_status swin_window_attn_bwd(const void* q, const void* k, const void* v, const void* dout, void* dq,
                                 void* dk, void* dv, swin_dtype dt, swin_dtype grad_dt, int B, int H, int W,
                                 int heads, int d, int M, int shift, swin_partition partition, swin_mode mode,
                                 const float* tau,
                                 const float* bias_table, const float* rope_freqs, float* dtable, float* dtau,
                                 float* drope, void* workspace, size_t workspace_bytes, swin_stream_t stream) {
  // the forward's checks with dq standing for out (dtype, shape, alignment,
  // mode parameters, dq against q, k, v)
  swin_status vs = swin::check_fwd_args(q, k, v, dq, dt, grad_dt, B, H, W, heads, d, M, shift, mode, tau,
                                        bias_table, nullptr, rope_freqs);
  if (vs != SWIN_OK) return vs;
  vs = check_partition(partition, shift);
  if (vs != SWIN_OK) return vs;
  if (!dout || !dk || !dv) return fail(SWIN_ERR_INVALID_ARG, "dout, dk and dv must be non-NULL");
  if (!aligned16(dout) || !aligned16(dk) || !aligned16(dv))
    return fail(SWIN_ERR_INVALID_ARG, "dout, dk and dv must be 16-byte aligned");
  if (d != 8 && d != 16 && d != 32 && d != 64)
    return fail(SWIN_ERR_UNSUPPORTED, "backward supports d in {8,16,32,64}, got %d", d);
  const size_t elems = (size_t)B * H * W * heads * d;
  const size_t ib = elems * (dt == SWIN_F32 ? 4 : 2), gb = elems * (grad_dt == SWIN_F32 ? 4 : 2);
  const void* ins[4] = {q, k, v, dout};
  void* outs[3] = {dq, dk, dv};
  for (int o = 0; o < 3; ++o) {
    for (int i = 0; i < 4; ++i)
      if (overlaps(outs[o], gb, ins[i], ib)) return fail(SWIN_ERR_INVALID_ARG, "dq, dk and dv must not overlap the inputs");
    for (int p = o + 1; p < 3; ++p)
      if (overlaps(outs[o], gb, outs[p], gb)) return fail(SWIN_ERR_INVALID_ARG, "dq, dk and dv must not overlap");
  }
  if (dtable && !bias_table) return fail(SWIN_ERR_INVALID_ARG, "dtable needs bias_table");
  if (dtau && mode != SWIN_MODE_COSINE_CPB) return fail(SWIN_ERR_INVALID_ARG, "dtau applies to the cosine mode only");
  if (drope && mode != SWIN_MODE_ROPE) return fail(SWIN_ERR_INVALID_ARG, "drope applies to the RoPE mode only");
  const size_t need = swin_window_attn_bwd_workspace_size(B, H, W, heads, d, M);
  if (!workspace || workspace_bytes < need)
    return fail(SWIN_ERR_INVALID_ARG, "workspace of %zu bytes needed, got %zu", need, workspace_bytes);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(SWIN_ERR_INVALID_ARG, "workspace must be 256-byte aligned");

  double* acc = static_cast<double*>(workspace);
  const size_t acc_bytes = (sizeof(double) * bwd_acc_doubles(heads, d, M) + 255) & ~size_t(255);
  swin::BwdArgs a;
  a.q = q; a.k = k; a.v = v; a.dout = dout; a.dq = dq; a.dk = dk; a.dv = dv;
  a.B = B; a.H = H; a.W = W; a.heads = heads; a.d = d; a.M = M; a.shift = shift; a.mode = (int)mode;
  a.part = (int)partition;
  a.tau = tau; a.table = mode == SWIN_MODE_ROPE ? nullptr : bias_table; a.rope = rope_freqs;
  size_t slot = 0;
  a.acc_base = acc;
  a.acc_table = dtable ? acc + slot : nullptr;
  slot += dtable ? (size_t)(2 * M - 1) * (2 * M - 1) * heads : 0;
  a.acc_tau = dtau ? acc + slot : nullptr;
  slot += dtau ? (size_t)heads : 0;
  a.acc_rope = drope ? acc + slot : nullptr;
  a.stats = reinterpret_cast<double2*>(static_cast<char*>(workspace) + acc_bytes);
  a.status = swin::status_word();
  if (!a.status) return fail(SWIN_ERR_CUDA, "could not resolve the device status word");
  return swin::launch_attn_bwd(a, dt == SWIN_BF16, grad_dt == SWIN_F32, dtable, dtau, drope,
                               reinterpret_cast<cudaStream_t>(stream));
}

static swin_status check_proj(const void* const* ptrs, int n, swin_dtype dt, swin_dtype out_dt, int tokens, int C) {
  for (int i = 0; i < n; ++i)
    if (!ptrs[i]) return fail(SWIN_ERR_INVALID_ARG, "tensor arguments must be non-NULL");
  for (int i = 0; i < n; ++i)
    if (!aligned16(ptrs[i])) return fail(SWIN_ERR_INVALID_ARG, "tensor arguments must be 16-byte aligned");
  if (dt != SWIN_F32 && dt != SWIN_BF16) return fail(SWIN_ERR_INVALID_ARG, "unknown dtype %d", (int)dt);
  if (out_dt != dt && !(dt == SWIN_BF16 && out_dt == SWIN_F32))
    return fail(SWIN_ERR_INVALID_ARG, "output dtype %d not allowed for input dtype %d", (int)out_dt, (int)dt);
  if (tokens < 1 || C < 1) return fail(SWIN_ERR_INVALID_ARG, "tokens and C must be >= 1");
  if ((long long)tokens * C * 3 >= (1ll << 31)) return fail(SWIN_ERR_UNSUPPORTED, "tokens*3C must be < 2^31");
  if (C % 8 != 0) return fail(SWIN_ERR_INVALID_ARG, "C must be a multiple of 8 (16-byte rows), got %d", C);
  return SWIN_OK;
}

static size_t align256(size_t n) { return (n + 255) & ~size_t(255); }

static swin_status check_ws(void* ws, size_t have, size_t need) {
  if (!ws || have < need) return fail(SWIN_ERR_INVALID_ARG, "workspace of %zu bytes needed, got %zu", need, have);
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return fail(SWIN_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  return SWIN_OK;
}

size_t swin_qkv_proj_workspace_size(int tokens, int C) {
  if (tokens < 1 || C < 1) return 0;
  return align256(sizeof(float) * (size_t)tokens * 3 * C);
}

size_t swin_proj_postnorm_workspace_size(int tokens, int C) {
  if (tokens < 1 || C < 1) return 0;
  return align256(sizeof(float) * (size_t)tokens * C);
}

swin_status swin_qkv_proj(const void* x, const void* w_qkv, const float* b_qkv, void* q, void* k, void* v,
                          swin_dtype dt, swin_dtype out_dt, int tokens, int C, void* workspace,
                          size_t workspace_bytes, swin_stream_t stream) {
  const void* ptrs[5] = {x, w_qkv, q, k, v};
  swin_status vs = check_proj(ptrs, 5, dt, out_dt, tokens, C);
  if (vs != SWIN_OK) return vs;
  const size_t need = swin_qkv_proj_workspace_size(tokens, C);
  if ((vs = check_ws(workspace, workspace_bytes, need)) != SWIN_OK) return vs;
  const size_t xb = (size_t)tokens * C * (dt == SWIN_F32 ? 4 : 2), ob = (size_t)tokens * C * (out_dt == SWIN_F32 ? 4 : 2);
  const void* outs[3] = {q, k, v};
  for (int i = 0; i < 3; ++i) {
    if (overlaps(outs[i], ob, x, xb) || overlaps(outs[i], ob, workspace, need))
      return fail(SWIN_ERR_INVALID_ARG, "q, k and v must not overlap x or the workspace");
    for (int j = i + 1; j < 3; ++j)
      if (overlaps(outs[i], ob, outs[j], ob)) return fail(SWIN_ERR_INVALID_ARG, "q, k and v must not overlap");
  }
  return swin::launch_qkv_proj(x, w_qkv, b_qkv, q, k, v, dt == SWIN_BF16, out_dt == SWIN_F32, tokens, C,
                               static_cast<float*>(workspace), reinterpret_cast<cudaStream_t>(stream));
}

swin_status swin_proj_postnorm_residual(const void* a, const void* w_o, const float* b_o, const void* x,
                                        const float* gamma, const float* beta, float eps, void* out, swin_dtype dt,
                                        swin_dtype out_dt, int tokens, int C, void* workspace, size_t workspace_bytes,
                                        swin_stream_t stream) {
  const void* ptrs[4] = {a, w_o, x, out};
  swin_status vs = check_proj(ptrs, 4, dt, out_dt, tokens, C);
  if (vs != SWIN_OK) return vs;
  if (!(eps > 0.0f)) return fail(SWIN_ERR_INVALID_ARG, "eps must be > 0");
  if (C > 1024) return fail(SWIN_ERR_UNSUPPORTED, "post-norm supports C <= 1024, got %d", C);
  const size_t need = swin_proj_postnorm_workspace_size(tokens, C);
  if ((vs = check_ws(workspace, workspace_bytes, need)) != SWIN_OK) return vs;
  const size_t xb = (size_t)tokens * C * (dt == SWIN_F32 ? 4 : 2), ob = (size_t)tokens * C * (out_dt == SWIN_F32 ? 4 : 2);
  if (overlaps(out, ob, x, xb) || overlaps(out, ob, a, xb) || overlaps(out, ob, workspace, need))
    return fail(SWIN_ERR_INVALID_ARG, "out must not overlap x, a or the workspace");
  return swin::launch_proj_postnorm(a, w_o, b_o, x, gamma, beta, eps, out, dt == SWIN_BF16, out_dt == SWIN_F32,
                                    tokens, C, static_cast<float*>(workspace), reinterpret_cast<cudaStream_t>(stream));
}

size_t swin_attn_block_workspace_size(int B, int H, int W, int heads, int d, int M, swin_mode mode, int have_table,
                                      swin_dtype dt) {
  if (B < 1 || H < 1 || W < 1 || heads < 1 || d < 1) return 0;
  const size_t tokens = (size_t)B * H * W, C = (size_t)heads * d;
  const size_t tb = align256(tokens * C * (dt == SWIN_F32 ? 4 : 2));
  return 4 * tb + align256(sizeof(float) * tokens * 3 * C) + swin_window_attn_workspace_size(M, heads, mode, have_table);
}

swin_status swin_attn_block_fwd(const void* x, const void* w_qkv, const float* b_qkv, const void* w_o,
                                const float* b_o, const float* gamma, const float* beta, float eps, void* out,
                                swin_dtype dt, swin_dtype out_dt, int B, int H, int W, int heads, int d, int M,
                                int shift, swin_partition partition, swin_mode mode, const float* tau,
                                const float* bias_table, const swin_cpb_weights* cpb, const float* rope_freqs,
                                void* workspace, size_t workspace_bytes, swin_stream_t stream) {
  if (B < 1 || H < 1 || W < 1 || heads < 1 || d < 1) return fail(SWIN_ERR_INVALID_ARG, "B, H, W, heads and d must be >= 1");
  const long long tokens = (long long)B * H * W;
  if (tokens >= (1ll << 31)) return fail(SWIN_ERR_UNSUPPORTED, "B*H*W must be < 2^31");
  const int C = heads * d;
  const void* ptrs[4] = {x, w_qkv, w_o, out};
  swin_status st = check_proj(ptrs, 4, dt, out_dt, (int)tokens, C);
  if (st != SWIN_OK) return st;
  const size_t need = swin_attn_block_workspace_size(B, H, W, heads, d, M, mode, bias_table != nullptr, dt);
  if ((st = check_ws(workspace, workspace_bytes, need)) != SWIN_OK) return st;
  const size_t tb = align256((size_t)tokens * C * (dt == SWIN_F32 ? 4 : 2));
  const size_t yb = align256(sizeof(float) * (size_t)tokens * 3 * C);
  const size_t ob = (size_t)tokens * C * (out_dt == SWIN_F32 ? 4 : 2);
  char* ws = static_cast<char*>(workspace);
  void *q = ws, *k = ws + tb, *v = ws + 2 * tb, *att = ws + 3 * tb;
  float* y = reinterpret_cast<float*>(ws + 4 * tb);
  if (overlaps(out, ob, x, (size_t)tokens * C * (dt == SWIN_F32 ? 4 : 2)))
    return fail(SWIN_ERR_INVALID_ARG, "out must not overlap x");
  if (overlaps(out, ob, workspace, need) || overlaps(x, tb, workspace, need))
    return fail(SWIN_ERR_INVALID_ARG, "x and out must not overlap the workspace");
  // every attention argument is checked before the first launch
  st = swin::check_fwd_args(q, k, v, att, dt, dt, B, H, W, heads, d, M, shift, mode, tau, bias_table, cpb,
                            rope_freqs);
  if (st != SWIN_OK) return st;
  st = check_partition(partition, shift);
  if (st != SWIN_OK) return st;
  if (!(eps > 0.0f)) return fail(SWIN_ERR_INVALID_ARG, "eps must be > 0");
  if (C > 1024) return fail(SWIN_ERR_UNSUPPORTED, "post-norm supports C <= 1024, got %d", C);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  st = swin::launch_qkv_proj(x, w_qkv, b_qkv, q, k, v, dt == SWIN_BF16, false, (int)tokens, C, y, s);
  if (st != SWIN_OK) return st;
  st = swin_window_attn_fwd_ex(q, k, v, att, dt, dt, B, H, W, heads, d, M, shift, partition, mode, tau, bias_table,
                               cpb, rope_freqs, ws + 4 * tb + yb, workspace_bytes - 4 * tb - yb, stream);
  if (st != SWIN_OK) return st;
  return swin::launch_proj_postnorm(att, w_o, b_o, x, gamma, beta, eps, out, dt == SWIN_BF16, out_dt == SWIN_F32,
                                    (int)tokens, C, y, s);
}

swin_status swin_index_tables(int H, int W, int M, int shift, int32_t* tok_window,
                              int32_t* tok_region, int32_t* tok_local, int32_t* rel_index,
                              swin_stream_t stream) {
  if (H < 1 || W < 1) return fail(SWIN_ERR_INVALID_ARG, "H and W must be >= 1");
  if (M < 1 || M > 64) return fail(SWIN_ERR_INVALID_ARG, "M=%d outside [1, 64]", M);
  if (shift < 0 || shift >= M) return fail(SWIN_ERR_INVALID_ARG, "shift=%d outside [0, M)", shift);
  if ((long long)H * W >= (1ll << 31)) return fail(SWIN_ERR_UNSUPPORTED, "H*W must be < 2^31");
  return swin::launch_index_tables(H, W, M, shift, tok_window, tok_region, tok_local, rel_index,
                                   reinterpret_cast<cudaStream_t>(stream));
}

swin_status swin_debug_set(int flags, long long wait_limit_cycles) {
  if (flags & ~1) return fail(SWIN_ERR_INVALID_ARG, "unknown debug flags 0x%x", flags);
  swin::tc_set_debug(flags, wait_limit_cycles);
  return SWIN_OK;
}

swin_status swin_stream_status(swin_stream_t stream) {
  cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(SWIN_ERR_CUDA, "stream synchronize: %s", cudaGetErrorString(e));
  int* w = swin::status_word();
  if (!w) return fail(SWIN_ERR_CUDA, "could not resolve the device status word");
  int val = 0, zero = 0;
  if (cudaMemcpy(&val, w, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess ||
      cudaMemcpy(w, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
    return fail(SWIN_ERR_CUDA, "reading the device status word failed");
  if (val & swin::kStatusRangeCheck)
    return fail(SWIN_ERR_CUDA, "a range check of the SWIN_DEBUG build failed (an index outside its buffer; "
                               "the access was skipped)");
  if (val & SWIN_ERR_TIMEOUT) return fail(SWIN_ERR_TIMEOUT, "a kernel's bounded wait ran out");
  if (val & SWIN_ERR_UNSUPPORTED)
    return fail(SWIN_ERR_UNSUPPORTED, "an operand left the fp16 range on the tensor-core path (a RoPE-rotated k or a V entry of magnitude >= 65504)");
  if (val != 0) return fail(SWIN_ERR_CUDA, "unknown device status %d", val);
  return SWIN_OK;
}

}  // extern "C"
