/*
 * swin_attn.h — C ABI of libswinattn.so: shifted-window multi-head
 * self-attention (forward and gradients) on a 2-D token grid, for NVIDIA
 * B200 (sm_100a).
 *
 * What is computed.  For an image b, head h and query token i at grid
 * position (y_i, x_i), the attended keys are the tokens j that share i's
 * segment on both axes, where each axis of length L is cut at s + kM
 * (k integer) and clipped to [0, L).  This is the attention that Swin's
 * cyclic shift by s, MxM window partition and region mask give; here the
 * shift and partition are index arithmetic, nothing is rolled or copied.
 * Padding never exists: a grid side that M does not divide ends in a shorter
 * segment.  The score of a pair (i, j) is
 *   SWIN_MODE_DOT_BIAS   q.k / sqrt(d) + T[r(i,j)][h]
 *        "Swin Transformer V2: Scaling Up Capacity and Resolution", eq. 1;
 *   SWIN_MODE_COSINE_CPB cos(q, k) / max(tau_h, 0.01) + T[r(i,j)][h]
 *        same page, §3.2 / eq. 2 and the window_attention pseudocode; T is
 *        either given or produced by the Log-CPB meta network G of §3.3
 *        (eq. 3, eq. 4), see swin_cpb_eval;
 *   SWIN_MODE_ROPE       (R(p_i) q).(R(p_j) k) / sqrt(d), no bias
 *        "FLASHSWIN ..." abstract: window-local learnable 2-D RoPE with exact
 *        softmax attention and no materialised score matrix.
 * followed by a softmax over the attended keys and a weighted sum of v.
 * r(i,j) = (dy + M - 1) * (2M - 1) + (dx + M - 1) with (dy, dx) = query
 * position minus key position.  RoPE: channels [0, d/2) rotate pairs
 * (2t, 2t+1) by p_y * w[0][t], channels [d/2, d) by p_x * w[1][t], t < d/4,
 * with window-local coordinates p = (coordinate - s) mod M.
 *
 * Memory.  Every tensor pointer is DEVICE memory owned by the caller.  Q, K,
 * V and O are dense row-major [B][H][W][heads][d] (channel fastest), Q, K, V
 * of one dtype (fp32 or bf16), O of the same dtype or fp32; 16-byte aligned;
 * O must not overlap Q, K or V.
 * The library allocates no device memory for a call; scratch comes from the
 * caller's workspace (size from swin_window_attn_workspace_size).
 *
 * Streams and errors.  Calls are asynchronous on the given stream (NULL =
 * legacy default stream) and return after enqueueing.  Argument errors return
 * SWIN_ERR_INVALID_ARG or SWIN_ERR_UNSUPPORTED without launching anything;
 * launch failures return SWIN_ERR_CUDA.  Kernels never trap: a bounded wait
 * that runs out records SWIN_ERR_TIMEOUT in a device status word, which
 * swin_stream_status reads (after synchronising the stream) and clears.
 * swin_last_error returns a message for the last failure on this host thread.
 * The library caches device addresses of its own variables per device, so it
 * must not be used across a cudaDeviceReset.
 */
#ifndef SWIN_ATTN_H
#define SWIN_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Binary-compatible with cudaStream_t / CUstream. */
typedef struct CUstream_st* swin_stream_t;

typedef enum {
  SWIN_OK = 0,
  SWIN_ERR_INVALID_ARG = 1, /* bad shape, pointer, alignment or value */
  SWIN_ERR_UNSUPPORTED = 2, /* valid, but outside what the kernels cover */
  SWIN_ERR_CUDA = 3,        /* a CUDA runtime / driver call failed */
  SWIN_ERR_TIMEOUT = 4      /* a device-side bounded wait ran out */
} swin_status;

typedef enum {
  SWIN_MODE_DOT_BIAS = 0,
  SWIN_MODE_COSINE_CPB = 1,
  SWIN_MODE_ROPE = 2
} swin_mode;

typedef enum { SWIN_F32 = 0, SWIN_BF16 = 1 } swin_dtype;

/* How an axis of length L is cut into windows of M tokens.
 *   SWIN_PARTITION_SHIFTED      segments with boundaries at shift + kM (Swin's
 *        shifted windows; the page's window partition, described above);
 *        window-local coordinate (y - shift) mod M.
 *   SWIN_PARTITION_INTERLEAVED  G = ceil(L / M) windows per axis; window a
 *        holds the tokens a + G i, i < M, inside the axis ("Iwin Transformer:
 *        Hierarchical Vision Transformer using Interleaved Windows", abstract:
 *        interleaved window attention; the pages give no index formula, this
 *        strided grid is the reading taken); window-local coordinate i; shift
 *        must be 0.  A window then spans the whole image.
 * Bias-table offsets and RoPE positions use the window-local coordinates in
 * both partitions. */
typedef enum { SWIN_PARTITION_SHIFTED = 0, SWIN_PARTITION_INTERLEAVED = 1 } swin_partition;

/* Weights of the Log-CPB meta network G ("Swin Transformer V2", §3.3, eq. 3):
 *   G(dx_hat, dy_hat) = w2 . relu(w1 . (dx_hat, dy_hat) + b1) + b2
 * with dx_hat = sign(dx) * ln(1 + |dx|) (eq. 4).  All device fp32:
 *   w1 [hidden][2], b1 [hidden] or NULL (zero), w2 [heads][hidden],
 *   b2 [heads] or NULL (zero).  The page's code uses hidden = 512. */
typedef struct {
  int hidden;
  const float* w1;
  const float* b1;
  const float* w2;
  const float* b2;
} swin_cpb_weights;

/* swin_cpb_eval — evaluate G once for every offset of an MxM window and store
 * the bias table ("Swin Transformer V2", §3.3: precompute the biases for
 * inference; eq. 3, eq. 4).
 *   M          window size, 1 <= M <= 64
 *   heads      1 <= heads <= 64
 *   g          weights (device pointers), 1 <= g->hidden <= 4096
 *   table_out  device fp32 [(2M-1)^2][heads], row (dy+M-1)*(2M-1)+(dx+M-1)
 * Computed in fp32 with the CUDA math library's logarithm. */
swin_status swin_cpb_eval(int M, int heads, const swin_cpb_weights* g, float* table_out,
                          swin_stream_t stream);

/* Forms of G's input transform and output ("Swin Transformer V2" wiki card,
 * "Paper vs code": the released code departs from eq. 3 / eq. 4). */
typedef enum {
  SWIN_CPB_PAPER = 0, /* eq. 4 on raw offsets: sign(d) ln(1 + |d|); B = G (as swin_cpb_eval) */
  SWIN_CPB_CODE = 1   /* d' = 8 d / (Mp - 1), Mp the pretrained window (M if none);
                         sign(d') log2(1 + |d'|) / log2(8); B = 16 sigmoid(G), in (0, 16) */
} swin_cpb_form;

/* swin_cpb_eval_form — swin_cpb_eval with a choice of form.  pretrained_M is
 * the window G was trained at (0: M itself); a table for a larger test-time
 * window M then extrapolates G beyond the trained coordinate range (§3.3:
 * transfer across window sizes).  With Mp == 1 every coordinate is 0.
 *   form          a swin_cpb_form
 *   pretrained_M  0 or 1 <= pretrained_M <= 64 (SWIN_CPB_CODE only; must be 0
 *                 for SWIN_CPB_PAPER, whose transform has no normaliser)
 * Other arguments, layout and errors as swin_cpb_eval. */
swin_status swin_cpb_eval_form(int M, int heads, const swin_cpb_weights* g, swin_cpb_form form,
                               int pretrained_M, float* table_out, swin_stream_t stream);

/* swin_window_attn_fwd — the shifted-window attention forward pass.
 *   q, k, v, out   device [B][H][W][heads][d]; q, k, v of dtype dt, out of
 *                  dtype out_dt (out_dt == dt, or SWIN_F32 output for SWIN_BF16
 *                  inputs: the same fp32 result before its final rounding;
 *                  a bf16 output is that fp32 result rounded to nearest even)
 *   B, H, W        batch and grid, each >= 1; B*H*W*heads*d < 2^31
 *   heads, d       heads >= 1; d in {8, 16, 32, 64} for SWIN_F32; d == 32 for
 *                  SWIN_BF16 (the tensor-core path); RoPE needs d % 4 == 0
 *   M, shift       window size 1 <= M <= 64, shift 0 <= shift < M
 *   mode           a swin_mode
 *   tau            device fp32 [heads], SWIN_MODE_COSINE_CPB only (else NULL);
 *                  the kernel uses max(tau, 0.01)
 *   bias_table     device fp32 [(2M-1)^2][heads] or NULL (modes 0 and 1;
 *                  NULL in mode 1 means "evaluate cpb"; NULL in mode 0 means
 *                  no bias); must be NULL in SWIN_MODE_ROPE
 *   cpb            mode 1 with bias_table == NULL: G's weights (host struct,
 *                  device arrays); the table is evaluated into the workspace
 *                  on the same stream; may be NULL otherwise
 *   rope_freqs     device fp32 [2][d/4] (row axis, then column axis),
 *                  SWIN_MODE_ROPE only
 *   workspace      device scratch of at least
 *                  swin_window_attn_workspace_size(...) bytes, 256-byte
 *                  aligned (may be NULL when that size is 0)
 *   stream         CUDA stream
 * Asynchronous; q/k/v must stay valid until the stream reaches the call.
 *
 * Arithmetic of the bf16, d == 32 path (tcgen05 tensor cores; taken when
 * there is no bias table or M <= 32, else the CUDA-core path runs; windows of
 * at most 64 tokens, M <= 8, use a kernel that loads rows into shared memory
 * instead of TMA tiles): q.k products of the bf16 inputs accumulate in fp32
 * (modes 0 and 1; mode 1 applies 1/|q|, 1/|k| and 1/tau in fp32 afterwards,
 * and the bias is added in fp32); mode 2 rotates q and k in fp32 and
 * multiplies them as fp16 (q scaled by an exact power of two; for M <= 8 as
 * fp16 hi + lo parts).  Probabilities (at most 2^8 times the running
 * maximum's) and V are carried in fp16, sums in fp32, and the row sum is
 * accumulated from the same fp16 probabilities that weight V.  A rotated k
 * entry or a V entry of magnitude 65504 or more saturates; the kernel then
 * records SWIN_ERR_UNSUPPORTED, which swin_stream_status reports. */
swin_status swin_window_attn_fwd(const void* q, const void* k, const void* v, void* out,
                                 swin_dtype dt, swin_dtype out_dt, int B, int H, int W,
                                 int heads, int d,
                                 int M, int shift, swin_mode mode,
                                 const float* tau, const float* bias_table,
                                 const swin_cpb_weights* cpb, const float* rope_freqs,
                                 void* workspace, size_t workspace_bytes,
                                 swin_stream_t stream);

/* swin_window_attn_fwd_ex — swin_window_attn_fwd with a choice of window
 * partition (a swin_partition; swin_window_attn_fwd is this call with
 * SWIN_PARTITION_SHIFTED).  Interleaved windows run on the CUDA cores for
 * every dtype (the tensor-core path gathers contiguous rectangles only).
 * Arguments, layout, workspace and errors otherwise as swin_window_attn_fwd;
 * an unknown partition, or a non-zero shift with interleaved windows, returns
 * SWIN_ERR_INVALID_ARG. */
swin_status swin_window_attn_fwd_ex(const void* q, const void* k, const void* v, void* out,
                                    swin_dtype dt, swin_dtype out_dt, int B, int H, int W, int heads,
                                    int d, int M, int shift, swin_partition partition, swin_mode mode,
                                    const float* tau, const float* bias_table,
                                    const swin_cpb_weights* cpb, const float* rope_freqs,
                                    void* workspace, size_t workspace_bytes, swin_stream_t stream);

/* swin_window_attn_fwd_noalloc — the same forward pass for callers that
 * cannot allocate device memory (a framework that owns every device byte
 * through its own pool, code running under stream capture, an embedding that
 * forbids allocation after start-up).  The pages have no counterpart: it only
 * changes where scratch lives.  Arguments as swin_window_attn_fwd, without a
 * workspace.  When the cosine mode must evaluate the CPB meta network, the
 * table goes into a fixed device array of the library (131072 floats, 512 KiB,
 * held on every GPU that loads the library until exit) instead of caller
 * scratch; (2M-1)^2 * heads above 131072 returns SWIN_ERR_UNSUPPORTED.  The
 * first call on a device looks the array's address up (cudaGetSymbolAddress)
 * and should come before any stream capture.  Argument errors return before
 * anything is enqueued, leaving the array untouched.  All calls share the array, and
 * calls whose kernels overlap on the GPU race on it: serialise them.  Every
 * table entry is rewritten on each call; the array keeps the last call's
 * table.  Allocates nothing. */
swin_status swin_window_attn_fwd_noalloc(const void* q, const void* k, const void* v, void* out,
                                         swin_dtype dt, swin_dtype out_dt, int B, int H, int W,
                                         int heads, int d, int M, int shift, swin_mode mode,
                                         const float* tau, const float* bias_table,
                                         const swin_cpb_weights* cpb, const float* rope_freqs,
                                         swin_stream_t stream);

/* Bytes of workspace swin_window_attn_fwd needs for these arguments
 * (have_table: whether bias_table is non-NULL).  0 when none is needed. */
size_t swin_window_attn_workspace_size(int M, int heads, swin_mode mode, int have_table);

/* swin_window_attn_bwd — gradients of swin_window_attn_fwd's output with
 * respect to its inputs and parameters, for training (the pages train every
 * model they describe; FlashSwin's abstract rests its training-memory claim
 * on attention that keeps no score matrix, and neither does this pass).  For
 * L = sum over all elements of dout * out, it writes dq, dk, dv = dL/dq,
 * dL/dk, dL/dv and, when asked, dtable = dL/dT, dtau = dL/dtau and
 * drope = dL/dw.  The softmax is recomputed from q, k, v; nothing from the
 * forward pass is needed.  Conventions:
 *   - tau below 0.01 is clamped, so its gradient is 0 there; at and above
 *     0.01 (compared as real numbers: the fp32 value nearest 0.01 lies just
 *     below it) the gradient passes ("Swin Transformer V2" §3.2);
 *   - a q or k row of norm at most 1e-12 (mode 1) has its norm held at
 *     1e-12, a constant;
 *   - the gradient of the CPB meta network's weights is not formed: in mode
 *     1, pass the table swin_cpb_eval produced and back-propagate dtable
 *     through G.
 *   q, k, v, dout    device [B][H][W][heads][d] of dtype dt (SWIN_F32 or
 *                    SWIN_BF16)
 *   dq, dk, dv       device [B][H][W][heads][d] of dtype grad_dt (== dt, or
 *                    SWIN_F32 for SWIN_BF16 inputs; a bf16 gradient is the
 *                    fp32 one rounded to nearest even); written, not added to;
 *                    must not overlap each other or the inputs
 *   B, H, W, heads, d, M, shift, mode, tau, rope_freqs
 *                    as swin_window_attn_fwd, except that d may be 8, 16, 32
 *                    or 64 for both dtypes
 *   partition        a swin_partition, as swin_window_attn_fwd_ex
 *   bias_table       device fp32 [(2M-1)^2][heads] or NULL, modes 0 and 1
 *                    (mode 1 takes the table, not the CPB weights)
 *   dtable           device fp32 [(2M-1)^2][heads] or NULL; needs bias_table
 *   dtau             device fp32 [heads] or NULL; mode 1 only
 *   drope            device fp32 [2][d/4] or NULL; mode 2 only
 *   workspace        device scratch of swin_window_attn_bwd_workspace_size
 *                    bytes, 256-byte aligned
 * Arithmetic.  SWIN_BF16 tensors with d == 32 and M <= 32 (either
 * partition): the tensor cores (tcgen05), the five products with fp16
 * operands and fp32 accumulation — q, k, v, dout converted exactly from bf16
 * inside fp16's range, RoPE-rotated q and k carried as fp16 hi + lo parts,
 * probabilities and dS in fp16 — and the softmax in fp32; an operand at or
 * beyond fp16's range saturates and the call reports SWIN_ERR_UNSUPPORTED
 * through swin_stream_status.  Otherwise the CUDA cores: double arithmetic
 * for SWIN_F32 tensors, fp32 for SWIN_BF16.  dq, dk, dv are deterministic.
 * Parameter gradients are summed by double atomic additions and rounded once
 * to fp32; the order of the additions varies, so between calls they may
 * differ in the last bit.
 * Errors as swin_window_attn_fwd: argument errors return before anything is
 * enqueued. */
swin_status swin_window_attn_bwd(const void* q, const void* k, const void* v, const void* dout,
                                 void* dq, void* dk, void* dv, swin_dtype dt, swin_dtype grad_dt,
                                 int B, int H, int W, int heads, int d, int M, int shift,
                                 swin_partition partition, swin_mode mode, const float* tau,
                                 const float* bias_table, const float* rope_freqs, float* dtable,
                                 float* dtau, float* drope,
                                 void* workspace, size_t workspace_bytes, swin_stream_t stream);

/* Bytes of workspace swin_window_attn_bwd needs: 16 per query row and head
 * (its log-sum-exp and D = dout . out, in double) plus the double
 * accumulators of the parameter gradients, rounded up to 256. */
size_t swin_window_attn_bwd_workspace_size(int B, int H, int W, int heads, int d, int M);

/* The steps either side of the attention in a Swin V2 block ("Swin
 * Transformer V2" wiki card, Method item 1 "Residual post-norm", §3.2,
 * fig. 1, and the swin_v2_block pseudocode): the block input x is projected
 * to q, k and v; after the attention, its output a is projected back and
 * layer-normalised before joining the residual path (post-norm: the norm sits
 * on the branch's output, not on its input).  All tensors are device arrays,
 * dense row-major, of dtype dt (fp32 or bf16), with C = heads * d channels per
 * token; the token order is the caller's ([B][H][W] for the attention).
 * Weights follow the usual linear-layer layout [out][in]; biases, gamma and
 * beta are fp32.  For bf16 inputs with C a multiple of 32 (at most 96 for
 * the qkv projection, 128 for the post-norm) each step is one tensor-core
 * kernel (tcgen05, bf16 products, fp32 accumulation, the epilogue in fp32)
 * that leaves the workspace untouched; otherwise the projection is a
 * cuBLASLt GEMM with fp32 accumulation into the caller's workspace (fp32)
 * and the bias, the post-norm and the residual add are this library's
 * kernels, in fp32.  Either way every output element is rounded once:
 * outputs of dtype out_dt (== dt, or SWIN_F32 for SWIN_BF16 inputs; a bf16
 * output is the fp32 one rounded to nearest even).  Pointers 16-byte
 * aligned, workspaces 256-byte aligned; C a multiple of 8.  Asynchronous on
 * the stream. */

/* q = x Wq^T + bq, k = x Wk^T + bk, v = x Wv^T + bv, with
 *   x        [tokens][C]
 *   w_qkv    [3C][C]: the rows of Wq, then Wk, then Wv
 *   b_qkv    fp32 [3C] or NULL (no bias)
 *   q, k, v  [tokens][C] each (= [B][H][W][heads][d]) of dtype out_dt; must
 *            not overlap x, each other or the workspace
 *   workspace  swin_qkv_proj_workspace_size(tokens, C) bytes (tokens x 3C
 *            fp32: the product before the bias) */
swin_status swin_qkv_proj(const void* x, const void* w_qkv, const float* b_qkv, void* q, void* k, void* v,
                          swin_dtype dt, swin_dtype out_dt, int tokens, int C, void* workspace,
                          size_t workspace_bytes, swin_stream_t stream);
size_t swin_qkv_proj_workspace_size(int tokens, int C);

/* out = x + LN(a Wo^T + bo), LN(y) = (y - mean(y)) / sqrt(var(y) + eps) *
 * gamma + beta over the C channels of each token (biased variance), with
 *   a        [tokens][C], the attention output
 *   w_o      [C][C];  b_o fp32 [C] or NULL
 *   x        [tokens][C], the residual path (the block's input)
 *   gamma, beta  fp32 [C] or NULL (1 and 0);  eps > 0 (1e-5 is the usual)
 *   out      [tokens][C] of dtype out_dt; must not overlap x, a or the
 *            workspace; C <= 1024
 *   workspace  swin_proj_postnorm_workspace_size(tokens, C) bytes (the fp32
 *            projection) */
swin_status swin_proj_postnorm_residual(const void* a, const void* w_o, const float* b_o, const void* x,
                                        const float* gamma, const float* beta, float eps, void* out, swin_dtype dt,
                                        swin_dtype out_dt, int tokens, int C, void* workspace, size_t workspace_bytes,
                                        swin_stream_t stream);
size_t swin_proj_postnorm_workspace_size(int tokens, int C);

/* The attention half of a Swin V2 block (the swin_v2_block pseudocode's first
 * two lines): swin_qkv_proj, swin_window_attn_fwd_ex, then
 * swin_proj_postnorm_residual, on one stream.  x and out are
 * [B][H][W][heads * d], out of dtype out_dt; the attention arguments are
 * swin_window_attn_fwd_ex's; out must not overlap x.  q, k, v and the
 * attention output are stored in dtype dt between the steps.  The workspace
 * (swin_attn_block_workspace_size bytes, 256-byte aligned) holds them, the
 * fp32 projections and the attention's own workspace.  Every argument is
 * checked before the first launch. */
swin_status swin_attn_block_fwd(const void* x, const void* w_qkv, const float* b_qkv, const void* w_o,
                                const float* b_o, const float* gamma, const float* beta, float eps, void* out,
                                swin_dtype dt, swin_dtype out_dt, int B, int H, int W, int heads, int d, int M,
                                int shift,
                                swin_partition partition, swin_mode mode, const float* tau, const float* bias_table,
                                const swin_cpb_weights* cpb, const float* rope_freqs, void* workspace,
                                size_t workspace_bytes, swin_stream_t stream);

/* Bytes of workspace swin_attn_block_fwd needs (0 for invalid sizes). */
size_t swin_attn_block_workspace_size(int B, int H, int W, int heads, int d, int M, swin_mode mode, int have_table,
                                      swin_dtype dt);

/* swin_index_tables — Swin's bookkeeping for an HxW grid in the rolled frame
 * (pad to Hp = ceil(H/M)*M, Wp likewise; roll by -shift; cut MxM windows), as
 * the kernels' index arithmetic sees it.  For testing; any output may be NULL.
 *   tok_window [H][W]  window id (u / M) * (Wp / M) + (v / M), with
 *                      u = (y - shift) mod Hp, v = (x - shift) mod Wp
 *   tok_region [H][W]  band label ry * 3 + rx; along an axis the band is 0
 *                      for u < Hp - M, 1 for u < Hp - shift, else 2 (0 when
 *                      shift == 0)
 *   tok_local  [H][W]  (u mod M) * M + (v mod M)
 *   rel_index  [M*M][M*M]  r(i, j) for window-local positions i, j
 * All int32 device arrays.  1 <= M <= 64, 0 <= shift < M, H, W >= 1. */
swin_status swin_index_tables(int H, int W, int M, int shift, int32_t* tok_window,
                              int32_t* tok_region, int32_t* tok_local, int32_t* rel_index,
                              swin_stream_t stream);

/* Synchronise the stream, then return and clear the device status word of the
 * current device (SWIN_OK, or SWIN_ERR_TIMEOUT if a kernel's bounded wait ran
 * out since the last call); SWIN_ERR_CUDA if the synchronisation failed. */
swin_status swin_stream_status(swin_stream_t stream);

/* Message describing the last non-OK status returned on this host thread
 * ("" if none).  The pointer stays valid until the next call on the thread. */
const char* swin_last_error(void);

/* Test hook for the failure path (no counterpart in the pages).  flags bit 0
 * makes every later tensor-core launch wait on a barrier that nothing
 * completes, so its bounded wait runs out, the kernel records
 * SWIN_ERR_TIMEOUT and returns cleanly; wait_limit_cycles (<= 0: default of
 * about two seconds) bounds every wait of those launches.  flags = 0 restores
 * normal operation.  Process-wide; not thread-safe against concurrent calls. */
swin_status swin_debug_set(int flags, long long wait_limit_cycles);

/* Library version, major * 10000 + minor * 100 + patch. */
int swin_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SWIN_ATTN_H */
