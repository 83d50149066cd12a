/*
 * Shifted-window attention oracle — TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, double-precision CPU statement of what the shifted-window
 * attention path computes.  Only the test suite, the package's smoke check and
 * the CPU-baseline leg of the benchmark may load this library; the product
 * path (libswinattn.so and its Python binding) never calls it.  It shares no
 * code, header, table or constant with the CUDA sources.
 *
 * Sources (all pages are read for what they compute; nothing is copied):
 *  [V2]  "Swin Transformer V2: Scaling Up Capacity and Resolution" (wiki card),
 *        Method: eq. 1 (dot-product attention plus bias B), eq. 2 (scaled
 *        cosine attention, tau per head kept at or above 0.01, §3.2),
 *        eq. 3 / eq. 4 (log-spaced continuous position bias, §3.3), the
 *        "window_attention" and "continuous_bias" pseudocode blocks, and the
 *        hyperparameter table (meta network G hidden width 512 in the code).
 *  [FS]  "FLASHSWIN: Unlocking Large Windows and Dense Tokens in Swin Vision
 *        Transformers with Memory Efficient Attention", Abstract: exact softmax
 *        attention inside each window, position information from window-local
 *        learnable 2D RoPE, no additive bias.
 *  [V2-pitfalls] Pitfalls, "Window divisibility": shift offsets with even or
 *        odd window sizes.
 *  [V2-code] "Paper vs code": the released code's CPB coordinates (offset
 *        scaled by 8 / (window - 1), sign(x) log2(1 + |x|) / log2(8)) and its
 *        16 sigmoid bound on G's output.
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *  R1  Shift mechanism (not spelled out; Swin V1 is cited only): along each
 *      axis the grid is cut into segments whose boundaries sit at s + kM,
 *      clipped to [0, L).  Two tokens attend to each other iff they lie in the
 *      same segment on both axes.  This is the attention that a cyclic roll by
 *      -s, an MxM window partition and a region mask produce.
 *  R2  Masked pairs get weight exactly zero.
 *  R3  A grid side not divisible by M: segments are clipped at the grid edge;
 *      padding tokens never exist here.
 *  R5  Offset sign and table layout: delta = query - key; table row
 *      (dy+M-1)*(2M-1) + (dx+M-1), heads innermost.
 *  R6  eq. 4's "sign(x)" is read as sign(delta x); log is natural (the worked
 *      example's 2.079 = ln 8 and 2.773 = ln 16); G takes (dx_hat, dy_hat).
 *  R7  G = Linear(2, hidden) -> ReLU -> Linear(hidden, heads); NULL biases = 0.
 *  R8  tau_eff = max(tau, 0.01); cosine mode has no 1/sqrt(d).
 *  R9  Vector norms clamped below at 1e-12.
 *  R10 RoPE: the first d/2 channels rotate with the window-local row
 *      coordinate, the last d/2 with the column coordinate; pairs (2t, 2t+1)
 *      inside each half rotate by p * omega[axis][t], t < d/4; the window-local
 *      coordinate is p = (y - s) mod M; RoPE touches q and k only; the score
 *      is scaled by 1/sqrt(d); no bias.
 *  R17 Interleaved windows ("Iwin Transformer", abstract only): the strided
 *      partition described at win_of below; the same three scores, with
 *      window-local coordinates in place of the shifted ones; no shift.
 *  R15 The code form of G ([V2] "Paper vs code"): the normaliser is the
 *      pretrained window Mp (the window itself when none is given); a window
 *      of 1 (Mp - 1 = 0) has only offset 0, whose coordinate is 0.
 *  R16 Gradients (the pages train the model but state no backward): the
 *      chain rule through the definitions above; the tau clamp passes the
 *      gradient for tau >= 0.01 and none below; a norm held at its 1e-12
 *      floor is a constant.
 *
 * Parity pins live in tests/test_oracle_*.py.  The CPB meta-network beyond
 * its W2 = 0 special case and a float64 library Linear stack is arithmetic
 * only; see the pins there.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Segment id of coordinate y along an axis under reading R1: boundaries at
 * s + kM.  Shifting the axis by (M - s) mod M turns them into multiples of M. */
int oracle_segment_of(int M, int s, int y) {
    return (y + (M - s) % M) / M;
}

/* The two partitions of an axis of length L into windows of M tokens:
 *   part 0, shifted (R1): the window is the segment under boundaries s + kM;
 *     the window-local coordinate is (y - s) mod M; the offset of two tokens
 *     of one window is the difference of their coordinates.
 *   part 1, interleaved ("Iwin Transformer" abstract, reading R17): with
 *     G = ceil(L / M) windows per axis, window a holds the tokens a + G i,
 *     i < M, that lie inside the axis, i.e. the window is y mod G and the
 *     window-local coordinate is i = y div G; offsets are differences of i. */
static int win_of(int part, int L, int M, int s, int y) {
    if (part == 0) return oracle_segment_of(M, s, y);
    return y % ((L + M - 1) / M);
}

static int loc_of(int part, int L, int M, int s, int y) {
    if (part == 0) return ((y - s) % M + M) % M;
    return y / ((L + M - 1) / M);
}

static int off_of(int part, int L, int M, int s, int yq, int yk) {
    if (part == 0) return yq - yk;
    return loc_of(part, L, M, s, yq) - loc_of(part, L, M, s, yk);
}

/* eq. 4: signed natural-log map of one offset component (reading R6). */
double oracle_log_map(double delta) {
    double sgn = (delta > 0.0) ? 1.0 : ((delta < 0.0) ? -1.0 : 0.0);
    return sgn * log(1.0 + fabs(delta));
}

/* Log-spaced coordinates for every offset of an MxM window:
 * out[((dy+M-1)*(2M-1) + (dx+M-1))*2 + {0,1}] = (dx_hat, dy_hat). */
void oracle_log_coords(int M, double* out) {
    int R = 2 * M - 1;
    for (int dy = -(M - 1); dy <= M - 1; ++dy)
        for (int dx = -(M - 1); dx <= M - 1; ++dx) {
            size_t row = (size_t)(dy + M - 1) * R + (dx + M - 1);
            out[row * 2 + 0] = oracle_log_map((double)dx);
            out[row * 2 + 1] = oracle_log_map((double)dy);
        }
}

/* eq. 3 with the default G of §3.3: a two-layer MLP with a ReLU between.
 * w1 [hidden][2], b1 [hidden] or NULL, w2 [heads][hidden], b2 [heads] or NULL.
 * table [(2M-1)^2][heads]. */
void oracle_cpb_table(int M, int heads, int hidden,
                      const double* w1, const double* b1,
                      const double* w2, const double* b2, double* table) {
    int R = 2 * M - 1;
    double* coords = (double*)malloc(sizeof(double) * (size_t)R * R * 2);
    double* hid = (double*)malloc(sizeof(double) * (size_t)hidden);
    oracle_log_coords(M, coords);
    for (int r = 0; r < R * R; ++r) {
        double in0 = coords[r * 2 + 0], in1 = coords[r * 2 + 1];
        for (int j = 0; j < hidden; ++j) {
            double a = w1[j * 2 + 0] * in0 + w1[j * 2 + 1] * in1 + (b1 ? b1[j] : 0.0);
            hid[j] = a > 0.0 ? a : 0.0;
        }
        for (int h = 0; h < heads; ++h) {
            double acc = b2 ? b2[h] : 0.0;
            for (int j = 0; j < hidden; ++j) acc += w2[(size_t)h * hidden + j] * hid[j];
            table[(size_t)r * heads + h] = acc;
        }
    }
    free(hid);
    free(coords);
}

/* The released code's form of G ("Swin Transformer V2" wiki card, "Paper vs
 * code"): each offset component is first scaled by 8 / (Mp - 1), Mp the
 * window G was pretrained at (a window of 1 has only offset 0: coordinate 0),
 * then mapped by sign(x) log2(1 + |x|) / log2(8); the MLP's output is bounded
 * as 16 sigmoid(G). */
double oracle_log2_map(double delta, int Mp) {
    double x = Mp > 1 ? delta * 8.0 / (double)(Mp - 1) : 0.0;
    double sgn = (x > 0.0) ? 1.0 : ((x < 0.0) ? -1.0 : 0.0);
    return sgn * log2(1.0 + fabs(x)) / log2(8.0);
}

void oracle_cpb_table_code(int M, int Mp, int heads, int hidden,
                           const double* w1, const double* b1,
                           const double* w2, const double* b2, double* table) {
    int R = 2 * M - 1;
    double* hid = (double*)malloc(sizeof(double) * (size_t)hidden);
    for (int dy = -(M - 1); dy <= M - 1; ++dy)
        for (int dx = -(M - 1); dx <= M - 1; ++dx) {
            size_t r = (size_t)(dy + M - 1) * R + (dx + M - 1);
            double in0 = oracle_log2_map((double)dx, Mp), in1 = oracle_log2_map((double)dy, Mp);
            for (int j = 0; j < hidden; ++j) {
                double a = w1[j * 2 + 0] * in0 + w1[j * 2 + 1] * in1 + (b1 ? b1[j] : 0.0);
                hid[j] = a > 0.0 ? a : 0.0;
            }
            for (int h = 0; h < heads; ++h) {
                double z = b2 ? b2[h] : 0.0;
                for (int j = 0; j < hidden; ++j) z += w2[(size_t)h * hidden + j] * hid[j];
                table[r * heads + h] = 16.0 / (1.0 + exp(-z));
            }
        }
    free(hid);
}

/* Swin-style bookkeeping tables, built by literally simulating the cyclic
 * roll of a padded grid (pad to a multiple of M, roll by -s, cut MxM windows,
 * label the three bands of the last window row/column).
 *   tok_window[y*W+x] : window index wy*nWx + wx in the rolled frame
 *   tok_region[y*W+x] : band label ry*3 + rx (0 when s == 0)
 *   tok_local[y*W+x]  : (u mod M)*M + (v mod M)
 *   rel_index[i*N+j]  : (yi-yj+M-1)*(2M-1) + (xi-xj+M-1) for window-local
 *                       positions i, j (N = M*M).  Any pointer may be NULL. */
void oracle_index_tables(int H, int W, int M, int s,
                         int32_t* tok_window, int32_t* tok_region,
                         int32_t* tok_local, int32_t* rel_index) {
    int Hp = ((H + M - 1) / M) * M, Wp = ((W + M - 1) / M) * M;
    int nWx = Wp / M;
    /* Rolled frame: position (u, v) holds original (y, x) = ((u+s)%Hp, (v+s)%Wp).
     * Build it by moving every element of the padded grid, as a roll does. */
    int* orig_y = (int*)malloc(sizeof(int) * (size_t)Hp * Wp);
    int* orig_x = (int*)malloc(sizeof(int) * (size_t)Hp * Wp);
    for (int y = 0; y < Hp; ++y)
        for (int x = 0; x < Wp; ++x) {
            int u = ((y - s) % Hp + Hp) % Hp;  /* roll by -s moves y to y - s */
            int v = ((x - s) % Wp + Wp) % Wp;
            orig_y[u * Wp + v] = y;
            orig_x[u * Wp + v] = x;
        }
    for (int u = 0; u < Hp; ++u)
        for (int v = 0; v < Wp; ++v) {
            int y = orig_y[u * Wp + v], x = orig_x[u * Wp + v];
            if (y >= H || x >= W) continue; /* padding token */
            int ry = 0, rx = 0;
            if (s > 0) {
                ry = (u < Hp - M) ? 0 : ((u < Hp - s) ? 1 : 2);
                rx = (v < Wp - M) ? 0 : ((v < Wp - s) ? 1 : 2);
            }
            size_t t = (size_t)y * W + x;
            if (tok_window) tok_window[t] = (u / M) * nWx + (v / M);
            if (tok_region) tok_region[t] = ry * 3 + rx;
            if (tok_local) tok_local[t] = (u % M) * M + (v % M);
        }
    if (rel_index) {
        int N = M * M, R = 2 * M - 1;
        for (int i = 0; i < N; ++i)
            for (int j = 0; j < N; ++j) {
                int yi = i / M, xi = i % M, yj = j / M, xj = j % M;
                rel_index[(size_t)i * N + j] = (yi - yj + M - 1) * R + (xi - xj + M - 1);
            }
    }
    free(orig_y);
    free(orig_x);
}

/* Rotate channels [base, base + d/2) of x in place by position p (reading R10). */
static void rope_half(double* x, int d, int base, int p, const double* omega) {
    for (int t = 0; t < d / 4; ++t) {
        double th = (double)p * omega[t];
        double c = cos(th), sn = sin(th);
        double a = x[base + 2 * t], b = x[base + 2 * t + 1];
        x[base + 2 * t] = a * c - b * sn;
        x[base + 2 * t + 1] = a * sn + b * c;
    }
}

static double norm_clamped(const double* x, int d) {
    double ss = 0.0;
    for (int e = 0; e < d; ++e) ss += x[e] * x[e];
    double n = sqrt(ss);
    return n > 1e-12 ? n : 1e-12;
}

/* Shifted-window multi-head attention, one query token (all heads) at a time.
 *
 *  q, k, v  [B][H][W][heads][d]
 *  part     0: shifted windows (shift s); 1: interleaved windows (s must be 0)
 *  mode 0   eq. 1: q.k/sqrt(d) + table[rel][h]
 *  mode 1   eq. 2: cos(q,k)/max(tau_h, 0.01) + table[rel][h]
 *  mode 2   FlashSwin: (R(p_i) q).(R(p_j) k)/sqrt(d), rope_freqs [2][d/4]
 *  table    [(2M-1)^2][heads] (modes 0 and 1; NULL means zero bias)
 *  queries  flat token ids b*H*W + y*W + x to evaluate (NULL: all, in order)
 *  out      [nq][heads][d]
 * Returns 0, or -1 on an argument the definition does not cover. */
int oracle_window_attn(const double* q, const double* k, const double* v, double* out,
                       int B, int H, int W, int heads, int d, int M, int s, int part, int mode,
                       const double* tau, const double* table, const double* rope_freqs,
                       const int64_t* queries, int64_t nq, int nthreads) {
    if (B < 1 || H < 1 || W < 1 || heads < 1 || d < 1 || M < 1 || s < 0 || s >= M) return -1;
    if (part < 0 || part > 1 || (part == 1 && s != 0)) return -1;
    if (mode == 2 && (d % 4 != 0 || !rope_freqs)) return -1;
    if (mode == 1 && !tau) return -1;
    if (mode < 0 || mode > 2) return -1;
    int64_t total = (int64_t)B * H * W;
    if (!queries) nq = total;
    int R = 2 * M - 1;
    size_t C = (size_t)heads * d;
    double rsd = 1.0 / sqrt((double)d);
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
#pragma omp parallel
    {
        /* per-thread scratch: key list, logits, rotated copies */
        int maxkeys = H * W;
        int* ky = (int*)malloc(sizeof(int) * (size_t)maxkeys);
        int* kx = (int*)malloc(sizeof(int) * (size_t)maxkeys);
        double* logit = (double*)malloc(sizeof(double) * (size_t)maxkeys);
        double* qi = (double*)malloc(sizeof(double) * (size_t)d);
        double* kj = (double*)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(dynamic, 16)
        for (int64_t n = 0; n < nq; ++n) {
            int64_t tok = queries ? queries[n] : n;
            int b = (int)(tok / ((int64_t)H * W));
            int yi = (int)((tok / W) % H), xi = (int)(tok % W);
            /* R1 / R17: key set = same window on both axes */
            int sy = win_of(part, H, M, s, yi), sx = win_of(part, W, M, s, xi);
            int nk = 0;
            for (int y = 0; y < H; ++y) {
                if (win_of(part, H, M, s, y) != sy) continue;
                for (int x = 0; x < W; ++x) {
                    if (win_of(part, W, M, s, x) != sx) continue;
                    ky[nk] = y; kx[nk] = x; ++nk;
                }
            }
            for (int h = 0; h < heads; ++h) {
                const double* qsrc = q + ((size_t)tok) * C + (size_t)h * d;
                for (int e = 0; e < d; ++e) qi[e] = qsrc[e];
                double qn = 1.0;
                if (mode == 1) qn = norm_clamped(qi, d);
                if (mode == 2) {
                    int py = loc_of(part, H, M, s, yi), px = loc_of(part, W, M, s, xi);
                    rope_half(qi, d, 0, py, rope_freqs);
                    rope_half(qi, d, d / 2, px, rope_freqs + d / 4);
                }
                double mx = -INFINITY;
                for (int j = 0; j < nk; ++j) {
                    size_t ktok = ((size_t)b * H + ky[j]) * W + kx[j];
                    const double* ksrc = k + ktok * C + (size_t)h * d;
                    for (int e = 0; e < d; ++e) kj[e] = ksrc[e];
                    double lg;
                    if (mode == 2) {
                        int py = loc_of(part, H, M, s, ky[j]), px = loc_of(part, W, M, s, kx[j]);
                        rope_half(kj, d, 0, py, rope_freqs);
                        rope_half(kj, d, d / 2, px, rope_freqs + d / 4);
                    }
                    double dot = 0.0;
                    for (int e = 0; e < d; ++e) dot += qi[e] * kj[e];
                    if (mode == 0) {
                        lg = dot * rsd;
                    } else if (mode == 1) {
                        double kn = norm_clamped(kj, d);
                        double t = tau[h] > 0.01 ? tau[h] : 0.01;
                        lg = dot / (qn * kn) / t;
                    } else {
                        lg = dot * rsd;
                    }
                    if (mode != 2 && table) {
                        int dy = off_of(part, H, M, s, yi, ky[j]), dx = off_of(part, W, M, s, xi, kx[j]);
                        lg += table[(size_t)((dy + M - 1) * R + (dx + M - 1)) * heads + h];
                    }
                    logit[j] = lg;
                    if (lg > mx) mx = lg;
                }
                /* exact two-pass softmax, then the weighted sum of values */
                double den = 0.0;
                for (int j = 0; j < nk; ++j) { logit[j] = exp(logit[j] - mx); den += logit[j]; }
                double* o = out + (size_t)n * C + (size_t)h * d;
                for (int e = 0; e < d; ++e) o[e] = 0.0;
                for (int j = 0; j < nk; ++j) {
                    size_t ktok = ((size_t)b * H + ky[j]) * W + kx[j];
                    const double* vsrc = v + ktok * C + (size_t)h * d;
                    double w = logit[j] / den;
                    for (int e = 0; e < d; ++e) o[e] += w * vsrc[e];
                }
            }
        }
        free(ky); free(kx); free(logit); free(qi); free(kj);
    }
    return 0;
}

/* Gradients of the shifted-window attention (the chain rule through the
 * forward above, written out; the softmax is recomputed, nothing is stored
 * between passes).  With L = sum(dout . out), P the softmax weights of query
 * i over its key set, g_i = dout_i:
 *   dv_j   = sum_i P_ij g_i
 *   dP_ij  = g_i . v_j,   D_i = sum_j P_ij dP_ij,   dl_ij = P_ij (dP_ij - D_i)
 * and dl_ij flows into the score:
 *   mode 0  l = q.k/sqrt(d) + T[r]:  dq_i += dl k_j/sqrt(d), dk_j += dl q_i/sqrt(d), dT[r] += dl
 *   mode 1  l = c/t + T[r], c = q.k/(|q||k|), t = max(tau, 0.01):
 *           dc/dq = k/(|q||k|) - c q/|q|^2 (the second term absent when |q| is
 *           clamped at 1e-12, R9), the same with q and k swapped;
 *           dtau += -dl c/t^2 when tau >= 0.01 (reading R16: the clamp passes
 *           the gradient from 0.01 up), else nothing
 *   mode 2  l = (R_i q_i).(R_j k_j)/sqrt(d): the rotated vectors take the
 *           mode-0 gradients, which rotate back by R^T; a pair rotated by
 *           theta = p omega_t has d(Rx)/dtheta = (-(Rx)_1, (Rx)_0), so
 *           domega_t += p (dRx . d(Rx)/dtheta) over every query and key.
 * Outputs are overwritten (zeroed first).  dtable [(2M-1)^2][heads], dtau
 * [heads] and drope [2][d/4] may be NULL.  Returns 0, or -1 as the forward. */
int oracle_window_attn_bwd(const double* q, const double* k, const double* v, const double* dout,
                           double* dq, double* dk, double* dv, double* dtable, double* dtau, double* drope,
                           int B, int H, int W, int heads, int d, int M, int s, int part, int mode,
                           const double* tau, const double* table, const double* rope_freqs, int nthreads) {
    if (B < 1 || H < 1 || W < 1 || heads < 1 || d < 1 || M < 1 || s < 0 || s >= M) return -1;
    if (part < 0 || part > 1 || (part == 1 && s != 0)) return -1;
    if (mode == 2 && (d % 4 != 0 || !rope_freqs)) return -1;
    if (mode == 1 && !tau) return -1;
    if (mode < 0 || mode > 2) return -1;
    const int R = 2 * M - 1;
    const size_t C = (size_t)heads * d, ntok = (size_t)B * H * W;
    const double rsd = 1.0 / sqrt((double)d);
    memset(dq, 0, sizeof(double) * ntok * C);
    memset(dk, 0, sizeof(double) * ntok * C);
    memset(dv, 0, sizeof(double) * ntok * C);
    if (dtable) memset(dtable, 0, sizeof(double) * (size_t)R * R * heads);
    if (dtau) memset(dtau, 0, sizeof(double) * (size_t)heads);
    if (drope) memset(drope, 0, sizeof(double) * 2 * (size_t)(d / 4));
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
#pragma omp parallel
    {
        const size_t HW = (size_t)H * W;
        int* ky = (int*)malloc(sizeof(int) * HW);
        int* kx = (int*)malloc(sizeof(int) * HW);
        double* pw = (double*)malloc(sizeof(double) * HW);     /* softmax weights of one query */
        double* cw = (double*)malloc(sizeof(double) * HW);     /* mode 1: cosines of one query */
        double* kr = (double*)malloc(sizeof(double) * HW * d); /* keys of the image-head, rotated in mode 2 */
        double* qr = (double*)malloc(sizeof(double) * HW * d); /* queries, rotated in mode 2 */
        double* dkr = (double*)malloc(sizeof(double) * HW * d);
        double* nrm = (double*)malloc(sizeof(double) * HW);    /* mode 1: clamped norms */
        unsigned char* clamped = (unsigned char*)malloc(HW);
        double* gq = (double*)malloc(sizeof(double) * (size_t)d);
        double* my_dtable = dtable ? (double*)calloc((size_t)R * R * heads, sizeof(double)) : NULL;
        double* my_dtau = dtau ? (double*)calloc((size_t)heads, sizeof(double)) : NULL;
        double* my_drope = drope ? (double*)calloc(2 * (size_t)(d / 4), sizeof(double)) : NULL;
#pragma omp for schedule(dynamic, 1)
        for (int bh = 0; bh < B * heads; ++bh) {
            const int b = bh / heads, h = bh % heads;
            /* this image-head's queries and keys, rotated in mode 2 */
            for (size_t t = 0; t < HW; ++t) {
                const size_t tok = (size_t)b * HW + t;
                const int y = (int)(t / W), x = (int)(t % W);
                for (int e = 0; e < d; ++e) {
                    qr[t * d + e] = q[tok * C + (size_t)h * d + e];
                    kr[t * d + e] = k[tok * C + (size_t)h * d + e];
                    dkr[t * d + e] = 0.0;
                }
                if (mode == 1) {
                    double ss = 0.0;
                    for (int e = 0; e < d; ++e) ss += kr[t * d + e] * kr[t * d + e];
                    nrm[t] = sqrt(ss) > 1e-12 ? sqrt(ss) : 1e-12;
                    clamped[t] = !(sqrt(ss) > 1e-12);
                }
                if (mode == 2) {
                    const int py = loc_of(part, H, M, s, y), px = loc_of(part, W, M, s, x);
                    rope_half(qr + t * d, d, 0, py, rope_freqs);
                    rope_half(qr + t * d, d, d / 2, px, rope_freqs + d / 4);
                    rope_half(kr + t * d, d, 0, py, rope_freqs);
                    rope_half(kr + t * d, d, d / 2, px, rope_freqs + d / 4);
                }
            }
            const double tt = mode == 1 ? (tau[h] > 0.01 ? tau[h] : 0.01) : 1.0;
            for (size_t ti = 0; ti < HW; ++ti) {
                const size_t tok = (size_t)b * HW + ti;
                const int yi = (int)(ti / W), xi = (int)(ti % W);
                const int sy = win_of(part, H, M, s, yi), sx = win_of(part, W, M, s, xi);
                int nk = 0;
                for (int y = 0; y < H; ++y) {
                    if (win_of(part, H, M, s, y) != sy) continue;
                    for (int x = 0; x < W; ++x) {
                        if (win_of(part, W, M, s, x) != sx) continue;
                        ky[nk] = y; kx[nk] = x; ++nk;
                    }
                }
                const double* qi = qr + ti * d;
                double qn = 1.0;
                int qclamped = 0;
                if (mode == 1) {
                    double qss = 0.0;
                    for (int e = 0; e < d; ++e) qss += qi[e] * qi[e];
                    qclamped = !(sqrt(qss) > 1e-12);
                    qn = qclamped ? 1e-12 : sqrt(qss);
                }
                /* forward: logits, softmax, output */
                double mx = -INFINITY;
                for (int j = 0; j < nk; ++j) {
                    const size_t tj = (size_t)ky[j] * W + kx[j];
                    const double* kj = kr + tj * d;
                    double dot = 0.0;
                    for (int e = 0; e < d; ++e) dot += qi[e] * kj[e];
                    double lg;
                    if (mode == 1) {
                        cw[j] = dot / (qn * nrm[tj]);
                        lg = cw[j] / tt;
                    } else {
                        lg = dot * rsd;
                    }
                    if (mode != 2 && table)
                        lg += table[(size_t)((off_of(part, H, M, s, yi, ky[j]) + M - 1) * R + (off_of(part, W, M, s, xi, kx[j]) + M - 1)) * heads + h];
                    pw[j] = lg;
                    if (lg > mx) mx = lg;
                }
                double den = 0.0;
                for (int j = 0; j < nk; ++j) { pw[j] = exp(pw[j] - mx); den += pw[j]; }
                for (int j = 0; j < nk; ++j) pw[j] /= den;
                const double* g = dout + tok * C + (size_t)h * d;
                /* D_i = sum_j P_ij (g . v_j) */
                double Dsum = 0.0;
                for (int j = 0; j < nk; ++j) {
                    const size_t tj = ((size_t)b * H + ky[j]) * W + kx[j];
                    const double* vj = v + tj * C + (size_t)h * d;
                    double dp = 0.0;
                    for (int e = 0; e < d; ++e) dp += g[e] * vj[e];
                    Dsum += pw[j] * dp;
                }
                for (int e = 0; e < d; ++e) gq[e] = 0.0;
                for (int j = 0; j < nk; ++j) {
                    const size_t tj = (size_t)ky[j] * W + kx[j];
                    const size_t gtj = (size_t)b * HW + tj;
                    const double* vj = v + gtj * C + (size_t)h * d;
                    double* dvj = dv + gtj * C + (size_t)h * d;
                    double dp = 0.0;
                    for (int e = 0; e < d; ++e) {
                        dp += g[e] * vj[e];
                        dvj[e] += pw[j] * g[e];
                    }
                    const double dl = pw[j] * (dp - Dsum);
                    const double* kj = kr + tj * d;
                    double* dkj = dkr + tj * d;
                    if (mode == 1) {
                        const double c = cw[j], kn = nrm[tj], a = dl / tt;
                        for (int e = 0; e < d; ++e) {
                            gq[e] += a * (kj[e] / (qn * kn) - (qclamped ? 0.0 : c * qi[e] / (qn * qn)));
                            dkj[e] += a * (qi[e] / (qn * kn) - (clamped[tj] ? 0.0 : c * kj[e] / (kn * kn)));
                        }
                        if (my_dtau && tau[h] >= 0.01) my_dtau[h] += -dl * c / (tt * tt);
                    } else {
                        for (int e = 0; e < d; ++e) {
                            gq[e] += dl * kj[e] * rsd;
                            dkj[e] += dl * qi[e] * rsd;
                        }
                    }
                    if (mode != 2 && my_dtable)
                        my_dtable[(size_t)((off_of(part, H, M, s, yi, ky[j]) + M - 1) * R + (off_of(part, W, M, s, xi, kx[j]) + M - 1)) * heads + h] += dl;
                }
                /* gq is the gradient of the (rotated, in mode 2) query */
                double* dqi = dq + tok * C + (size_t)h * d;
                if (mode == 2) {
                    const int pos[2] = {loc_of(part, H, M, s, yi), loc_of(part, W, M, s, xi)};
                    for (int half = 0; half < 2; ++half)
                        for (int t = 0; t < d / 4; ++t) {
                            const int e0 = half * (d / 2) + 2 * t;
                            const double th = (double)pos[half] * rope_freqs[half * (d / 4) + t];
                            const double c = cos(th), sn = sin(th);
                            /* R^T applied to the gradient pair */
                            dqi[e0] = gq[e0] * c + gq[e0 + 1] * sn;
                            dqi[e0 + 1] = -gq[e0] * sn + gq[e0 + 1] * c;
                            if (my_drope) my_drope[half * (d / 4) + t] +=
                                (double)pos[half] * (gq[e0] * -qi[e0 + 1] + gq[e0 + 1] * qi[e0]);
                        }
                } else {
                    for (int e = 0; e < d; ++e) dqi[e] = gq[e];
                }
            }
            /* keys: rotate the accumulated gradients back (mode 2) */
            for (size_t tj = 0; tj < HW; ++tj) {
                const size_t gtj = (size_t)b * HW + tj;
                double* dkj = dk + gtj * C + (size_t)h * d;
                const double* g2 = dkr + tj * d;
                if (mode == 2) {
                    const int y = (int)(tj / W), x = (int)(tj % W);
                    const int pos[2] = {loc_of(part, H, M, s, y), loc_of(part, W, M, s, x)};
                    const double* kj = kr + tj * d;
                    for (int half = 0; half < 2; ++half)
                        for (int t = 0; t < d / 4; ++t) {
                            const int e0 = half * (d / 2) + 2 * t;
                            const double th = (double)pos[half] * rope_freqs[half * (d / 4) + t];
                            const double c = cos(th), sn = sin(th);
                            dkj[e0] = g2[e0] * c + g2[e0 + 1] * sn;
                            dkj[e0 + 1] = -g2[e0] * sn + g2[e0 + 1] * c;
                            if (my_drope) my_drope[half * (d / 4) + t] +=
                                (double)pos[half] * (g2[e0] * -kj[e0 + 1] + g2[e0 + 1] * kj[e0]);
                        }
                } else {
                    for (int e = 0; e < d; ++e) dkj[e] = g2[e];
                }
            }
        }
#pragma omp critical
        {
            if (my_dtable) for (size_t i = 0; i < (size_t)R * R * heads; ++i) dtable[i] += my_dtable[i];
            if (my_dtau) for (int i = 0; i < heads; ++i) dtau[i] += my_dtau[i];
            if (my_drope) for (int i = 0; i < 2 * (d / 4); ++i) drope[i] += my_drope[i];
        }
        free(ky); free(kx); free(pw); free(cw); free(kr); free(qr); free(dkr); free(nrm); free(clamped); free(gq);
        free(my_dtable); free(my_dtau); free(my_drope);
    }
    return 0;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
