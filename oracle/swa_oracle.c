/*
 * swa_oracle.c -- plain fp64 CPU oracle of the causal sliding-window attention layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may include, link, load or call
 * this file; only the tests, the smoke check and the benchmark's CPU-baseline leg use it.
 * It shares no code with the CUDA library.
 *
 * What it computes, in the order the pages state it, one query row at a time:
 *
 *   1. RoPE on q and k  (intelliparadigm "GPT-2 for $73", section 2.2, the QK-norm snippet
 *      "q, k = normalize(apply_rope(q)), normalize(apply_rope(k))"; kongchang speedrun explainer,
 *      "RoPE" paragraph: rotation matrices that make scores depend on relative position).
 *      Reading taken where the pages are silent: pairs are (i, i + D/2) for i < D/2, the
 *      frequency of pair i is theta_i = base^(-2i/D), and position t rotates the pair
 *      (a, b) -> (a cos(t theta_i) - b sin(t theta_i), a sin(t theta_i) + b cos(t theta_i)).
 *      Angles and their cos/sin are taken in fp64.
 *   2. Parameter-free RMS normalisation after RoPE (same section 2.1/2.2: RMSNorm with no
 *      gamma/beta; PaperWeekly repost, "QK Normalization ... after RoPE"):
 *      xhat = x / sqrt(mean_D(x^2) + eps).
 *   3. Gated value embedding on VE layers (PaperWeekly repost, "Value Embeddings"
 *      paragraph: ve = value_embeds[layer](token_ids); gate = 2*sigmoid(ve_gate(x[:, :, :32]));
 *      v = v + gate*ve).  Reading: ve_gate is a bias-free linear map Wg [32, H], one gate per
 *      head, broadcast over D.  This oracle does its own lookup ve = table[ids].
 *   4. Scaled dot-product attention with the causal mask including the diagonal ("Let's
 *      reproduce GPT-2 (124M)" notes, section 3, the attention listing and the paragraph on
 *      the lower-triangular mask): s_j = qhat_i . khat_j / sqrt(D), softmax over the visible
 *      keys, out_i = sum_j p_j v'_j.  The window (intelliparadigm section 3.2, "local window
 *      (1024 tokens)") is read as W keys including the query itself: key j is visible to
 *      query i iff 0 <= i - j < W; window <= 0 or >= T means full causal.
 *   5. The log-sum-exp of the scaled scores per row (natural log): lse_i = M + ln(sum exp(s - M)).
 *
 * Nothing is blocked, fused or reordered beyond this definition.  The only parallelism is
 * an OpenMP split over independent (position) and (query row) indices.
 *
 * Parity mode (round_bf16 = 1) rounds qhat, khat and v' to bf16 (round to nearest even)
 * after the fp64 prologue, because the tensor-core operands of the GPU path are bf16; the
 * attention itself stays fp64.  Pure mode (round_bf16 = 0) is fp64 throughout.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* bf16 bit pattern -> double, exactly (bf16 is the top half of an IEEE binary32). */
static double bf16_to_double(uint16_t h) {
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* double -> nearest bf16 value (ties to even), returned as a double.  bf16 keeps 8
 * significant bits; frexp gives x = m * 2^e with 0.5 <= |m| < 1, so m * 2^8 lies in
 * [128, 256) and rounding it to an integer in the current (nearest-even) mode rounds x to
 * 8 significant bits in one step, with no intermediate float rounding. */
static double round_to_bf16(double x) {
    if (x == 0.0 || !isfinite(x)) return x;
    int e;
    double m = frexp(x, &e);
    double r = nearbyint(ldexp(m, 8));
    return ldexp(r, e - 8);
}

static void rope_inplace(double* x, int D, int t, double base) {
    const int half = D / 2;
    for (int i = 0; i < half; ++i) {
        double theta = pow(base, -2.0 * (double)i / (double)D);
        double ang = (double)t * theta;
        double c = cos(ang), s = sin(ang);
        double a = x[i], b = x[i + half];
        x[i] = a * c - b * s;
        x[i + half] = a * s + b * c;
    }
}

static void rmsnorm_inplace(double* x, int D, double eps) {
    double ss = 0.0;
    for (int d = 0; d < D; ++d) ss += x[d] * x[d];
    double r = 1.0 / sqrt(ss / (double)D + eps);
    for (int d = 0; d < D; ++d) x[d] *= r;
}

/* q or k row (b, t, h) -> qhat/khat in out[D]. */
static void prologue_qk(const uint16_t* src, int T, int H, int D, int b, int t, int h,
                        double base, double eps, int use_rope, int use_qknorm, int round_bf16,
                        double* out) {
    const uint16_t* row = src + (((size_t)b * T + t) * H + h) * (size_t)D;
    for (int d = 0; d < D; ++d) out[d] = bf16_to_double(row[d]);
    if (use_rope) rope_inplace(out, D, t, base);
    if (use_qknorm) rmsnorm_inplace(out, D, eps);
    if (round_bf16)
        for (int d = 0; d < D; ++d) out[d] = round_to_bf16(out[d]);
}

/* v row (b, t, h) -> v' = v + 2 sigmoid(x[b,t,:32] . Wg[:, h]) * table[ids[b,t], h*D:(h+1)*D]. */
static void prologue_v(const uint16_t* v, const int64_t* ids, const uint16_t* table,
                       const uint16_t* x, int C, const uint16_t* Wg,
                       int T, int H, int D, int b, int t, int h, int round_bf16, double* out) {
    const uint16_t* row = v + (((size_t)b * T + t) * H + h) * (size_t)D;
    for (int d = 0; d < D; ++d) out[d] = bf16_to_double(row[d]);
    if (ids != NULL) {
        const uint16_t* xr = x + ((size_t)b * T + t) * (size_t)C;
        double z = 0.0;
        for (int c = 0; c < 32; ++c) z += bf16_to_double(xr[c]) * bf16_to_double(Wg[c * H + h]);
        double gate = 2.0 / (1.0 + exp(-z));
        int64_t id = ids[(size_t)b * T + t];
        const uint16_t* ve = table + (size_t)id * (size_t)H * D + (size_t)h * D;
        for (int d = 0; d < D; ++d) out[d] += gate * bf16_to_double(ve[d]);
    }
    if (round_bf16)
        for (int d = 0; d < D; ++d) out[d] = round_to_bf16(out[d]);
}

static int ids_in_range(const int64_t* ids, int64_t n, int vocab) {
    for (int64_t i = 0; i < n; ++i)
        if (ids[i] < 0 || ids[i] >= vocab) return 0;
    return 1;
}

static int visible(int i, int j, int W, int convention) {
    int diff = i - j;
    if (diff < 0) return 0;
    return convention == 0 ? (diff < W) : (diff <= W);
}

/* Key j is visible to query i: inside the causal window and, when document ids are given (doc_b,
 * the ids of this batch row), in the same document. */
static int visible_doc(int i, int j, int W, int convention, const int64_t* doc_b) {
    return visible(i, j, W, convention) && (doc_b == NULL || doc_b[j] == doc_b[i]);
}

/* One attention row: qhat_i against khat[0..T), v'[0..T) of one (b, h). */
static void attention_row(const double* qh, const double* kh, const double* vp, int T, int D,
                          int i, int W, int convention, const int64_t* doc_b, double* out,
                          double* lse, double* s) {
    const double scale = 1.0 / sqrt((double)D);
    double M = -INFINITY;
    for (int j = 0; j < T; ++j) {
        if (!visible_doc(i, j, W, convention, doc_b)) continue;
        double acc = 0.0;
        for (int d = 0; d < D; ++d) acc += qh[d] * kh[(size_t)j * D + d];
        s[j] = acc * scale;
        if (s[j] > M) M = s[j];
    }
    double L = 0.0;
    for (int j = 0; j < T; ++j)
        if (visible_doc(i, j, W, convention, doc_b)) L += exp(s[j] - M);
    for (int d = 0; d < D; ++d) out[d] = 0.0;
    for (int j = 0; j < T; ++j) {
        if (!visible_doc(i, j, W, convention, doc_b)) continue;
        double p = exp(s[j] - M) / L;
        for (int d = 0; d < D; ++d) out[d] += p * vp[(size_t)j * D + d];
    }
    *lse = M + log(L);
}

int swa_oracle_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * q             bf16 bit patterns, (B, T, H, D) contiguous: H query heads.
 * k, v          bf16 bit patterns, (B, T, Hkv, D): Hkv key/value heads, Hkv divides H; query head
 *               h reads key/value head h / (H / Hkv) (grouped-query attention; Hkv == H is the
 *               ordinary multi-head layer).
 * ids, table    VE token ids (B, T) and table [vocab, Hkv*D] bf16; ids == NULL means no VE.
 * x, C          x (B, T, C) bf16; the gate reads channels 0..31.
 * Wg            [32, Hkv] bf16.
 * window        <= 0 or >= T: full causal.
 * doc           (swa_oracle_forward_doc_gqa) document ids (B, T) or NULL: key j is visible to
 *               query i only if doc[b, j] == doc[b, i] as well (a document-boundary mask; RoPE
 *               positions stay the positions t in the sequence).
 * rows/n_rows   flat query ids ((b*H + h)*T + i), sorted ascending; rows == NULL: every row.
 * out           rows == NULL: (B, T, H, D) fp64; else [n_rows, D].
 * lse           rows == NULL: (B, H, T) fp64;   else [n_rows].
 * Returns 0, or -1 on bad arguments / allocation failure.
 */
int swa_oracle_forward_doc_gqa(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                               const int64_t* ids, const uint16_t* table, int vocab,
                               const uint16_t* x, int C, const uint16_t* Wg,
                               int B, int T, int H, int Hkv, int D, int window, double rope_base,
                               double eps, int round_bf16, int use_rope, int use_qknorm,
                               int window_convention, const int64_t* doc, const int64_t* rows,
                               int64_t n_rows, double* out, double* lse) {
    if (B < 1 || T < 1 || H < 1 || D < 2 || (D % 2) != 0) return -1;
    if (Hkv < 1 || Hkv > H || (H % Hkv) != 0) return -1;
    const int G = H / Hkv;
    if (ids != NULL && (table == NULL || x == NULL || Wg == NULL || C < 32 || vocab < 1)) return -1;
    if (ids != NULL && !ids_in_range(ids, (int64_t)B * T, vocab)) return -1;
    const int W = (window <= 0 || window >= T) ? T : window;
    const int64_t total_rows = (int64_t)B * H * T;
    if (rows == NULL) n_rows = total_rows;

    double* kh = (double*)malloc(sizeof(double) * (size_t)T * D);
    double* vp = (double*)malloc(sizeof(double) * (size_t)T * D);
    if (!kh || !vp) { free(kh); free(vp); return -1; }
    int rc = 0;

    int64_t r0 = 0;
    while (r0 < n_rows) {
        /* The run of requested rows that share one (b, h). */
        int64_t id0 = rows ? rows[r0] : r0;
        if (id0 < 0 || id0 >= total_rows) { rc = -1; break; }
        int64_t bh = id0 / T;
        int64_t r1 = r0 + 1;
        while (r1 < n_rows && (rows ? rows[r1] : r1) / T == bh) ++r1;
        const int b = (int)(bh / H), h = (int)(bh % H);
        const int hk = h / G;                       /* this query head's key/value head */

        #pragma omp parallel for schedule(static)
        for (int t = 0; t < T; ++t) {
            prologue_qk(k, T, Hkv, D, b, t, hk, rope_base, eps, use_rope, use_qknorm, round_bf16,
                        kh + (size_t)t * D);
            prologue_v(v, ids, table, x, C, Wg, T, Hkv, D, b, t, hk, round_bf16, vp + (size_t)t * D);
        }

        int bad = 0;
        #pragma omp parallel
        {
            double* qh = (double*)malloc(sizeof(double) * (size_t)D);
            double* s = (double*)malloc(sizeof(double) * (size_t)T);
            double* o = (double*)malloc(sizeof(double) * (size_t)D);
            const int ok = (qh != NULL && s != NULL && o != NULL);
            #pragma omp for schedule(dynamic, 16)
            for (int64_t r = r0; r < r1; ++r) {
                if (!ok) {
                    #pragma omp atomic write
                    bad = 1;
                    continue;
                }
                int64_t id = rows ? rows[r] : r;
                int i = (int)(id % T);
                double l;
                prologue_qk(q, T, H, D, b, i, h, rope_base, eps, use_rope, use_qknorm,
                            round_bf16, qh);
                attention_row(qh, kh, vp, T, D, i, W, window_convention,
                              doc ? doc + (size_t)b * T : NULL, o, &l, s);
                if (rows) {
                    memcpy(out + (size_t)r * D, o, sizeof(double) * (size_t)D);
                    lse[r] = l;
                } else {
                    memcpy(out + (((size_t)b * T + i) * H + h) * (size_t)D, o,
                           sizeof(double) * (size_t)D);
                    lse[((size_t)b * H + h) * T + i] = l;
                }
            }
            free(qh); free(s); free(o);
        }
        if (bad) { rc = -1; break; }
        r0 = r1;
    }
    free(kh); free(vp);
    return rc;
}

/* Without document ids: the causal window alone. */
int swa_oracle_forward_gqa(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                           const int64_t* ids, const uint16_t* table, int vocab,
                           const uint16_t* x, int C, const uint16_t* Wg,
                           int B, int T, int H, int Hkv, int D, int window, double rope_base,
                           double eps, int round_bf16, int use_rope, int use_qknorm,
                           int window_convention, const int64_t* rows, int64_t n_rows,
                           double* out, double* lse) {
    return swa_oracle_forward_doc_gqa(q, k, v, ids, table, vocab, x, C, Wg, B, T, H, Hkv, D, window,
                                      rope_base, eps, round_bf16, use_rope, use_qknorm,
                                      window_convention, NULL, rows, n_rows, out, lse);
}

/* The multi-head layer: every tensor has H heads. */
int swa_oracle_forward(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                       const int64_t* ids, const uint16_t* table, int vocab,
                       const uint16_t* x, int C, const uint16_t* Wg,
                       int B, int T, int H, int D, int window, double rope_base, double eps,
                       int round_bf16, int use_rope, int use_qknorm, int window_convention,
                       const int64_t* rows, int64_t n_rows, double* out, double* lse) {
    return swa_oracle_forward_gqa(q, k, v, ids, table, vocab, x, C, Wg, B, T, H, H, D, window,
                                  rope_base, eps, round_bf16, use_rope, use_qknorm,
                                  window_convention, rows, n_rows, out, lse);
}

/* The prologue alone, for the pins on RoPE / RMS / gate: qhat (B,T,H,D), khat and v'
 * (B,T,Hkv,D) as fp64. */
int swa_oracle_prologue_gqa(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                            const int64_t* ids, const uint16_t* table, int vocab,
                            const uint16_t* x, int C, const uint16_t* Wg,
                            int B, int T, int H, int Hkv, int D, double rope_base, double eps,
                            int round_bf16, int use_rope, int use_qknorm,
                            double* qh, double* kh, double* vp) {
    if (B < 1 || T < 1 || H < 1 || D < 2 || (D % 2) != 0) return -1;
    if (Hkv < 1 || Hkv > H || (H % Hkv) != 0) return -1;
    if (ids != NULL && (table == NULL || x == NULL || Wg == NULL || C < 32 || vocab < 1)) return -1;
    if (ids != NULL && !ids_in_range(ids, (int64_t)B * T, vocab)) return -1;
    #pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b)
        for (int t = 0; t < T; ++t) {
            for (int h = 0; h < H; ++h)
                prologue_qk(q, T, H, D, b, t, h, rope_base, eps, use_rope, use_qknorm, round_bf16,
                            qh + (((size_t)b * T + t) * H + h) * (size_t)D);
            for (int h = 0; h < Hkv; ++h) {
                size_t off = (((size_t)b * T + t) * Hkv + h) * (size_t)D;
                prologue_qk(k, T, Hkv, D, b, t, h, rope_base, eps, use_rope, use_qknorm, round_bf16, kh + off);
                prologue_v(v, ids, table, x, C, Wg, T, Hkv, D, b, t, h, round_bf16, vp + off);
            }
        }
    return 0;
}

int swa_oracle_prologue(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                        const int64_t* ids, const uint16_t* table, int vocab,
                        const uint16_t* x, int C, const uint16_t* Wg,
                        int B, int T, int H, int D, double rope_base, double eps,
                        int round_bf16, int use_rope, int use_qknorm,
                        double* qh, double* kh, double* vp) {
    return swa_oracle_prologue_gqa(q, k, v, ids, table, vocab, x, C, Wg, B, T, H, H, D, rope_base,
                                   eps, round_bf16, use_rope, use_qknorm, qh, kh, vp);
}

/* Exposed for the rounding pin: double -> bf16 value, ties to even. */
double swa_oracle_round_bf16(double x) { return round_to_bf16(x); }

/* -----------------------------------------------------------------------------------------
 * Backward: the gradient of the layer, for training.
 *
 * The pages train this layer (the speedrun explainer's attention section and the GPT-2
 * notes train end to end; the forward keeps the log-sum-exp so the backward can rebuild the
 * softmax).  The backward is the chain rule through the five forward steps above, taken in
 * reverse, for the scalar loss
 *
 *     loss = sum_{b,t,h,d} dout[b,t,h,d] * out[b,t,h,d] + sum_{b,h,t} dlse[b,h,t] * lse[b,h,t].
 *
 *   5/4. Attention.  For query row i with visible keys J: P_ij = exp(s_ij - lse_i),
 *        dP_ij = dout_i . v'_j, delta_i = sum_j P_ij dP_ij (the softmax Jacobian's rank-one
 *        term), dS_ij = P_ij (dP_ij - delta_i) + P_ij dlse_i (d lse_i / d s_ij = P_ij).
 *        Then dqhat_i = sum_j dS_ij khat_j / sqrt(D), dkhat_j = sum_i dS_ij qhat_i / sqrt(D),
 *        dv'_j = sum_i P_ij dout_i.  Under grouped-query attention the key/value gradients
 *        sum over the query heads that read the head.
 *   3.   Gate: v' = v + g ve with g = 2 sigma(z), z = sum_{c<32} x_c Wg[c, h]:
 *        dv = dv', dve = g dv', dz = (dv' . ve) * 2 sigma(z)(1 - sigma(z)),
 *        dx_c = sum_h dz_h Wg[c, h], dWg[c, h] = sum_{b,t} dz[b,t,h] x[b,t,c].
 *   2.   RMS: y = r x with r = (mean(x^2) + eps)^(-1/2); d r / d x_e = -r^3 x_e / D, so
 *        dx = r dy - (r^3 / D) (x . dy) x.
 *   1.   RoPE rotates each pair by +t theta_i; its transpose rotates by -t theta_i.
 *
 * Parity mode (round_bf16 = 1) recomputes qhat, khat, v' rounded to bf16 as the forward does
 * and passes the gradient straight through the rounding (it has no derivative); pure mode is
 * the exact gradient of the fp64 layer.
 * ----------------------------------------------------------------------------------------- */

/* The transpose of rope_inplace.  Rotation by -a equals F R(a) F with F = diag(1, -1) on each
 * pair, so the second half is negated around the forward rotation (negation is exact). */
static void rope_transpose_inplace(double* g, int D, int t, double base) {
    const int half = D / 2;
    for (int i = half; i < D; ++i) g[i] = -g[i];
    rope_inplace(g, D, t, base);
    for (int i = half; i < D; ++i) g[i] = -g[i];
}

/* dL/d(row of q or k) from dy = dL/d(qhat or khat) for row (b, t, h): rebuilds the rotated,
 * un-normalised row xr (scratch of D) and applies the RMS and RoPE steps in reverse. */
static void prologue_qk_backward(const uint16_t* src, int T, int H, int D, int b, int t, int h,
                                 double base, double eps, int use_rope, int use_qknorm,
                                 const double* dy, double* dx, double* xr) {
    const uint16_t* row = src + (((size_t)b * T + t) * H + h) * (size_t)D;
    for (int d = 0; d < D; ++d) xr[d] = bf16_to_double(row[d]);
    if (use_rope) rope_inplace(xr, D, t, base);
    if (use_qknorm) {
        double sq = 0.0, xdy = 0.0;
        for (int d = 0; d < D; ++d) {
            sq += xr[d] * xr[d];
            xdy += xr[d] * dy[d];
        }
        const double r = 1.0 / sqrt(sq / (double)D + eps);
        const double coef = r * r * r * xdy / (double)D;
        for (int d = 0; d < D; ++d) dx[d] = r * dy[d] - coef * xr[d];
    } else {
        for (int d = 0; d < D; ++d) dx[d] = dy[d];
    }
    if (use_rope) rope_transpose_inplace(dx, D, t, base);
}

static double dot_d(const double* a, const double* b, int D) {
    double acc = 0.0;
    for (int d = 0; d < D; ++d) acc += a[d] * b[d];
    return acc;
}

/* Keys j visible to query i are those with i in [j, j + reach]. */
static int key_reach(int W, int window_convention) {
    return window_convention == 0 ? W - 1 : W;
}

/* khat and v' of every position of key/value head hk of batch row b, as the forward computes
 * them (rounded to bf16 in parity mode). */
static void bwd_kv_prologue(const uint16_t* k, const uint16_t* v, const int64_t* ids,
                            const uint16_t* table, const uint16_t* x, int C, const uint16_t* Wg,
                            int T, int Hkv, int D, int b, int hk, double rope_base, double eps,
                            int round_bf16, int use_rope, int use_qknorm, double* kh, double* vp) {
    #pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t) {
        prologue_qk(k, T, Hkv, D, b, t, hk, rope_base, eps, use_rope, use_qknorm,
                    round_bf16, kh + (size_t)t * D);
        prologue_v(v, ids, table, x, C, Wg, T, Hkv, D, b, t, hk, round_bf16,
                   vp + (size_t)t * D);
    }
}

/* Row pass for query row i of one (b, h): scores against the visible keys (scratch s of T),
 * lse_i, delta_i = sum_j P_ij dP_ij and, if dqi is not NULL, dqhat_i = sum_j dS_ij khat_j / sqrt(D).
 * gi is dout of the row, gl its dlse; doc_b, if not NULL, the document ids of this batch row. */
static void bwd_query_row(const double* qi, const double* gi, double gl, const double* kh,
                          const double* vp, int T, int D, int i, int W, int window_convention,
                          const int64_t* doc_b, double inv_sqrt_d, double* s, double* lse_i,
                          double* delta_i, double* dqi) {
    double M = -INFINITY;
    for (int j = 0; j < T; ++j) {
        if (!visible_doc(i, j, W, window_convention, doc_b)) continue;
        s[j] = dot_d(qi, kh + (size_t)j * D, D) * inv_sqrt_d;
        if (s[j] > M) M = s[j];
    }
    double L = 0.0;
    for (int j = 0; j < T; ++j)
        if (visible_doc(i, j, W, window_convention, doc_b)) L += exp(s[j] - M);
    const double li = M + log(L);
    double dl = 0.0;
    for (int j = 0; j < T; ++j)
        if (visible_doc(i, j, W, window_convention, doc_b))
            dl += exp(s[j] - li) * dot_d(gi, vp + (size_t)j * D, D);
    *lse_i = li;
    *delta_i = dl;
    if (dqi == NULL) return;
    for (int d = 0; d < D; ++d) dqi[d] = 0.0;
    for (int j = 0; j < T; ++j) {
        if (!visible_doc(i, j, W, window_convention, doc_b)) continue;
        const double p = exp(s[j] - li);
        const double ds = p * (dot_d(gi, vp + (size_t)j * D, D) - dl) + p * gl;
        for (int d = 0; d < D; ++d) dqi[d] += ds * kh[(size_t)j * D + d] * inv_sqrt_d;
    }
}

/* Key pass for key row j of one (b, h): adds sum_i dS_ij qhat_i / sqrt(D) to dkj and
 * sum_i P_ij dout_i to dvj over the queries i in [j, i_end] that see key j (and, with document
 * ids, share its document).  qh, lse, delta are indexed by query position; dout / dlse are the
 * full tensors. */
static void bwd_key_row(const double* kj, const double* vj, const double* qh, const double* lse,
                        const double* delta, const double* dout, const double* dlse, int b, int h,
                        int T, int H, int D, int j, int i_end, const int64_t* doc_b,
                        double inv_sqrt_d, double* dkj, double* dvj) {
    for (int i = j; i <= i_end; ++i) {
        if (doc_b != NULL && doc_b[i] != doc_b[j]) continue;    /* another document */
        const double* qi = qh + (size_t)i * D;
        const double* gi = dout + (((size_t)b * T + i) * H + h) * (size_t)D;
        const double gl = dlse ? dlse[((size_t)b * H + h) * T + i] : 0.0;
        const double p = exp(dot_d(qi, kj, D) * inv_sqrt_d - lse[i]);
        const double ds = p * (dot_d(gi, vj, D) - delta[i]) + p * gl;
        for (int d = 0; d < D; ++d) {
            dkj[d] += ds * qi[d] * inv_sqrt_d;
            dvj[d] += p * gi[d];
        }
    }
}

/* dk, dv (and on value-embedding layers dve and dz) of key/value row (b, t, hk) from its dkhat and
 * dv'.  dk_out / dv_out / dve_out receive D values; *dz_out the gate-logit gradient. */
static void bwd_kv_outputs(const uint16_t* k, const int64_t* ids, const uint16_t* table,
                           const uint16_t* x, int C, const uint16_t* Wg, int T, int Hkv, int D,
                           int b, int t, int hk, double rope_base, double eps, int use_rope,
                           int use_qknorm, const double* dkt, const double* dvt, double* dk_out,
                           double* dv_out, double* dve_out, double* dz_out, double* xr) {
    prologue_qk_backward(k, T, Hkv, D, b, t, hk, rope_base, eps, use_rope, use_qknorm, dkt, dk_out, xr);
    for (int d = 0; d < D; ++d) dv_out[d] = dvt[d];
    if (ids == NULL) return;
    const uint16_t* xt = x + ((size_t)b * T + t) * (size_t)C;
    double z = 0.0;
    for (int c = 0; c < 32; ++c)
        z += bf16_to_double(xt[c]) * bf16_to_double(Wg[(size_t)c * Hkv + hk]);
    const double sig = 1.0 / (1.0 + exp(-z));
    const int64_t id = ids[(size_t)b * T + t];
    const uint16_t* ve = table + (size_t)id * (size_t)Hkv * D + (size_t)hk * D;
    double dgate = 0.0;
    for (int d = 0; d < D; ++d) {
        dve_out[d] = 2.0 * sig * dvt[d];
        dgate += dvt[d] * bf16_to_double(ve[d]);
    }
    *dz_out = dgate * 2.0 * sig * (1.0 - sig);
}

/*
 * Inputs as swa_oracle_forward_gqa, plus
 *   dout   fp64 (B, T, H, D): dL/d out.
 *   dlse   fp64 (B, H, T):    dL/d lse, or NULL for zero.
 * Outputs (fp64, written in full):
 *   dq            (B, T, H, D)
 *   dk, dv        (B, T, Hkv, D)
 *   dve           (B, T, Hkv, D): dL/d(the looked-up value-embedding row at (b, t)); the table's
 *                 gradient is its scatter-add over ids.  VE layers only (NULL otherwise).
 *   dx            (B, T, 32): dL/d x[b, t, c] for the 32 gate channels (channels >= 32 do not
 *                 reach the layer).  VE layers only.
 *   dWg           [32, Hkv].  VE layers only.
 *   doc           (swa_oracle_backward_doc_gqa) document ids (B, T) or NULL, as in the forward.
 * Returns 0, or -1 on bad arguments / allocation failure.
 */
int swa_oracle_backward_doc_gqa(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                const int64_t* ids, const uint16_t* table, int vocab,
                                const uint16_t* x, int C, const uint16_t* Wg,
                                int B, int T, int H, int Hkv, int D, int window, double rope_base,
                                double eps, int round_bf16, int use_rope, int use_qknorm,
                                int window_convention, const int64_t* doc, const double* dout,
                                const double* dlse, double* dq, double* dk, double* dv, double* dve,
                                double* dx, double* dWg) {
    if (B < 1 || T < 1 || H < 1 || D < 2 || (D % 2) != 0) return -1;
    if (Hkv < 1 || Hkv > H || (H % Hkv) != 0) return -1;
    if (dout == NULL || dq == NULL || dk == NULL || dv == NULL) return -1;
    if (ids != NULL && (table == NULL || x == NULL || Wg == NULL || C < 32 || vocab < 1)) return -1;
    if (ids != NULL && (dve == NULL || dx == NULL || dWg == NULL)) return -1;
    if (ids != NULL && !ids_in_range(ids, (int64_t)B * T, vocab)) return -1;
    const int G = H / Hkv;
    const int W = (window <= 0 || window >= T) ? T : window;
    const int reach = key_reach(W, window_convention);
    const double inv_sqrt_d = 1.0 / sqrt((double)D);
    const size_t TD = (size_t)T * D;

    double* kh = (double*)malloc(sizeof(double) * TD);
    double* vp = (double*)malloc(sizeof(double) * TD);
    double* qh = (double*)malloc(sizeof(double) * TD);
    double* dkh = (double*)malloc(sizeof(double) * TD);
    double* dvp = (double*)malloc(sizeof(double) * TD);
    double* dqh = (double*)malloc(sizeof(double) * TD);
    double* lse = (double*)malloc(sizeof(double) * (size_t)T);
    double* delta = (double*)malloc(sizeof(double) * (size_t)T);
    double* dz = (double*)calloc((size_t)B * T * Hkv, sizeof(double));
    int rc = 0;
    if (!kh || !vp || !qh || !dkh || !dvp || !dqh || !lse || !delta || !dz) { rc = -1; goto done; }

    for (int b = 0; b < B && rc == 0; ++b) {
        for (int hk = 0; hk < Hkv && rc == 0; ++hk) {
            bwd_kv_prologue(k, v, ids, table, x, C, Wg, T, Hkv, D, b, hk, rope_base, eps, round_bf16,
                            use_rope, use_qknorm, kh, vp);
            memset(dkh, 0, sizeof(double) * TD);
            memset(dvp, 0, sizeof(double) * TD);

            for (int g = 0; g < G; ++g) {
                const int h = hk * G + g;
                #pragma omp parallel for schedule(static)
                for (int i = 0; i < T; ++i)
                    prologue_qk(q, T, H, D, b, i, h, rope_base, eps, use_rope, use_qknorm,
                                round_bf16, qh + (size_t)i * D);

                /* Row pass: lse_i, delta_i and dqhat_i, one query row at a time. */
                int bad = 0;
                #pragma omp parallel
                {
                    double* s = (double*)malloc(sizeof(double) * (size_t)T);
                    #pragma omp for schedule(dynamic, 8)
                    for (int i = 0; i < T; ++i) {
                        if (s == NULL) {
                            #pragma omp atomic write
                            bad = 1;
                            continue;
                        }
                        const double* gi = dout + (((size_t)b * T + i) * H + h) * (size_t)D;
                        const double gl = dlse ? dlse[((size_t)b * H + h) * T + i] : 0.0;
                        bwd_query_row(qh + (size_t)i * D, gi, gl, kh, vp, T, D, i, W, window_convention,
                                      doc ? doc + (size_t)b * T : NULL, inv_sqrt_d, s, &lse[i], &delta[i],
                                      dqh + (size_t)i * D);
                    }
                    free(s);
                }
                if (bad) { rc = -1; break; }

                /* Key pass: dkhat_j and dv'_j, one key row at a time, over the queries that
                 * see key j. */
                #pragma omp parallel for schedule(dynamic, 8)
                for (int j = 0; j < T; ++j) {
                    const int i_end = (j + reach < T - 1) ? j + reach : T - 1;
                    bwd_key_row(kh + (size_t)j * D, vp + (size_t)j * D, qh, lse, delta, dout, dlse, b, h,
                                T, H, D, j, i_end, doc ? doc + (size_t)b * T : NULL, inv_sqrt_d,
                                dkh + (size_t)j * D, dvp + (size_t)j * D);
                }

                /* dq rows of head h. */
                #pragma omp parallel
                {
                    double* xr = (double*)malloc(sizeof(double) * (size_t)D);
                    #pragma omp for schedule(static)
                    for (int i = 0; i < T; ++i) {
                        if (xr == NULL) {
                            #pragma omp atomic write
                            bad = 1;
                            continue;
                        }
                        prologue_qk_backward(q, T, H, D, b, i, h, rope_base, eps, use_rope,
                                             use_qknorm, dqh + (size_t)i * D,
                                             dq + (((size_t)b * T + i) * H + h) * (size_t)D, xr);
                    }
                    free(xr);
                }
                if (bad) { rc = -1; break; }
            }
            if (rc != 0) break;

            /* dk, dv and the gate of key/value head hk. */
            int bad = 0;
            #pragma omp parallel
            {
                double* xr = (double*)malloc(sizeof(double) * (size_t)D);
                #pragma omp for schedule(static)
                for (int t = 0; t < T; ++t) {
                    if (xr == NULL) {
                        #pragma omp atomic write
                        bad = 1;
                        continue;
                    }
                    const size_t off = (((size_t)b * T + t) * Hkv + hk) * (size_t)D;
                    double dzt = 0.0;
                    bwd_kv_outputs(k, ids, table, x, C, Wg, T, Hkv, D, b, t, hk, rope_base, eps, use_rope,
                                   use_qknorm, dkh + (size_t)t * D, dvp + (size_t)t * D, dk + off, dv + off,
                                   ids ? dve + off : NULL, &dzt, xr);
                    if (ids != NULL) dz[((size_t)b * T + t) * Hkv + hk] = dzt;
                }
                free(xr);
            }
            if (bad) rc = -1;
        }
    }

    if (rc == 0 && ids != NULL) {
        /* Gate inputs and weights from dz: dx sums over heads, dWg over positions. */
        #pragma omp parallel for schedule(static)
        for (int64_t bt = 0; bt < (int64_t)B * T; ++bt)
            for (int c = 0; c < 32; ++c) {
                double acc = 0.0;
                for (int hk = 0; hk < Hkv; ++hk)
                    acc += dz[(size_t)bt * Hkv + hk] * bf16_to_double(Wg[(size_t)c * Hkv + hk]);
                dx[(size_t)bt * 32 + c] = acc;
            }
        for (int c = 0; c < 32; ++c)
            for (int hk = 0; hk < Hkv; ++hk) {
                double acc = 0.0;
                for (int64_t bt = 0; bt < (int64_t)B * T; ++bt)
                    acc += dz[(size_t)bt * Hkv + hk] * bf16_to_double(x[(size_t)bt * C + c]);
                dWg[(size_t)c * Hkv + hk] = acc;
            }
    }

done:
    free(kh); free(vp); free(qh); free(dkh); free(dvp); free(dqh); free(lse); free(delta); free(dz);
    return rc;
}

/*
 * The same gradient at sampled rows only, for checks at sizes where the full backward is too slow:
 *   qrows[n_q]  flat query ids ((b*H + h)*T + i): dq of those rows -> dq_rows [n_q, D];
 *   krows[n_k]  flat key/value ids ((b*Hkv + hk)*T + j): dk, dv (and dve on value-embedding
 *               layers) of those rows -> dk_rows, dv_rows, dve_rows [n_k, D].
 * Each requested value is computed by the same helpers, in the same order, as in
 * swa_oracle_backward_gqa, from the query rows it depends on (those of its own row, or, for a
 * key row j, the queries in [j, j + W - 1] of every query head of its group), so it equals the full
 * backward's value bit for bit.  Returns 0, or -1 on bad arguments / allocation failure.
 */
/* Without document ids: the causal window alone. */
int swa_oracle_backward_gqa(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                            const int64_t* ids, const uint16_t* table, int vocab,
                            const uint16_t* x, int C, const uint16_t* Wg,
                            int B, int T, int H, int Hkv, int D, int window, double rope_base,
                            double eps, int round_bf16, int use_rope, int use_qknorm,
                            int window_convention, const double* dout, const double* dlse,
                            double* dq, double* dk, double* dv, double* dve, double* dx,
                            double* dWg) {
    return swa_oracle_backward_doc_gqa(q, k, v, ids, table, vocab, x, C, Wg, B, T, H, Hkv, D, window,
                                       rope_base, eps, round_bf16, use_rope, use_qknorm,
                                       window_convention, NULL, dout, dlse, dq, dk, dv, dve, dx, dWg);
}

int swa_oracle_backward_rows_gqa(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                 const int64_t* ids, const uint16_t* table, int vocab,
                                 const uint16_t* x, int C, const uint16_t* Wg,
                                 int B, int T, int H, int Hkv, int D, int window, double rope_base,
                                 double eps, int round_bf16, int use_rope, int use_qknorm,
                                 int window_convention, const double* dout, const double* dlse,
                                 const int64_t* qrows, int64_t n_q, double* dq_rows,
                                 const int64_t* krows, int64_t n_k, double* dk_rows,
                                 double* dv_rows, double* dve_rows) {
    if (B < 1 || T < 1 || H < 1 || D < 2 || (D % 2) != 0) return -1;
    if (Hkv < 1 || Hkv > H || (H % Hkv) != 0) return -1;
    if (dout == NULL || n_q < 0 || n_k < 0) return -1;
    if (n_q > 0 && (qrows == NULL || dq_rows == NULL)) return -1;
    if (n_k > 0 && (krows == NULL || dk_rows == NULL || dv_rows == NULL)) return -1;
    if (ids != NULL && (table == NULL || x == NULL || Wg == NULL || C < 32 || vocab < 1)) return -1;
    if (ids != NULL && n_k > 0 && dve_rows == NULL) return -1;
    if (ids != NULL && !ids_in_range(ids, (int64_t)B * T, vocab)) return -1;
    for (int64_t r = 0; r < n_q; ++r)
        if (qrows[r] < 0 || qrows[r] >= (int64_t)B * H * T) return -1;
    for (int64_t r = 0; r < n_k; ++r)
        if (krows[r] < 0 || krows[r] >= (int64_t)B * Hkv * T) return -1;
    const int G = H / Hkv;
    const int W = (window <= 0 || window >= T) ? T : window;
    const int reach = key_reach(W, window_convention);
    const double inv_sqrt_d = 1.0 / sqrt((double)D);
    const size_t TD = (size_t)T * D;

    double* kh = (double*)malloc(sizeof(double) * TD);
    double* vp = (double*)malloc(sizeof(double) * TD);
    double* qh = (double*)malloc(sizeof(double) * TD);
    double* dkh = (double*)malloc(sizeof(double) * TD);
    double* dvp = (double*)malloc(sizeof(double) * TD);
    double* dqh = (double*)malloc(sizeof(double) * TD);
    double* lse = (double*)malloc(sizeof(double) * (size_t)T);
    double* delta = (double*)malloc(sizeof(double) * (size_t)T);
    char* need = (char*)malloc((size_t)T);       /* 1: lse/delta needed; 2: dqhat needed too */
    char* kneed = (char*)malloc((size_t)T);      /* requested key rows of this (b, hk) */
    int rc = 0;
    if (!kh || !vp || !qh || !dkh || !dvp || !dqh || !lse || !delta || !need || !kneed) { rc = -1; goto done; }

    for (int b = 0; b < B && rc == 0; ++b) {
        for (int hk = 0; hk < Hkv && rc == 0; ++hk) {
            int any = 0;
            memset(kneed, 0, (size_t)T);
            for (int64_t r = 0; r < n_k; ++r)
                if (krows[r] / T == (int64_t)b * Hkv + hk) { kneed[krows[r] % T] = 1; any = 1; }
            for (int64_t r = 0; r < n_q && !any; ++r) {
                const int64_t bh = qrows[r] / T;
                if (bh / H == b && (int)(bh % H) / G == hk) any = 1;
            }
            if (!any) continue;
            bwd_kv_prologue(k, v, ids, table, x, C, Wg, T, Hkv, D, b, hk, rope_base, eps, round_bf16,
                            use_rope, use_qknorm, kh, vp);
            memset(dkh, 0, sizeof(double) * TD);
            memset(dvp, 0, sizeof(double) * TD);
            for (int g = 0; g < G; ++g) {
                const int h = hk * G + g;
                memset(need, 0, (size_t)T);
                int any_h = 0;
                for (int64_t r = 0; r < n_q; ++r)
                    if (qrows[r] / T == (int64_t)b * H + h) { need[qrows[r] % T] = 2; any_h = 1; }
                for (int j = 0; j < T; ++j) {
                    if (!kneed[j]) continue;
                    const int i_end = (j + reach < T - 1) ? j + reach : T - 1;
                    for (int i = j; i <= i_end; ++i)
                        if (need[i] == 0) need[i] = 1;
                    any_h = 1;
                }
                if (!any_h) continue;
                int bad = 0;
                #pragma omp parallel
                {
                    double* s = (double*)malloc(sizeof(double) * (size_t)T);
                    #pragma omp for schedule(dynamic, 8)
                    for (int i = 0; i < T; ++i) {
                        if (!need[i]) continue;
                        if (s == NULL) {
                            #pragma omp atomic write
                            bad = 1;
                            continue;
                        }
                        prologue_qk(q, T, H, D, b, i, h, rope_base, eps, use_rope, use_qknorm,
                                    round_bf16, qh + (size_t)i * D);
                        const double* gi = dout + (((size_t)b * T + i) * H + h) * (size_t)D;
                        const double gl = dlse ? dlse[((size_t)b * H + h) * T + i] : 0.0;
                        bwd_query_row(qh + (size_t)i * D, gi, gl, kh, vp, T, D, i, W, window_convention,
                                      NULL, inv_sqrt_d, s, &lse[i], &delta[i],
                                      need[i] == 2 ? dqh + (size_t)i * D : NULL);
                    }
                    free(s);
                }
                if (bad) { rc = -1; break; }
                #pragma omp parallel for schedule(dynamic, 1)
                for (int j = 0; j < T; ++j) {
                    if (!kneed[j]) continue;
                    const int i_end = (j + reach < T - 1) ? j + reach : T - 1;
                    bwd_key_row(kh + (size_t)j * D, vp + (size_t)j * D, qh, lse, delta, dout, dlse, b, h,
                                T, H, D, j, i_end, NULL, inv_sqrt_d, dkh + (size_t)j * D, dvp + (size_t)j * D);
                }
                double* xr = (double*)malloc(sizeof(double) * (size_t)D);
                if (xr == NULL) { rc = -1; break; }
                for (int64_t r = 0; r < n_q; ++r)
                    if (qrows[r] / T == (int64_t)b * H + h) {
                        const int i = (int)(qrows[r] % T);
                        prologue_qk_backward(q, T, H, D, b, i, h, rope_base, eps, use_rope, use_qknorm,
                                             dqh + (size_t)i * D, dq_rows + (size_t)r * D, xr);
                    }
                free(xr);
            }
            if (rc != 0) break;
            double* xr = (double*)malloc(sizeof(double) * (size_t)D);
            if (xr == NULL) { rc = -1; break; }
            for (int64_t r = 0; r < n_k; ++r) {
                if (krows[r] / T != (int64_t)b * Hkv + hk) continue;
                const int j = (int)(krows[r] % T);
                double dzj = 0.0;
                bwd_kv_outputs(k, ids, table, x, C, Wg, T, Hkv, D, b, j, hk, rope_base, eps, use_rope,
                               use_qknorm, dkh + (size_t)j * D, dvp + (size_t)j * D, dk_rows + (size_t)r * D,
                               dv_rows + (size_t)r * D, ids ? dve_rows + (size_t)r * D : NULL, &dzj, xr);
            }
            free(xr);
        }
    }

done:
    free(kh); free(vp); free(qh); free(dkh); free(dvp); free(dqh); free(lse); free(delta);
    free(need); free(kneed);
    return rc;
}

/* -----------------------------------------------------------------------------------------
 * The projection before the path, fused with the prologue: q, k, v = x Wqkv^T, then RoPE, RMS and
 * the value-embedding gate as above.
 *
 * The pages build q, k, v of each layer with bias-free linear maps of the layer input x ("Let's
 * reproduce GPT-2 (124M)" notes, section 3, the attention listing: one projection to 3C split
 * into q, k, v; the speedrun explainer and intelliparadigm "GPT-2 for $73", section 2: separate
 * bias-free q, k, v maps, key/value width kv_dim).  Reading: one weight in the linear layer's
 * layout, Wqkv [(H + 2 Hkv) D, C] (rows 0 .. H D - 1 give q, then Hkv D rows of k, then Hkv D of
 * v), y[n] = sum_c x[c] Wqkv[n, c] summed in fp64 over c in order; the gate reads the first 32
 * channels of the same x.  Outputs as swa_oracle_prologue_gqa: qhat (B,T,H,D), khat and v'
 * (B,T,Hkv,D) in fp64, rounded to bf16 in parity mode.
 * ----------------------------------------------------------------------------------------- */

/* x[b,t,:] . Wqkv[n,:] in fp64, c in order. */
static double proj_dot(const uint16_t* xr, const uint16_t* Wqkv, int C, int n) {
    const uint16_t* w = Wqkv + (size_t)n * C;
    double acc = 0.0;
    for (int c = 0; c < C; ++c) acc += bf16_to_double(xr[c]) * bf16_to_double(w[c]);
    return acc;
}

int swa_oracle_qkv_prologue_gqa(const uint16_t* x, int C, const uint16_t* Wqkv,
                                const int64_t* ids, const uint16_t* table, int vocab,
                                const uint16_t* Wg, int B, int T, int H, int Hkv, int D,
                                double rope_base, double eps, int round_bf16, int use_rope,
                                int use_qknorm, double* qh, double* kh, double* vp) {
    if (B < 1 || T < 1 || H < 1 || D < 2 || (D % 2) != 0 || C < 1 || x == NULL || Wqkv == NULL) return -1;
    if (Hkv < 1 || Hkv > H || (H % Hkv) != 0) return -1;
    if (ids != NULL && (table == NULL || Wg == NULL || C < 32 || vocab < 1)) return -1;
    if (ids != NULL && !ids_in_range(ids, (int64_t)B * T, vocab)) return -1;
    int bad = 0;
    #pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b)
        for (int t = 0; t < T; ++t) {
            const uint16_t* xr = x + ((size_t)b * T + t) * (size_t)C;
            double* row = (double*)malloc(sizeof(double) * (size_t)D);
            if (row == NULL) {
                #pragma omp atomic write
                bad = 1;
                continue;
            }
            /* q heads, then k heads: projection, RoPE, RMS */
            for (int part = 0; part < 2; ++part) {
                const int heads = part == 0 ? H : Hkv;
                const int n0 = part == 0 ? 0 : H * D;
                double* dst = part == 0 ? qh : kh;
                for (int h = 0; h < heads; ++h) {
                    for (int d = 0; d < D; ++d) row[d] = proj_dot(xr, Wqkv, C, n0 + h * D + d);
                    if (use_rope) rope_inplace(row, D, t, rope_base);
                    if (use_qknorm) rmsnorm_inplace(row, D, eps);
                    double* o = dst + (((size_t)b * T + t) * heads + h) * (size_t)D;
                    for (int d = 0; d < D; ++d) o[d] = round_bf16 ? round_to_bf16(row[d]) : row[d];
                }
            }
            /* v heads: projection plus the gated value embedding */
            for (int h = 0; h < Hkv; ++h) {
                double gate = 0.0;
                const uint16_t* ve = NULL;
                if (ids != NULL) {
                    double z = 0.0;
                    for (int c = 0; c < 32; ++c) z += bf16_to_double(xr[c]) * bf16_to_double(Wg[c * Hkv + h]);
                    gate = 2.0 / (1.0 + exp(-z));
                    ve = table + (size_t)ids[(size_t)b * T + t] * (size_t)Hkv * D + (size_t)h * D;
                }
                double* o = vp + (((size_t)b * T + t) * Hkv + h) * (size_t)D;
                for (int d = 0; d < D; ++d) {
                    double val = proj_dot(xr, Wqkv, C, (H + Hkv) * D + h * D + d);
                    if (ve != NULL) val += gate * bf16_to_double(ve[d]);
                    o[d] = round_bf16 ? round_to_bf16(val) : val;
                }
            }
            free(row);
        }
    return bad ? -1 : 0;
}
