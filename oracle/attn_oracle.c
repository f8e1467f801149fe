/*
 * attn_oracle.c -- plain, slow, fp64 CPU attention.  TEST INFRASTRUCTURE ONLY.
 *
 * This file is the correctness oracle for the CUDA library in
 * io_aware_exact_flashattention_b200/.  Only the test suite, the package's
 * smoke check and the benchmark's CPU-baseline leg may load it.  It shares no
 * code, header, table or helper with the CUDA path, and the CUDA path never
 * calls it.
 *
 * What it computes is the textbook ("naive", materialising) attention that the
 * pages set against FlashAttention:
 *   - "I/O-Aware Kernels", section "The Memory Bottleneck": scores Q K^T, a
 *     softmax over each row of the k x k score matrix, then the product with V.
 *   - "FlashAttention & IO-aware attention", section "Code": the score of a
 *     query/key pair is their dot product divided by sqrt(d) (here: times the
 *     caller's `scale`, which the configurations set to 1/sqrt(d)).
 *   - Same page, section "Direct answer": the streamed (online) softmax is the
 *     exact one-shot softmax, so the one-shot form below is the definition the
 *     fused kernel must reproduce up to rounding.
 *
 * For every query row the whole score row is materialised in fp64, its maximum
 * M taken, Z = sum_j exp(s_j - M) formed, and
 *     LSE = M + ln Z,        O = sum_j exp(s_j - LSE) * v_j.
 * There is no blocking, no online recurrence and no reordering beyond that.
 *
 * Readings of points the pages leave open (the pages never mention a causal
 * mask or grouped-query head sharing beyond naming GQA):
 *   - causal: key j is visible to query i when j <= i + (Skv - Sq)
 *     (bottom-right alignment; equals j <= i when Sq == Skv).  Masked keys are
 *     excluded exactly.  A row with no visible key has O = 0 and LSE = -inf.
 *   - GQA: query head h reads key/value head h / (Hq / Hkv).
 *   - LSE is in natural-log units of the scaled scores.
 *
 * Layouts (row-major, contiguous): q/o [B,Hq,Sq,d], k/v [B,Hkv,Skv,d],
 * lse [B,Hq,Sq].  Decode: q/o [B,Hq,d], caches [B,Hkv,Lmax,d], seqlens [B].
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* Keys [0, n_vis) of one head against one query row.  s is scratch of >= n_vis
 * doubles.  Materialises the full score row (one-shot softmax). */
static void attn_one_row(const double *q, const double *k, const double *v,
                         int64_t n_vis, int d, double scale, double *s,
                         double *o, double *lse)
{
    if (n_vis <= 0) {
        for (int t = 0; t < d; ++t) o[t] = 0.0;
        *lse = -INFINITY;
        return;
    }
    double m = -INFINITY;
    for (int64_t j = 0; j < n_vis; ++j) {
        const double *kj = k + j * (int64_t)d;
        double acc = 0.0;
        for (int t = 0; t < d; ++t) acc += q[t] * kj[t];
        s[j] = scale * acc;
        if (s[j] > m) m = s[j];
    }
    double z = 0.0;
    for (int64_t j = 0; j < n_vis; ++j) z += exp(s[j] - m);
    const double l = m + log(z);
    for (int t = 0; t < d; ++t) o[t] = 0.0;
    for (int64_t j = 0; j < n_vis; ++j) {
        const double w = exp(s[j] - l);
        const double *vj = v + j * (int64_t)d;
        for (int t = 0; t < d; ++t) o[t] += w * vj[t];
    }
    *lse = l;
}

static int64_t visible_keys(int64_t i, int64_t Sq, int64_t Skv, int causal)
{
    if (!causal) return Skv;
    int64_t n = i + (Skv - Sq) + 1;
    if (n < 0) n = 0;
    if (n > Skv) n = Skv;
    return n;
}

/* Full forward pass.  Returns 0, or -1 on a bad argument. */
int oracle_attn_fwd(const double *q, const double *k, const double *v,
                    double *o, double *lse, int B, int Hq, int Hkv, int Sq,
                    int Skv, int d, int causal, double scale)
{
    if (B < 0 || Hq <= 0 || Hkv <= 0 || Sq < 0 || Skv < 0 || d <= 0) return -1;
    if (Hq % Hkv != 0) return -1;
    const int group = Hq / Hkv;
    const int64_t rows = (int64_t)B * Hq * Sq;
    int err = 0;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(Skv > 0 ? Skv : 1));
        if (!s) {
#pragma omp atomic write
            err = 1;
        } else {
#pragma omp for schedule(dynamic, 16)
            for (int64_t r = 0; r < rows; ++r) {
                const int64_t i = r % Sq;
                const int64_t bh = r / Sq;
                const int64_t h = bh % Hq;
                const int64_t b = bh / Hq;
                const int64_t g = h / group;
                const double *kh = k + ((b * Hkv + g) * (int64_t)Skv) * d;
                const double *vh = v + ((b * Hkv + g) * (int64_t)Skv) * d;
                attn_one_row(q + r * d, kh, vh, visible_keys(i, Sq, Skv, causal),
                             d, scale, s, o + r * d, lse + r);
            }
            free(s);
        }
    }
    return err ? -1 : 0;
}

/* Selected rows of the forward pass.  rows[3*n] holds (b, h, i) triples; the
 * outputs are o_rows[n, d] and lse_rows[n].  Used to check full-size launches
 * at sampled outputs. */
int oracle_attn_rows(const double *q_rows, const double *k, const double *v,
                     const int64_t *rows, int64_t n, double *o_rows,
                     double *lse_rows, int B, int Hq, int Hkv, int Sq, int Skv,
                     int d, int causal, double scale)
{
    if (Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || d <= 0) return -1;
    const int group = Hq / Hkv;
    int err = 0;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(Skv > 0 ? Skv : 1));
        if (!s) {
#pragma omp atomic write
            err = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t r = 0; r < n; ++r) {
                const int64_t b = rows[3 * r], h = rows[3 * r + 1], i = rows[3 * r + 2];
                if (b < 0 || b >= B || h < 0 || h >= Hq || i < 0 || i >= Sq) {
#pragma omp atomic write
                    err = 1;
                    continue;
                }
                const int64_t g = h / group;
                const double *kh = k + ((b * Hkv + g) * (int64_t)Skv) * d;
                const double *vh = v + ((b * Hkv + g) * (int64_t)Skv) * d;
                attn_one_row(q_rows + r * d, kh, vh, visible_keys(i, Sq, Skv, causal),
                             d, scale, s, o_rows + r * d, lse_rows + r);
            }
            free(s);
        }
    }
    return err ? -1 : 0;
}

/* Single-query decode: the forward pass with Sq = 1, no mask, and key count
 * seqlens[b] (positions >= seqlens[b] of the cache are never read).  This is
 * the 1 x S score vector of "FlashAttention & IO-aware attention", section
 * "Direct answer". */
int oracle_decode(const double *q, const double *kc, const double *vc,
                  const int32_t *seqlens, double *o, double *lse, int B, int Hq,
                  int Hkv, int Lmax, int d, double scale)
{
    if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || d <= 0 || Lmax < 0) return -1;
    for (int b = 0; b < B; ++b)
        if (seqlens[b] < 0 || seqlens[b] > Lmax) return -1;
    const int group = Hq / Hkv;
    int err = 0;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(Lmax > 0 ? Lmax : 1));
        if (!s) {
#pragma omp atomic write
            err = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t r = 0; r < (int64_t)B * Hq; ++r) {
                const int64_t b = r / Hq, h = r % Hq, g = h / group;
                const double *kh = kc + ((b * Hkv + g) * (int64_t)Lmax) * d;
                const double *vh = vc + ((b * Hkv + g) * (int64_t)Lmax) * d;
                attn_one_row(q + r * d, kh, vh, seqlens[b], d, scale, s, o + r * d, lse + r);
            }
            free(s);
        }
    }
    return err ? -1 : 0;
}

/* Split-KV partials of the decode step: the KV length of sequence b is cut
 * into num_splits chunks of ceil(L_b / num_splits) keys; chunk c covers
 * [c*cs, min(L_b, (c+1)*cs)).  For each chunk the one-shot softmax over that
 * chunk alone gives a normalised partial output and the chunk's LSE.  An
 * empty chunk has o = 0 and lse = -inf.  (Splitting the KV length across SMs
 * is the FlashDecoding idea named in "FlashAttention & IO-aware attention",
 * sections "Deep dive" and "Interviewer follow-ups".)
 * Outputs: o_part [B,Hq,num_splits,d], lse_part [B,Hq,num_splits]. */
int oracle_split_partials(const double *q, const double *kc, const double *vc,
                          const int32_t *seqlens, double *o_part, double *lse_part,
                          int B, int Hq, int Hkv, int Lmax, int d, int num_splits,
                          double scale)
{
    if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || d <= 0 || num_splits < 1) return -1;
    for (int b = 0; b < B; ++b)
        if (seqlens[b] < 0 || seqlens[b] > Lmax) return -1;
    const int group = Hq / Hkv;
    int err = 0;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(Lmax > 0 ? Lmax : 1));
        if (!s) {
#pragma omp atomic write
            err = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t r = 0; r < (int64_t)B * Hq * num_splits; ++r) {
                const int64_t c = r % num_splits;
                const int64_t bh = r / num_splits;
                const int64_t b = bh / Hq, h = bh % Hq, g = h / group;
                const int64_t L = seqlens[b];
                const int64_t cs = (L + num_splits - 1) / num_splits;
                int64_t lo = c * cs, hi = lo + cs;
                if (lo > L) lo = L;
                if (hi > L) hi = L;
                const double *kh = kc + ((b * Hkv + g) * (int64_t)Lmax + lo) * d;
                const double *vh = vc + ((b * Hkv + g) * (int64_t)Lmax + lo) * d;
                attn_one_row(q + bh * d, kh, vh, hi - lo, d, scale, s,
                             o_part + r * d, lse_part + r);
            }
            free(s);
        }
    }
    return err ? -1 : 0;
}

/* Split-KV partials with chunk boundaries on multiples of `align` keys:
 * cs = ceil(ceil(L_b / num_splits) / align) * align and chunk c covers
 * [c*cs, min(L_b, (c+1)*cs)); otherwise as oracle_split_partials (align = 1
 * is that function's rule).  A decode over a paged cache uses align = 128 so
 * that every 128-key tile of a chunk starts on a tile boundary.
 * Outputs: o_part [B,Hq,num_splits,d], lse_part [B,Hq,num_splits]. */
int oracle_split_partials_aligned(const double *q, const double *kc, const double *vc,
                                  const int32_t *seqlens, double *o_part, double *lse_part,
                                  int B, int Hq, int Hkv, int Lmax, int d, int num_splits,
                                  int align, double scale)
{
    if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || d <= 0 || num_splits < 1 ||
        align < 1)
        return -1;
    for (int b = 0; b < B; ++b)
        if (seqlens[b] < 0 || seqlens[b] > Lmax) return -1;
    const int group = Hq / Hkv;
    int err = 0;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(Lmax > 0 ? Lmax : 1));
        if (!s) {
#pragma omp atomic write
            err = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t r = 0; r < (int64_t)B * Hq * num_splits; ++r) {
                const int64_t c = r % num_splits;
                const int64_t bh = r / num_splits;
                const int64_t b = bh / Hq, h = bh % Hq, g = h / group;
                const int64_t L = seqlens[b];
                const int64_t cs0 = (L + num_splits - 1) / num_splits;
                const int64_t cs = (cs0 + align - 1) / align * align;
                int64_t lo = c * cs, hi = lo + cs;
                if (lo > L) lo = L;
                if (hi > L) hi = L;
                const double *kh = kc + ((b * Hkv + g) * (int64_t)Lmax + lo) * d;
                const double *vh = vc + ((b * Hkv + g) * (int64_t)Lmax + lo) * d;
                attn_one_row(q + bh * d, kh, vh, hi - lo, d, scale, s,
                             o_part + r * d, lse_part + r);
            }
            free(s);
        }
    }
    return err ? -1 : 0;
}

/* Merge of split partials.  With M = max_c lse_c the merged statistics are
 * LSE = M + ln sum_c exp(lse_c - M) and O = sum_c exp(lse_c - LSE) * o_c: the
 * e^(m - m_new) rescale rule of the online softmax ("FlashAttention &
 * IO-aware attention", section "Direct answer") applied between chunks.  All
 * chunks empty gives O = 0, LSE = -inf. */
int oracle_combine(const double *o_part, const double *lse_part, double *o,
                   double *lse, int B, int Hq, int num_splits, int d)
{
    if (B < 0 || Hq <= 0 || num_splits < 1 || d <= 0) return -1;
    for (int64_t r = 0; r < (int64_t)B * Hq; ++r) {
        const double *ls = lse_part + r * num_splits;
        double m = -INFINITY;
        for (int c = 0; c < num_splits; ++c)
            if (ls[c] > m) m = ls[c];
        double *orow = o + r * d;
        for (int t = 0; t < d; ++t) orow[t] = 0.0;
        if (m == -INFINITY) {
            lse[r] = -INFINITY;
            continue;
        }
        double z = 0.0;
        for (int c = 0; c < num_splits; ++c) z += exp(ls[c] - m);
        const double l = m + log(z);
        for (int c = 0; c < num_splits; ++c) {
            const double w = exp(ls[c] - l);
            const double *oc = o_part + (r * num_splits + c) * d;
            for (int t = 0; t < d; ++t) orow[t] += w * oc[t];
        }
        lse[r] = l;
    }
    return 0;
}

/* Gradients of the forward pass above for a loss L with dL/dO = dO.
 * "Tracing Tiled QKV Data Movement in FlashAttention's Memory Hierarchy"
 * (closing takeaways) notes that the backward pass recomputes the attention
 * matrix instead of storing it; the pages give no formulas, so this is the
 * derivative of the definition, written out with the full row materialised:
 *   P_ij  = exp(s_ij - LSE_i) over the visible keys,  s_ij = scale * q_i.k_j
 *   dP_ij = dO_i . v_j
 *   dS_ij = P_ij * (dP_ij - sum_l P_il dP_il)       (softmax Jacobian)
 *   dq_i  = scale * sum_j dS_ij k_j
 *   dk_j  = scale * sum_i dS_ij q_i   (over every query head of the group)
 *   dv_j  = sum_i P_ij dO_i           (likewise)
 * A row with no visible key contributes nothing.  Parallel over (b, kv head)
 * so each thread owns the dk/dv rows it accumulates.
 * Layouts: q, dO, dq [B,Hq,Sq,d]; k, v, dk, dv [B,Hkv,Skv,d]. */
int oracle_attn_bwd(const double *q, const double *k, const double *v, const double *dO,
                    double *dq, double *dk, double *dv, int B, int Hq, int Hkv, int Sq,
                    int Skv, int d, int causal, double scale)
{
    if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || Sq < 0 || Skv < 0 || d <= 0) return -1;
    const int group = Hq / Hkv;
    int err = 0;
#pragma omp parallel
    {
        double *p = (double *)malloc(sizeof(double) * (size_t)(Skv > 0 ? Skv : 1));
        double *dp = (double *)malloc(sizeof(double) * (size_t)(Skv > 0 ? Skv : 1));
        if (!p || !dp) {
#pragma omp atomic write
            err = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t bg = 0; bg < (int64_t)B * Hkv; ++bg) {
                const int64_t b = bg / Hkv, g = bg % Hkv;
                const double *kh = k + bg * (int64_t)Skv * d;
                const double *vh = v + bg * (int64_t)Skv * d;
                double *dkh = dk + bg * (int64_t)Skv * d;
                double *dvh = dv + bg * (int64_t)Skv * d;
                for (int64_t t = 0; t < (int64_t)Skv * d; ++t) { dkh[t] = 0.0; dvh[t] = 0.0; }
                for (int64_t h = g * group; h < (g + 1) * group; ++h) {
                    const int64_t bh = b * Hq + h;
                    for (int64_t i = 0; i < Sq; ++i) {
                        const double *qi = q + (bh * Sq + i) * d;
                        const double *doi = dO + (bh * Sq + i) * d;
                        double *dqi = dq + (bh * Sq + i) * d;
                        for (int t = 0; t < d; ++t) dqi[t] = 0.0;
                        const int64_t n = visible_keys(i, Sq, Skv, causal);
                        if (n <= 0) continue;
                        double m = -INFINITY;
                        for (int64_t j = 0; j < n; ++j) {
                            double acc = 0.0;
                            for (int t = 0; t < d; ++t) acc += qi[t] * kh[j * d + t];
                            p[j] = scale * acc;
                            if (p[j] > m) m = p[j];
                        }
                        double z = 0.0;
                        for (int64_t j = 0; j < n; ++j) z += exp(p[j] - m);
                        const double lse = m + log(z);
                        double dsum = 0.0;
                        for (int64_t j = 0; j < n; ++j) {
                            p[j] = exp(p[j] - lse);
                            double acc = 0.0;
                            for (int t = 0; t < d; ++t) acc += doi[t] * vh[j * d + t];
                            dp[j] = acc;
                            dsum += p[j] * acc;
                        }
                        for (int64_t j = 0; j < n; ++j) {
                            const double ds = p[j] * (dp[j] - dsum);
                            for (int t = 0; t < d; ++t) {
                                dqi[t] += scale * ds * kh[j * d + t];
                                dkh[j * d + t] += scale * ds * qi[t];
                                dvh[j * d + t] += p[j] * doi[t];
                            }
                        }
                    }
                }
            }
        }
        free(p);
        free(dp);
    }
    return err ? -1 : 0;
}

/* --- 8-bit floating-point inputs ------------------------------------------
 * "FlashAttention & IO-aware attention", section "Deep dive", names
 * FlashAttention-3's FP8 variant and says nothing more.  The reading used
 * here: Q, K and V arrive as E4M3 codes (the OCP 8-bit format with 4 exponent
 * bits, bias 7, 3 mantissa bits, no infinities, NaN = S.1111.111) with one
 * fp32 dequantisation factor per (batch, key/value head) for each of Q, K and
 * V; the real input is factor * value(code).  The attention of those real
 * inputs is then the one-shot definition above, unchanged. */

/* Value of one E4M3 code, written out from the format's definition. */
static double e4m3_value(uint8_t c)
{
    const int sign = (c >> 7) & 1;
    const int e = (c >> 3) & 15;
    const int m = c & 7;
    double mag;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        mag = ldexp((double)m / 8.0, -6);          /* subnormal: 0.m * 2^(1-7) */
    else
        mag = ldexp(1.0 + (double)m / 8.0, e - 7); /* normal: 1.m * 2^(e-7) */
    return sign ? -mag : mag;
}

int oracle_e4m3_decode(const uint8_t *codes, int64_t n, double *out)
{
    if (n < 0 || (n > 0 && (codes == NULL || out == NULL)))
        return -1;
    for (int64_t i = 0; i < n; ++i)
        out[i] = e4m3_value(codes[i]);
    return 0;
}

/* x8 [B,H,S,d] E4M3 codes -> out [B,H,S,d] real values: head h of batch b is
 * scaled by descale[b * Hkv + h / (H / Hkv)] (H = Hq for queries, H = Hkv for
 * keys and values, where the map is the identity).  descale == NULL means 1. */
int oracle_dequant_heads(const uint8_t *x8, const double *descale, double *out, int B, int H,
                         int Hkv, int S, int d)
{
    if (B < 0 || H < 1 || Hkv < 1 || S < 0 || d < 1 || H % Hkv != 0)
        return -1;
    const int group = H / Hkv;
    for (int64_t b = 0; b < B; ++b)
        for (int64_t h = 0; h < H; ++h) {
            const int64_t g = h / group;
            const double f = descale ? descale[b * Hkv + g] : 1.0;
            const int64_t base = ((b * H + h) * (int64_t)S) * d;
            for (int64_t i = 0; i < (int64_t)S * d; ++i)
                out[base + i] = f * e4m3_value(x8[base + i]);
        }
    return 0;
}

/* --- Blockwise feed-forward after attention ---------------------------------
 * "I/O-Aware Kernels", section "Blockwise Parallel Transformers": the
 * feed-forward network acts on every token independently, so it can run on a
 * query block as soon as that block's attention is done, and only that
 * block's activations are ever materialised.  The result is that of the
 * unblocked layer, which is what this oracle computes.  Reading of what the
 * page leaves open: the network's input for token t is the concatenation over
 * query heads of the attention output, x_t = (O[b,0,t,:], ..., O[b,Hq-1,t,:])
 * of width D = Hq * d; the network is two bias-free linear maps with the erf
 * form of GELU between them: y_t = W2 gelu(W1 x_t), W1 [F, D], W2 [D, F]. */

static double gelu(double h)
{
    return 0.5 * h * (1.0 + erf(h / sqrt(2.0)));
}

/* hid [F] = gelu(W1 x_t) for one token. */
static void ffn_token_hidden(const double *xt, const double *w1, int D, int F, double *hid)
{
    for (int f = 0; f < F; ++f) {
        const double *w = w1 + (int64_t)f * D;
        double acc = 0.0;
        for (int i = 0; i < D; ++i) acc += w[i] * xt[i];
        hid[f] = gelu(acc);
    }
}

/* hidden [n, F] = gelu(W1 x) per token (the activations between the two maps). */
int oracle_ffn_hidden(const double *x, const double *w1, double *hid, int64_t n, int D, int F)
{
    if (n < 0 || D < 1 || F < 1)
        return -1;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < n; ++t)
        ffn_token_hidden(x + t * D, w1, D, F, hid + t * F);
    return 0;
}

/* x [n, D] -> y [n, D]; hidden [F] per token in scratch. */
int oracle_ffn(const double *x, const double *w1, const double *w2, double *y, int64_t n,
               int D, int F)
{
    if (n < 0 || D < 1 || F < 1)
        return -1;
    int err = 0;
#pragma omp parallel
    {
        double *hid = (double *)malloc(sizeof(double) * (size_t)F);
        if (!hid) {
#pragma omp atomic write
            err = 1;
        } else {
#pragma omp for schedule(static)
            for (int64_t t = 0; t < n; ++t) {
                ffn_token_hidden(x + t * D, w1, D, F, hid);
                double *yt = y + t * D;
                for (int i = 0; i < D; ++i) {
                    const double *w = w2 + (int64_t)i * F;
                    double acc = 0.0;
                    for (int f = 0; f < F; ++f) acc += w[f] * hid[f];
                    yt[i] = acc;
                }
            }
            free(hid);
        }
    }
    return err ? -1 : 0;
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
