/*
 * oracle/attn_ref.c -- TEST INFRASTRUCTURE ONLY.
 *
 * Plain, slow, fp64 CPU oracle for the exact attention forward pass
 *     O = softmax(scale * Q K^T + mask) V,   LSE_i = ln sum_j exp(scale * q_i . k_j)
 * written straight from the definition: for every query row the full score
 * row S_i and probability row P_i are materialised, then O_i = P_i V.
 *
 * Sources for what is computed:
 *   - "FlashAttention 与边缘设备上的注意力内存瓶颈", section 2 (standard
 *     attention forms S and P, both N x N) and section 3.2 (the tiled method
 *     stays exact, so its result is this definition).
 *   - "FlashAttention：把注意力从公式写成数据流", opening paragraph (S = QK^T,
 *     then softmax, then multiply by V) and section "精度、掩码和边界情况"
 *     (masked positions never enter the normaliser; tail blocks).
 * Readings where the pages are silent (causal alignment, key_lens, LSE,
 * fully masked rows) are the ones the library documents in include/fa.h:
 *   - causal is bottom-right aligned: key j is visible to query i iff
 *     j <= i + (N_k - N_q);
 *   - key_lens[b] (NULL = all keys) is clamped to [0, N_k]; keys j >= it are masked;
 *   - both masks combine with AND; the valid keys of row i are therefore the
 *     prefix [0, lim_i);
 *   - a row with no valid key has O = 0 and LSE = -inf.
 *   - sliding window (attn_ref_fp64_window only): with window_left = W >= 0
 *     key j is also masked when j < i + (N_k - N_q) - W, so row i sees the
 *     keys [lo_i, lim_i), lo_i = max(0, i + N_k - N_q - W): at most the W
 *     keys before its diagonal position plus that position.  This is the
 *     local-attention mask of the "mask variants" the second page's section
 *     "精度、掩码和边界情况" groups with causal and padding masks.
 *   - additive positional bias (attn_ref_fp64_bias only): with per-head slopes
 *     m_h, S_ij += -m_h * |i + (N_k - N_q) - j| on the visible entries (a
 *     linear distance penalty from the row's diagonal position, the
 *     "additive positional bias" mask variant).
 *   - custom positional bias table (attn_ref_fp64_bias_table only): a caller's
 *     per-head table T_h of 2R+1 values indexed by the key's position relative
 *     to the row's diagonal position, clamped to [-R, R]:
 *         S_ij += T_h[clamp(j - (i + N_k - N_q), -R, R) + R]
 *     (any function of relative position within R, constant beyond it: the
 *     general "custom positional bias" of the same section).
 *
 * Nothing here is shared with the CUDA path.  Only tests/, the package's
 * graft entry smoke check and bench.py's CPU baseline may call it.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* bf16 bit pattern -> fp64, exact (bf16 is the top half of an fp32). */
static double bf16_bits_to_f64(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Threads for the following calls (n >= 1); used to time the oracle on one core. */
void oracle_set_num_threads(int n) {
#ifdef _OPENMP
    if (n >= 1) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* Number of valid keys of query row i: the prefix [0, lim) of the key axis. */
static int64_t row_limit(int64_t i, int64_t b, const int32_t *key_lens,
                         int64_t Nq, int64_t Nk, int causal) {
    int64_t kl = Nk;
    if (key_lens) {
        kl = key_lens[b];
        if (kl < 0) kl = 0;
        if (kl > Nk) kl = Nk;
    }
    int64_t lim = kl;
    if (causal) {
        int64_t c = i + (Nk - Nq) + 1; /* keys j <= i + Nk - Nq */
        if (c < 0) c = 0;
        if (c < lim) lim = c;
    }
    return lim;
}

/* First valid key of row i under a sliding window of W keys (W < 0: none). */
static int64_t row_start(int64_t i, int64_t Nq, int64_t Nk, int64_t W) {
    if (W < 0) return 0;
    int64_t lo = i + (Nk - Nq) - W;
    return lo < 0 ? 0 : lo;
}

/*
 * One query row, straight from the definition.  The valid keys are
 * [lo, lim).  s_row and p_row are caller scratch of length Nk; on return they
 * hold S_i (masked entries -inf) and P_i (masked entries 0).
 */
static void one_row(const uint16_t *q_row, const uint16_t *k_head,
                    const uint16_t *v_head, int64_t Nk, int64_t d,
                    double scale, int64_t lo, int64_t lim, double slope, int64_t pos,
                    const float *table, int64_t R,
                    double *s_row, double *p_row, double *o_row, double *lse_out) {
    /* S_ij = scale * sum_c q_ic k_jc (- slope * |pos - j|) (+ table[...]) for
     * valid j, -inf for masked j. */
    for (int64_t j = 0; j < Nk; ++j) {
        if (j >= lo && j < lim) {
            double dot = 0.0;
            for (int64_t c = 0; c < d; ++c)
                dot += bf16_bits_to_f64(q_row[c]) * bf16_bits_to_f64(k_head[j * d + c]);
            s_row[j] = scale * dot;
            if (slope != 0.0) s_row[j] -= slope * (double)llabs(pos - j);
            if (table) {
                int64_t r = j - pos;
                if (r < -R) r = -R;
                if (r > R) r = R;
                s_row[j] += (double)table[r + R];
            }
        } else {
            s_row[j] = -INFINITY;
        }
    }
    if (lim <= lo) {
        for (int64_t j = 0; j < Nk; ++j) p_row[j] = 0.0;
        for (int64_t c = 0; c < d; ++c) o_row[c] = 0.0;
        *lse_out = -INFINITY;
        return;
    }
    /* softmax over the valid entries: subtract the row max, exp, normalise. */
    double m = -INFINITY;
    for (int64_t j = lo; j < lim; ++j)
        if (s_row[j] > m) m = s_row[j];
    double l = 0.0;
    for (int64_t j = 0; j < Nk; ++j) {
        p_row[j] = (j >= lo && j < lim) ? exp(s_row[j] - m) : 0.0;
        l += p_row[j];
    }
    for (int64_t j = 0; j < Nk; ++j) p_row[j] /= l;
    /* O_i = sum_j P_ij V_j */
    for (int64_t c = 0; c < d; ++c) o_row[c] = 0.0;
    for (int64_t j = lo; j < lim; ++j)
        for (int64_t c = 0; c < d; ++c)
            o_row[c] += p_row[j] * bf16_bits_to_f64(v_head[j * d + c]);
    *lse_out = m + log(l);
}

/*
 * Full forward.  q: bf16 bits [B,H,Nq,d]; k, v: bf16 bits [B,H,Nk,d];
 * key_lens: int32 [B] or NULL.  o: fp64 [B,H,Nq,d]; lse: fp64 [B,H,Nq].
 * p_out: NULL, or fp64 [B,H,Nq,Nk] receiving the materialised P.
 * scale is a double: the bf16 callers pass the fp32 value the GPU receives,
 * widened; the E4M3 wrapper passes the exact fp64 product of its three
 * score factors (scale * q_descale * k_descale).
 * Returns 0, or -1 on bad sizes / allocation failure.
 */
/*
 * Sliding-window forward (window_left = W >= 0 keys before the diagonal
 * position, see the header comment; W < 0 means no window and gives exactly
 * attn_ref_fp64).  Arguments otherwise as attn_ref_fp64.
 */
int attn_ref_fp64_bias(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                       const int32_t *key_lens, int64_t B, int64_t H, int64_t Nq,
                       int64_t Nk, int64_t d, double scale, int causal,
                       int64_t window_left, const float *slopes, double *o, double *lse,
                       double *p_out);

int attn_ref_fp64_window(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                         const int32_t *key_lens, int64_t B, int64_t H, int64_t Nq,
                         int64_t Nk, int64_t d, double scale, int causal,
                         int64_t window_left, double *o, double *lse, double *p_out) {
    return attn_ref_fp64_bias(q, k, v, key_lens, B, H, Nq, Nk, d, scale, causal, window_left,
                              NULL, o, lse, p_out);
}

/*
 * Forward with a sliding window (window_left < 0: none), a linear additive
 * positional bias (slopes: fp32 [H], one slope per head, or NULL: none) and a
 * custom positional bias table (table: fp32 [H, 2R+1], or NULL: none).
 */
static int attn_ref_general(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                            const int32_t *key_lens, int64_t B, int64_t H, int64_t Nq,
                            int64_t Nk, int64_t d, double scale, int causal,
                            int64_t window_left, const float *slopes, const float *table,
                            int64_t R, double *o, double *lse, double *p_out) {
    if (B < 0 || H < 0 || Nq < 0 || Nk < 0 || d <= 0 || R < 0) return -1;
    const double sc = (double)scale;
    const int64_t rows = B * H * Nq;
    int failed = 0;
#pragma omp parallel
    {
        double *s_row = (double *)malloc(sizeof(double) * (size_t)(Nk > 0 ? Nk : 1));
        double *p_row = (double *)malloc(sizeof(double) * (size_t)(Nk > 0 ? Nk : 1));
        if (!s_row || !p_row) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 16)
            for (int64_t r = 0; r < rows; ++r) {
                const int64_t i = r % Nq;
                const int64_t bh = r / Nq;
                const int64_t b = bh / H;
                const int64_t lim = row_limit(i, b, key_lens, Nq, Nk, causal);
                const int64_t lo = row_start(i, Nq, Nk, window_left);
                const double slope = slopes ? (double)slopes[bh % H] : 0.0;
                const float *tab = table ? table + (bh % H) * (2 * R + 1) : NULL;
                one_row(q + r * d, k + bh * Nk * d, v + bh * Nk * d, Nk, d, sc,
                        lo, lim, slope, i + (Nk - Nq), tab, R, s_row, p_row, o + r * d, lse + r);
                if (p_out) memcpy(p_out + r * Nk, p_row, sizeof(double) * (size_t)Nk);
            }
        }
        free(s_row);
        free(p_row);
    }
    return failed ? -1 : 0;
}

/* Forward with a sliding window and a linear additive positional bias. */
int attn_ref_fp64_bias(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                       const int32_t *key_lens, int64_t B, int64_t H, int64_t Nq,
                       int64_t Nk, int64_t d, double scale, int causal,
                       int64_t window_left, const float *slopes, double *o, double *lse,
                       double *p_out) {
    return attn_ref_general(q, k, v, key_lens, B, H, Nq, Nk, d, scale, causal, window_left,
                            slopes, NULL, 0, o, lse, p_out);
}

/*
 * Forward with a sliding window and a custom positional bias table:
 * table fp32 [H, 2R+1], R >= 0 (see the header comment).
 */
int attn_ref_fp64_bias_table(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                             const int32_t *key_lens, int64_t B, int64_t H, int64_t Nq,
                             int64_t Nk, int64_t d, double scale, int causal,
                             int64_t window_left, const float *table, int64_t R, double *o,
                             double *lse, double *p_out) {
    if (!table) return -1;
    return attn_ref_general(q, k, v, key_lens, B, H, Nq, Nk, d, scale, causal, window_left,
                            NULL, table, R, o, lse, p_out);
}

int attn_ref_fp64(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                  const int32_t *key_lens, int64_t B, int64_t H, int64_t Nq,
                  int64_t Nk, int64_t d, double scale, int causal, double *o,
                  double *lse, double *p_out) {
    return attn_ref_fp64_window(q, k, v, key_lens, B, H, Nq, Nk, d, scale, causal, -1,
                                o, lse, p_out);
}

/*
 * Same definition evaluated only on selected rows, for checking outputs of
 * problems too large to evaluate whole.  row_ids[n] are flat row indices
 * r = (b*H + h)*Nq + i.  o_rows: fp64 [n,d]; lse_rows: fp64 [n].
 */
int attn_ref_fp64_rows(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                       const int32_t *key_lens, int64_t B, int64_t H, int64_t Nq,
                       int64_t Nk, int64_t d, double scale, int causal,
                       const int64_t *row_ids, int64_t n, double *o_rows,
                       double *lse_rows) {
    if (B < 0 || H < 0 || Nq < 0 || Nk < 0 || d <= 0 || n < 0) return -1;
    const double sc = (double)scale;
    const int64_t rows = B * H * Nq;
    for (int64_t t = 0; t < n; ++t)
        if (row_ids[t] < 0 || row_ids[t] >= rows) return -1;
    int failed = 0;
#pragma omp parallel
    {
        double *s_row = (double *)malloc(sizeof(double) * (size_t)(Nk > 0 ? Nk : 1));
        double *p_row = (double *)malloc(sizeof(double) * (size_t)(Nk > 0 ? Nk : 1));
        if (!s_row || !p_row) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 4)
            for (int64_t t = 0; t < n; ++t) {
                const int64_t r = row_ids[t];
                const int64_t i = r % Nq;
                const int64_t bh = r / Nq;
                const int64_t b = bh / H;
                const int64_t lim = row_limit(i, b, key_lens, Nq, Nk, causal);
                one_row(q + r * d, k + bh * Nk * d, v + bh * Nk * d, Nk, d, sc,
                        0, lim, 0.0, i + (Nk - Nq), NULL, 0, s_row, p_row, o_rows + t * d,
                        lse_rows + t);
            }
        }
        free(s_row);
        free(p_row);
    }
    return failed ? -1 : 0;
}
