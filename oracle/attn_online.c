/*
 * oracle/attn_online.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A second CPU formulation of the same attention forward, in fp64, following
 * the online-softmax recurrence the pages describe: keys are visited in
 * blocks; for every block the running row maximum m, the running sum of
 * exponentials l and the output accumulator are updated, the old l and
 * accumulator being rescaled by exp(m_old - m_new).  The pages state that the
 * result is identical to standard attention and only the order of operations
 * differs, so this file must agree with attn_ref.c up to rounding:
 *   - "FlashAttention 与边缘设备上的注意力内存瓶颈", section 3.2 (online
 *     softmax keeps the current maximum and normaliser; result stays exact);
 *   - "FlashAttention：把注意力从公式写成数据流", section "分块与在线 softmax"
 *     (for each new block update max, exp-sum and output accumulator; same
 *     result as standard attention, only the execution order differs).
 *
 * Unlike attn_ref.c it decides visibility key by key with its own predicate
 * instead of a prefix length, so a mistake in either mask shows up as a
 * disagreement.  Convention: exp(-inf - (-inf)) is taken as 0 (a block whose
 * keys are all masked changes nothing).
 *
 * Shares no code with attn_ref.c or with the CUDA path.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static double widen_bf16(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Is key j visible to query i of batch b? */
static int key_visible(int64_t i, int64_t j, int64_t b, const int32_t *key_lens,
                       int64_t Nq, int64_t Nk, int causal) {
    if (j >= Nk) return 0;
    if (key_lens) {
        int64_t kl = key_lens[b];
        if (kl > Nk) kl = Nk;
        if (j >= kl) return 0; /* kl < 0 masks every key */
    }
    if (causal && j - i > Nk - Nq) return 0;
    return 1;
}

int attn_online_fp64(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                     const int32_t *key_lens, int64_t B, int64_t H, int64_t Nq,
                     int64_t Nk, int64_t d, float scale, int causal,
                     int64_t block, double *o, double *lse) {
    if (B < 0 || H < 0 || Nq < 0 || Nk < 0 || d <= 0 || block <= 0) return -1;
    const double sc = (double)scale;
    const int64_t rows = B * H * Nq;
    int failed = 0;
#pragma omp parallel
    {
        double *acc = (double *)malloc(sizeof(double) * (size_t)d);
        double *sblk = (double *)malloc(sizeof(double) * (size_t)block);
        if (!acc || !sblk) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 16)
            for (int64_t r = 0; r < rows; ++r) {
                const int64_t i = r % Nq;
                const int64_t bh = r / Nq;
                const int64_t b = bh / H;
                const uint16_t *qi = q + r * d;
                const uint16_t *kh = k + bh * Nk * d;
                const uint16_t *vh = v + bh * Nk * d;
                double m = -INFINITY, l = 0.0;
                for (int64_t c = 0; c < d; ++c) acc[c] = 0.0;
                for (int64_t j0 = 0; j0 < Nk; j0 += block) {
                    const int64_t nb = (Nk - j0 < block) ? (Nk - j0) : block;
                    double mblk = -INFINITY;
                    for (int64_t t = 0; t < nb; ++t) {
                        const int64_t j = j0 + t;
                        if (key_visible(i, j, b, key_lens, Nq, Nk, causal)) {
                            double dot = 0.0;
                            for (int64_t c = 0; c < d; ++c)
                                dot += widen_bf16(qi[c]) * widen_bf16(kh[j * d + c]);
                            sblk[t] = sc * dot;
                        } else {
                            sblk[t] = -INFINITY;
                        }
                        if (sblk[t] > mblk) mblk = sblk[t];
                    }
                    const double m_new = (mblk > m) ? mblk : m;
                    if (m_new == -INFINITY) continue; /* nothing visible yet */
                    const double alpha = (m == -INFINITY) ? 0.0 : exp(m - m_new);
                    l *= alpha;
                    for (int64_t c = 0; c < d; ++c) acc[c] *= alpha;
                    for (int64_t t = 0; t < nb; ++t) {
                        if (sblk[t] == -INFINITY) continue;
                        const double e = exp(sblk[t] - m_new);
                        l += e;
                        const uint16_t *vj = vh + (j0 + t) * d;
                        for (int64_t c = 0; c < d; ++c) acc[c] += e * widen_bf16(vj[c]);
                    }
                    m = m_new;
                }
                if (l > 0.0) {
                    for (int64_t c = 0; c < d; ++c) o[r * d + c] = acc[c] / l;
                    lse[r] = m + log(l);
                } else {
                    for (int64_t c = 0; c < d; ++c) o[r * d + c] = 0.0;
                    lse[r] = -INFINITY;
                }
            }
        }
        free(acc);
        free(sblk);
    }
    return failed ? -1 : 0;
}
