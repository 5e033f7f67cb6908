// fa_decode_kernel.cuh -- split-KV forward for one query row (decode) on the CUDA cores.
//
// With N_q = 1 every K/V tile meets a single query row: the products are
// matrix-vector products (128 multiply-adds per key for Q.K^T and as many for
// P.V), so the step is bound by reading K and V from HBM once, not by the
// tensor cores.  Issuing 128-row tensor-core tiles for one valid row spends a
// full tile of MMAs and softmax work per 128 keys; this kernel streams the keys
// through shared memory with TMA and does the arithmetic on the FMA pipe.
// It computes what the split-KV mode of fa_fwd_sm100_kernel computes (the same
// ranges of 128-key tiles, the same partial layout and arrival counters, the same
// merge by the last CTA of a row), with P kept in fp32.
//
// One CTA per (range s, head h, batch b); 288 threads:
//  * warp 8, one lane: TMA producer, the K and V tiles of the range through a
//    ring of kStages slots (one 128-key tile of K and one of V per slot);
//  * warps 0-7: warp w takes keys 16w .. 16w+15 of each tile.  Q.K: four lanes
//    per key, D/4 elements each, two passes of eight keys; online softmax over
//    the warp's keys (log2 domain, exact rescale of O per tile); P.V: lane l
//    owns O columns l*D/32 .. +D/32-1 and adds p_key * V[key] for the warp's 16
//    keys.  At the end the eight warps' (m, l, O) are combined in shared memory.
// Every wait is bounded; a wait that runs out records FA_ERR_DEVICE_TIMEOUT and
// the CTA still writes an empty range, as the tensor-core split mode does.
#pragma once

#include "fa_fwd_kernel.cuh"

namespace fa {

constexpr int kDecThreads = 288;
constexpr int kDecComputeWarps = 8;
constexpr int kDecProducerWarp = 8;
constexpr uint32_t kDecBarCompute = 7;   // named barrier over the compute warps

template <int D>
struct DecCfg {
    static_assert(D == 64 || D == 128, "head dim");
    static constexpr int kBoxes = D / 64;                  // 64-column boxes per tile row
    static constexpr int kTileBytes = 128 * D * 2;         // one 128-key tile of K (or V)
    static constexpr int kStages = (D == 128) ? 3 : 6;     // 192 KB of K/V in flight
    static constexpr int kKOff = 0;
    static constexpr int kVOff = kStages * kTileBytes;
    static constexpr int kRedOff = 2 * kStages * kTileBytes;           // [8 warps][m, l, O[D]] fp32
    static constexpr int kBarOff = kRedOff + kDecComputeWarps * (2 + D) * 4;
    static constexpr int kMiscOff = kBarOff + 2 * kStages * 8;         // abort flag, merge flag
    static constexpr int kSmemBytes = kMiscOff + 16 + 1024;
    static_assert(kSmemBytes <= 232448, "dynamic shared memory per CTA on sm_100");
};

// Address of the 16-byte chunk ch (0 .. D/8-1) of row r in a tile stored as
// 64-column boxes of 128 rows x 128 bytes with the 128-byte swizzle.
template <int D>
__device__ __forceinline__ uint32_t dec_chunk(uint32_t tile, int r, int ch) {
    return tile + (uint32_t)((ch >> 3) * kSwizzleBoxBytes + r * 128 + (((ch & 7) ^ (r & 7)) << 4));
}

template <int D>
__global__ void __launch_bounds__(kDecThreads, 1)
    fa_decode_splitkv_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                             const __nv_bfloat16* __restrict__ q, const FwdParams p) {
    using C = DecCfg<D>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw_base = smem_addr(smem_raw);
    const uint32_t base = (raw_base + 1023u) & ~1023u;
    uint8_t* const base_ptr = smem_raw + (base - raw_base);
    auto bar_full = [&](int s) { return base + C::kBarOff + 8u * (uint32_t)s; };
    auto bar_empty = [&](int s) { return base + C::kBarOff + 8u * (uint32_t)(C::kStages + s); };
    volatile int* const abort_flag = reinterpret_cast<volatile int*>(base_ptr + C::kMiscOff);
    volatile int* const merge_flag = reinterpret_cast<volatile int*>(base_ptr + C::kMiscOff + 4);
    float* const red = reinterpret_cast<float*>(base_ptr + C::kRedOff);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int split = (int)blockIdx.x;
    const int h = (int)blockIdx.y;
    const int b = (int)blockIdx.z;
    const int n_split = p.num_splits;
    int kl = p.Nk;
    if (p.key_lens != nullptr) {
        kl = p.key_lens[b];
        kl = kl < 0 ? 0 : (kl > p.Nk ? p.Nk : kl);
    }
    // the one query row (row 0, diagonal offset N_k - 1) sees keys [0, lim)
    const int lim = row_key_limit(0, kl, p.Nk - 1, p.causal);
    const int n_tiles = (lim + kBlockN - 1) / kBlockN;
    const int t_lo = (int)(((long long)split * n_tiles) / n_split);
    const int t_hi = (int)(((long long)(split + 1) * n_tiles) / n_split);
    const int n_t = t_hi - t_lo;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(bar_full(s), 1);
            mbar_init(bar_empty(s), kDecComputeWarps);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == kDecProducerWarp) {
        // ============================================================ TMA producer
        if (lane == 0 && n_t > 0) {
            prefetch_tensormap(&tm_k);
            prefetch_tensormap(&tm_v);
            const uint64_t pol = policy_evict_first();   // K and V are read once
            bool ok = true;
            int j = 0;
            for (; j < n_t; ++j) {
                const int s = j % C::kStages;
                ok = wait_bounded(bar_empty(s), (uint32_t)(((j / C::kStages) & 1) ^ 1), abort_flag, p.wait_limit);
                if (!ok) break;
                mbar_arrive_expect_tx(bar_full(s), 2u * (uint32_t)C::kTileBytes);
                const int key0 = (t_lo + j) * kBlockN;
                for (int bx = 0; bx < C::kBoxes; ++bx) {
                    tma_load_4d(base + C::kKOff + (uint32_t)(s * C::kTileBytes + bx * kSwizzleBoxBytes), &tm_k,
                                bar_full(s), bx * 64, key0, h, b, pol);
                    tma_load_4d(base + C::kVOff + (uint32_t)(s * C::kTileBytes + bx * kSwizzleBoxBytes), &tm_v,
                                bar_full(s), bx * 64, key0, h, b, pol);
                }
            }
            // every copy issued lands before the CTA exits (also after a give-up)
            for (int c2 = (j > C::kStages ? j - C::kStages : 0); c2 < j; ++c2)
                (void)wait_own_work(bar_full(c2 % C::kStages), (uint32_t)((c2 / C::kStages) & 1));
        }
        __syncwarp();
        return;   // the producer takes no part in the combine below (named barrier)
    }

    // ================================================================ compute warps
    constexpr int kCh = D / 32;   // 16-byte chunks of a K row per lane (four lanes per key)
    constexpr int kOw = D / 32;   // O columns per lane
    const int pq = lane & 3;      // which quarter of the key row
    const int kk = lane >> 2;     // which of the eight keys of a pass
    float qf[kCh * 8];
    {
        const __nv_bfloat16* qrow = q + ((size_t)b * p.H + h) * (size_t)D;   // N_q = 1: [B, H, 1, D]
#pragma unroll
        for (int c = 0; c < kCh; ++c) {
            const uint4 w4 = __ldg(reinterpret_cast<const uint4*>(qrow + (pq * kCh + c) * 8));
            const uint32_t wv[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                qf[c * 8 + 2 * e] = __uint_as_float(wv[e] << 16);
                qf[c * 8 + 2 * e + 1] = __uint_as_float(wv[e] & 0xffff0000u);
            }
        }
    }
    const float sc = p.scale_log2;
    float m_w = -INFINITY;   // running max of the warp's scores (log2 units)
    float l_w = 0.f;         // running sum of 2^(x - m_w)
    float o[kOw];
#pragma unroll
    for (int e = 0; e < kOw; ++e) o[e] = 0.f;
    bool ok = true;
    for (int j = 0; j < n_t; ++j) {
        const int s = j % C::kStages;
        const bool good = wait_bounded(bar_full(s), (uint32_t)((j / C::kStages) & 1), abort_flag, p.wait_limit);
        if (!__all_sync(0xffffffffu, good)) {
            ok = false;
            break;
        }
        const uint32_t kt = base + C::kKOff + (uint32_t)(s * C::kTileBytes);
        const uint32_t vt = base + C::kVOff + (uint32_t)(s * C::kTileBytes);
        const int key0 = (t_lo + j) * kBlockN;
        // scores of keys 16w + 8*pass + kk (log2 units), held by the key's four lanes
        float x[2];
#pragma unroll
        for (int pass = 0; pass < 2; ++pass) {
            const int r = warp * 16 + pass * 8 + kk;
            float acc = 0.f;
#pragma unroll
            for (int c = 0; c < kCh; ++c) {
                uint32_t w0, w1, w2, w3;
                asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                             : "=r"(w0), "=r"(w1), "=r"(w2), "=r"(w3)
                             : "r"(dec_chunk<D>(kt, r, pq * kCh + c)));
                const uint32_t wv[4] = {w0, w1, w2, w3};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    acc = fmaf(qf[c * 8 + 2 * e], __uint_as_float(wv[e] << 16), acc);
                    acc = fmaf(qf[c * 8 + 2 * e + 1], __uint_as_float(wv[e] & 0xffff0000u), acc);
                }
            }
            acc += __shfl_xor_sync(0xffffffffu, acc, 1);
            acc += __shfl_xor_sync(0xffffffffu, acc, 2);
            x[pass] = (key0 + r < lim) ? acc * sc : -INFINITY;
        }
        float mt = fmaxf(x[0], x[1]);
        mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 4));
        mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 8));
        mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 16));
        const float m_new = fmaxf(m_w, mt);
        if (m_new != -INFINITY) {
            const float alpha = ex2_approx(m_w - m_new);   // 0 while m_w is -inf
            const float p0 = ex2_approx(x[0] - m_new), p1 = ex2_approx(x[1] - m_new);
            float ps = p0 + p1;
            ps += __shfl_xor_sync(0xffffffffu, ps, 4);
            ps += __shfl_xor_sync(0xffffffffu, ps, 8);
            ps += __shfl_xor_sync(0xffffffffu, ps, 16);
            l_w = fmaf(l_w, alpha, ps);
            m_w = m_new;
#pragma unroll
            for (int e = 0; e < kOw; ++e) o[e] *= alpha;
#pragma unroll
            for (int pass = 0; pass < 2; ++pass) {
#pragma unroll
                for (int kq = 0; kq < 8; ++kq) {
                    const float pk = __shfl_sync(0xffffffffu, pass ? p1 : p0, kq * 4);
                    const int r = warp * 16 + pass * 8 + kq;
                    if constexpr (D == 128) {
                        uint32_t v0, v1;
                        asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];"
                                     : "=r"(v0), "=r"(v1)
                                     : "r"(dec_chunk<D>(vt, r, lane >> 1) + (uint32_t)((lane & 1) * 8)));
                        o[0] = fmaf(pk, __uint_as_float(v0 << 16), o[0]);
                        o[1] = fmaf(pk, __uint_as_float(v0 & 0xffff0000u), o[1]);
                        o[2] = fmaf(pk, __uint_as_float(v1 << 16), o[2]);
                        o[3] = fmaf(pk, __uint_as_float(v1 & 0xffff0000u), o[3]);
                    } else {
                        uint32_t v0;
                        asm volatile("ld.shared.b32 %0, [%1];"
                                     : "=r"(v0)
                                     : "r"(dec_chunk<D>(vt, r, lane >> 2) + (uint32_t)((lane & 3) * 4)));
                        o[0] = fmaf(pk, __uint_as_float(v0 << 16), o[0]);
                        o[1] = fmaf(pk, __uint_as_float(v0 & 0xffff0000u), o[1]);
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_empty(s));
    }

    // ---------------------------------------------------------------- combine the eight warps
    float* const rw = red + warp * (2 + D);
    if (lane == 0) {
        rw[0] = m_w;
        rw[1] = l_w;
    }
#pragma unroll
    for (int e = 0; e < kOw; ++e) rw[2 + lane * kOw + e] = o[e];
    const bool bad = named_bar_or(kDecBarCompute, kDecComputeWarps * 32, !ok);
    if (warp != 0) return;
    float mx = -INFINITY;
#pragma unroll
    for (int w = 0; w < kDecComputeWarps; ++w) mx = fmaxf(mx, red[w * (2 + D)]);
    float L = 0.f;
    float acc[kOw];
#pragma unroll
    for (int e = 0; e < kOw; ++e) acc[e] = 0.f;
    if (mx != -INFINITY) {
#pragma unroll
        for (int w = 0; w < kDecComputeWarps; ++w) {
            const float f = ex2_approx(red[w * (2 + D)] - mx);
            L = fmaf(red[w * (2 + D) + 1], f, L);
#pragma unroll
            for (int e = 0; e < kOw; ++e) acc[e] = fmaf(red[w * (2 + D) + 2 + lane * kOw + e], f, acc[e]);
        }
    }
    if (bad) L = 0.f;   // a wait ran out: an empty range (the status word says why)
    const float inv = (L > 0.f) ? 1.f / L : 0.f;
    const float lse = (L > 0.f) ? (mx + __log2f(L)) * 0.69314718055994531f : -INFINITY;
    const size_t rows_total = (size_t)p.B * p.H;   // N_q = 1
    const size_t rg = (size_t)b * p.H + h;
    if (n_split == 1) {
        // a single range: the final result
        __nv_bfloat16* dst = p.o_out + rg * D + lane * kOw;
#pragma unroll
        for (int e = 0; e < kOw; e += 2)
            *reinterpret_cast<uint32_t*>(dst + e) = pack_bf16x2(acc[e] * inv, acc[e + 1] * inv);
        if (lane == 0) p.lse[rg] = lse;
        return;
    }
    float* const op = p.o_part + ((size_t)split * rows_total + rg) * D + lane * kOw;
#pragma unroll
    for (int e = 0; e < kOw; ++e) op[e] = acc[e] * inv;
    if (lane == 0) p.lse_part[(size_t)split * rows_total + rg] = lse;
    __threadfence();   // the partial is visible before the arrival below
    __syncwarp();
    if (lane == 0) *merge_flag = split_arrive_last(p.split_counter + rg, p.split_ticket, n_split) ? 1 : 0;
    __syncwarp();
    if (!*merge_flag) return;
    // the last range of this row to arrive merges all of them (running-max rule):
    // the ranges' LSEs a range per lane, their partial O rows with eight loads in
    // flight per lane, so the merge is not a chain of dependent L2 round trips
    __threadfence();
    float ml = -INFINITY;
    for (int s0 = 0; s0 < n_split; s0 += 32) {
        const int sp = s0 + lane;
        if (sp < n_split) ml = fmaxf(ml, __ldcg(p.lse_part + (size_t)sp * rows_total + rg));
    }
#pragma unroll
    for (int sh = 16; sh > 0; sh >>= 1) ml = fmaxf(ml, __shfl_xor_sync(0xffffffffu, ml, sh));
    float wsum = 0.f;
    float out[kOw];
#pragma unroll
    for (int e = 0; e < kOw; ++e) out[e] = 0.f;
    if (ml != -INFINITY) {
        for (int s0 = 0; s0 < n_split; s0 += 32) {
            const int sp = s0 + lane;
            const float ls = (sp < n_split) ? __ldcg(p.lse_part + (size_t)sp * rows_total + rg) : -INFINITY;
            const float w = (ls == -INFINITY) ? 0.f : expf(ls - ml);
            wsum += w;
            const int cnt = min(32, n_split - s0);
#pragma unroll 8
            for (int t = 0; t < cnt; ++t) {
                const float wt = __shfl_sync(0xffffffffu, w, t);
                const float* src = p.o_part + ((size_t)(s0 + t) * rows_total + rg) * D + lane * kOw;
#pragma unroll
                for (int e = 0; e < kOw; ++e) out[e] = fmaf(wt, __ldcg(src + e), out[e]);
            }
        }
#pragma unroll
        for (int sh = 16; sh > 0; sh >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, sh);
    }
    const float winv = (wsum > 0.f) ? 1.f / wsum : 0.f;
    __nv_bfloat16* dst = p.o_out + rg * D + lane * kOw;
#pragma unroll
    for (int e = 0; e < kOw; e += 2)
        *reinterpret_cast<uint32_t*>(dst + e) = pack_bf16x2(out[e] * winv, out[e + 1] * winv);
    if (lane == 0) p.lse[rg] = (wsum > 0.f) ? ml + logf(wsum) : -INFINITY;
}

}  // namespace fa
