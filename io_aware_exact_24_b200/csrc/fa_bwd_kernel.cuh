// fa_bwd_kernel.cuh -- attention backward pass for sm_100a (B200).
//
// What it computes: given Q, K, V, the forward's O and LSE, and the upstream
// gradient dO, the gradients of O = softmax(scale * Q K^T + mask) V:
//   P  = exp(scale * Q K^T - LSE)  (recomputed from the saved LSE, never stored)
//   dV = P^T dO,   dP = dO V^T,   dS = P * (dP - D)  with D_i = dO_i . O_i,
//   dQ = scale * dS K,   dK = scale * dS^T Q.
// The pages name the backward pass and its recomputation of the attention
// matrix from the saved statistics ("FlashAttention：把注意力从公式写成数据流",
// section "用实验验证而不是背诵结论"; "[2205.14135] FlashAttention: Fast and
// Memory-Efficient Exact Attention with IO-Awareness", section
// "三、FLOPs（計算能力）並非 Speedup 的主因素"); the formulas are the chain rule
// of the forward's definition.
//
// Layout (one CTA per 128-key block of one (b, h); it walks the query tiles that
// can see its keys):
//  * warp 0 (one lane): TMA loads of K_j and V_j once, then Q_i and dO_i per
//    query tile (Q and dO in rings of their own: kStagesQ / kStagesO slots);
//  * warp 1 (one lane): the five tcgen05 MMAs of a tile --
//      S^T  = K_j Q_i^T   and  dP^T = V_j dO_i^T     (M = 128 keys, N = 128 queries;
//                                                      at d = 64 A = K_j / V_j from TMEM)
//      dV  += P^T dO_i    and  dK  += dS^T Q_i       (A = P^T / dS^T from TMEM, issued
//                                                      per compute pass)
//      dQ_i = dS K_j                                  (A = dS^T from shared memory,
//                                                      MN-major: M = queries)
//    dV and dK stay in TMEM for the whole CTA;
//  * warps 4-11, two per TMEM lane quadrant, each thread one key row: in two
//    passes of 32 queries each, P^T and dS^T from S^T and dP^T (exp2 domain,
//    masks), written back to TMEM as bf16 over the columns just read and, for
//    dS^T, to shared memory, each pass handed to the issuer on its own barrier;
//    then each thread reads half of one query row of dQ_i, stages it in shared
//    memory and adds it into the fp32 dQ accumulator in global memory with a TMA
//    tensor reduce-add (several key blocks update each query row); finally dV
//    and scale * dK go to global memory as bf16.  At d = 64 they first copy the
//    block's K and V rows into TMEM.
// Every mbarrier wait is bounded (as in the forward kernel); a wait that runs
// out records FA_ERR_DEVICE_TIMEOUT and the CTA winds down.
#pragma once

#include <type_traits>

#include "fa_fwd_kernel.cuh"

namespace fa {

constexpr int kBwdThreads = 384;
constexpr int kBwdProducerWarp = 0;
constexpr int kBwdMmaWarp = 1;
constexpr int kBwdComputeWarp0 = 4;     // warps 4..11: two per TMEM lane quadrant (warp % 4)
constexpr int kBwdComputeWarps = 8;
constexpr uint32_t kBwdBarCompute = 6;  // named barrier over the 8 compute warps

struct BwdParams {
    const float* lse;           // [B,H,Nq] the forward's LSE (natural log; -inf: no visible key)
    const float* dsum;          // [B,H,Nq] D_i = dO_i . O_i (fa_bwd_pre_kernel)
    float* dq_acc;              // [B,H,Nq,D] fp32 accumulator, zero on entry
    __nv_bfloat16* dk;          // [B,H,Nk,D]
    __nv_bfloat16* dv;          // [B,H,Nk,D]
    const int32_t* key_lens;    // [B] or nullptr
    int B, H, Nq, Nk;
    float scale;                // softmax scale
    float scale_log2;           // scale * log2(e)
    int causal;
    unsigned long long wait_limit;
};

template <int D>
struct BwdCfg {
    static_assert(D == 64 || D == 128, "head dim");
    static constexpr int kBoxes = D / 64;
    static constexpr int kTileBytes = 128 * D * 2;
    // Q and dO slots: two of each at d = 64, one of each at d = 128 (the room a
    // second pair would take holds half of the dQ staging there)
    static constexpr int kStagesQ = (D == 64) ? 2 : 1;
    static constexpr int kStagesO = (D == 64) ? 2 : 1;
    static constexpr int kKOff = 0;
    static constexpr int kVOff = kKOff + kTileBytes;
    static constexpr int kQOff = kVOff + kTileBytes;                  // [kStagesQ]
    static constexpr int kDOOff = kQOff + kStagesQ * kTileBytes;      // [kStagesO]
    static constexpr int kDSOff = kDOOff + kStagesO * kTileBytes;     // dS^T: 2 boxes of 64 queries
    // dQ staging for the tensor reduce (fp32, boxes of 32 columns x 128 rows, 128-byte
    // swizzle): box (g, 0) of compute-warp half g is dS^T box g (free between the dQ
    // product and the next tile's dS^T); at d = 128 box (g, 1) is extra box g here
    static constexpr int kDQ2Off = kDSOff + 2 * kSwizzleBoxBytes;
    static constexpr int kRowOff = kDQ2Off + (D == 128 ? 2 * kSwizzleBoxBytes : 0);   // [2][lse2 x128 | D x128] fp32
    static constexpr int kBarOff = kRowOff + 2 * 256 * 4;
    // barriers: kv_full, q_full[SQ], q_empty[SQ], o_full[SO], o_empty[SO], s_full,
    // p_full (pass 0), dq_full, s_free, drain, p_full (pass 1), kv_tmem
    static constexpr int kNumBars = 1 + 2 * kStagesQ + 2 * kStagesO + 7;
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;
    static constexpr int kSmemBytes = kMiscOff + 16 + 1024;
    static_assert(kSmemBytes <= 232448, "dynamic shared memory per CTA on sm_100");
    // TMEM columns: S^T (then P^T as bf16, then dQ) at 0; dP^T (then dS^T) at 128;
    // dV at 256; dK at 256 + D.  P^T of the 32 queries 32cb.. sits at columns
    // 32cb..32cb+15 (dS^T likewise from 128), so each compute warp overwrites only
    // columns it has itself read.  At d = 64 the block's K and V rows (bf16 pairs)
    // also live in TMEM, at 384 and 416: S^T and dP^T then take their A operand from
    // TMEM and read only Q / dO from shared memory.
    static constexpr bool kKVInTmem = (D == 64);
    static constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256, kColDK = 256 + D;
    static constexpr uint32_t kColK = 384, kColV = 384 + D / 2;
    static_assert(kColDK + D <= (kKVInTmem ? kColK : 512u) && (!kKVInTmem || kColV + D / 2 <= 512u),
                  "TMEM columns");
    // Instruction descriptors (kind::f16, D = f32, A = B = bf16, M = 128):
    //   S^T, dP^T: A K-major, B K-major, N = 128 (queries);
    //   dV, dK:    A from TMEM, B MN-major (dO / Q rows are queries), N = D;
    //   dQ:        A MN-major (dS^T in shared memory), B MN-major (K), N = D.
    static constexpr uint32_t kIdescST = (1u << 4) | (1u << 7) | (1u << 10) | (0u << 15) | (0u << 16) |
                                         ((128u >> 3) << 17) | ((128u >> 4) << 24);
    static constexpr uint32_t kIdescKV = (1u << 4) | (1u << 7) | (1u << 10) | (0u << 15) | (1u << 16) |
                                         (((uint32_t)D >> 3) << 17) | ((128u >> 4) << 24);
    static constexpr uint32_t kIdescQ = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (1u << 16) |
                                        (((uint32_t)D >> 3) << 17) | ((128u >> 4) << 24);
};

template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    fa_bwd_sm100_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                        const __grid_constant__ CUtensorMap tm_dq, const BwdParams p) {
    using C = BwdCfg<D>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw_base = smem_addr(smem_raw);
    const uint32_t base = (raw_base + 1023u) & ~1023u;
    uint8_t* const base_ptr = smem_raw + (base - raw_base);

    auto bar = [&](int i) { return base + C::kBarOff + 8u * (uint32_t)i; };
    const uint32_t bar_kv = bar(0);
    auto bar_q_full = [&](int s) { return bar(1 + s); };
    auto bar_q_empty = [&](int s) { return bar(1 + C::kStagesQ + s); };
    auto bar_o_full = [&](int s) { return bar(1 + 2 * C::kStagesQ + s); };
    auto bar_o_empty = [&](int s) { return bar(1 + 2 * C::kStagesQ + C::kStagesO + s); };
    constexpr int kB0 = 1 + 2 * C::kStagesQ + 2 * C::kStagesO;
    const uint32_t bar_s_full = bar(kB0);
    // P^T / dS^T of one compute pass written (pass h: queries 32h.. and 64 + 32h..)
    auto bar_p_full = [&](int half) { return bar(half == 0 ? kB0 + 1 : kB0 + 5); };
    const uint32_t bar_dq_full = bar(kB0 + 2);
    const uint32_t bar_s_free = bar(kB0 + 3);
    const uint32_t bar_drain = bar(kB0 + 4);
    const uint32_t bar_kv_tmem = bar(kB0 + 6);   // K and V rows copied into TMEM (d = 64)
    uint32_t* const tmem_holder = reinterpret_cast<uint32_t*>(base_ptr + C::kMiscOff);
    volatile int* const abort_flag = reinterpret_cast<volatile int*>(base_ptr + C::kMiscOff + 4);
    float* const rows = reinterpret_cast<float*>(base_ptr + C::kRowOff);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int k0 = (int)blockIdx.x * 128;
    const int h = blockIdx.y;
    const int b = blockIdx.z;
    const size_t bh = (size_t)b * p.H + h;
    int kl = p.Nk;
    if (p.key_lens != nullptr) {
        kl = p.key_lens[b];
        kl = kl < 0 ? 0 : (kl > p.Nk ? p.Nk : kl);
    }
    const int off = p.Nk - p.Nq;   // key j visible to query i iff j <= i + off (causal)
    const int num_m = (p.Nq + 127) / 128;
    // the first query that can see key k0 is k0 - off (causal); all queries otherwise
    int i_lo = 0;
    if (p.causal) {
        const long long f = (long long)k0 - off;
        i_lo = f <= 0 ? 0 : (int)(f / 128 < num_m ? f / 128 : num_m);
    }
    const int n_t = (k0 < kl && i_lo < num_m) ? num_m - i_lo : 0;

    if (warp == kBwdProducerWarp && lane == 0) {
        mbar_init(bar_kv, 1);
        for (int s = 0; s < C::kStagesQ; ++s) {
            mbar_init(bar_q_full(s), 1);
            mbar_init(bar_q_empty(s), 1);
        }
        for (int s = 0; s < C::kStagesO; ++s) {
            mbar_init(bar_o_full(s), 1);
            mbar_init(bar_o_empty(s), 1);
        }
        mbar_init(bar_s_full, 1);
        mbar_init(bar_p_full(0), kBwdComputeWarps);   // one arrival per compute warp and half
        mbar_init(bar_p_full(1), kBwdComputeWarps);
        mbar_init(bar_dq_full, 1);
        mbar_init(bar_s_free, kBwdComputeWarps);
        mbar_init(bar_drain, 1);
        mbar_init(bar_kv_tmem, kBwdComputeWarps);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
        prefetch_tensormap(&tm_do);
        prefetch_tensormap(&tm_dq);
    }
    if (warp == kBwdMmaWarp) {
        tmem_alloc(smem_addr(tmem_holder), 512);
        tmem_relinquish();
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    if (warp == kBwdProducerWarp) {
        // ============================================================ TMA producer
        if (lane == 0 && n_t > 0) {
            const uint64_t pol_keep = policy_evict_last();
            mbar_arrive_expect_tx(bar_kv, 2u * (uint32_t)C::kTileBytes);
            for (int bx = 0; bx < C::kBoxes; ++bx) {
                tma_load_4d(base + C::kKOff + bx * kSwizzleBoxBytes, &tm_k, bar_kv, bx * 64, k0, h, b,
                            policy_evict_first());
                tma_load_4d(base + C::kVOff + bx * kSwizzleBoxBytes, &tm_v, bar_kv, bx * 64, k0, h, b,
                            policy_evict_first());
            }
            bool ok = true;
            int nq = 0, no = 0;   // Q and dO copies issued
            for (int t = 0; t < n_t && ok; ++t) {
                const int q0 = (i_lo + t) * 128;
                const int sq = t % C::kStagesQ;
                ok = wait_bounded(bar_q_empty(sq), (uint32_t)(((t / C::kStagesQ) & 1) ^ 1), abort_flag, p.wait_limit);
                if (!ok) break;
                mbar_arrive_expect_tx(bar_q_full(sq), (uint32_t)C::kTileBytes);
                for (int bx = 0; bx < C::kBoxes; ++bx)
                    tma_load_4d(base + C::kQOff + sq * C::kTileBytes + bx * kSwizzleBoxBytes, &tm_q, bar_q_full(sq),
                                bx * 64, q0, h, b, pol_keep);
                ++nq;
                const int so = t % C::kStagesO;
                ok = wait_bounded(bar_o_empty(so), (uint32_t)(((t / C::kStagesO) & 1) ^ 1), abort_flag, p.wait_limit);
                if (!ok) break;
                mbar_arrive_expect_tx(bar_o_full(so), (uint32_t)C::kTileBytes);
                for (int bx = 0; bx < C::kBoxes; ++bx)
                    tma_load_4d(base + C::kDOOff + so * C::kTileBytes + bx * kSwizzleBoxBytes, &tm_do, bar_o_full(so),
                                bx * 64, q0, h, b, pol_keep);
                ++no;
            }
            // wind down: every copy issued lands before the CTA exits, also when a
            // consumer gave up after this producer issued its last copy (the waits
            // ignore the abort flag and keep the default limit, whatever the
            // caller's; on the normal path the phases are complete already).  Only
            // the newest copy of each slot can still be in flight.
            (void)wait_own_work(bar_kv, 0);
            for (int c2 = (nq > C::kStagesQ ? nq - C::kStagesQ : 0); c2 < nq; ++c2)
                (void)wait_own_work(bar_q_full(c2 % C::kStagesQ), (uint32_t)((c2 / C::kStagesQ) & 1));
            for (int c2 = (no > C::kStagesO ? no - C::kStagesO : 0); c2 < no; ++c2)
                (void)wait_own_work(bar_o_full(c2 % C::kStagesO), (uint32_t)((c2 / C::kStagesO) & 1));
        }
        __syncwarp();
    } else if (warp == kBwdMmaWarp) {
        // ============================================================ MMA issuer
        if (lane == 0 && n_t > 0) {
            bool ok = wait_bounded(bar_kv, 0, abort_flag, p.wait_limit);
            if (C::kKVInTmem && ok) ok = wait_bounded(bar_kv_tmem, 0, abort_flag, p.wait_limit);
            const uint32_t k_s = base + C::kKOff, v_s = base + C::kVOff, ds_s = base + C::kDSOff;
            for (int t = 0; t < n_t && ok; ++t) {
                const int sq = t % C::kStagesQ, so = t % C::kStagesO;
                ok = wait_bounded(bar_q_full(sq), (uint32_t)((t / C::kStagesQ) & 1), abort_flag, p.wait_limit);
                // the previous tile's dQ has been read out of the S columns
                if (ok && t > 0) ok = wait_bounded(bar_s_free, (uint32_t)((t - 1) & 1), abort_flag, p.wait_limit);
                if (!ok) break;
                tc_fence_after();
                const uint32_t q_s = base + C::kQOff + sq * C::kTileBytes;
                const uint32_t do_s = base + C::kDOOff + so * C::kTileBytes;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {   // S^T = K Q^T
                    const uint32_t koff = (uint32_t)((kk / 4) * kSwizzleBoxBytes + (kk % 4) * 32);
                    if constexpr (C::kKVInTmem)
                        umma_ts(tmem + C::kColS, tmem + C::kColK + 8u * (uint32_t)kk,
                                smem_desc_sw128(q_s + koff, 16, 1024), C::kIdescST, kk > 0 ? 1u : 0u);
                    else
                        umma_ss(tmem + C::kColS, smem_desc_sw128(k_s + koff, 16, 1024),
                                smem_desc_sw128(q_s + koff, 16, 1024), C::kIdescST, kk > 0 ? 1u : 0u);
                }
                // dO_i may land after Q_i (its slot frees when the previous tile's dV is done)
                ok = wait_bounded(bar_o_full(so), (uint32_t)((t / C::kStagesO) & 1), abort_flag, p.wait_limit);
                if (!ok) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {   // dP^T = V dO^T
                    const uint32_t koff = (uint32_t)((kk / 4) * kSwizzleBoxBytes + (kk % 4) * 32);
                    if constexpr (C::kKVInTmem)
                        umma_ts(tmem + C::kColDP, tmem + C::kColV + 8u * (uint32_t)kk,
                                smem_desc_sw128(do_s + koff, 16, 1024), C::kIdescST, kk > 0 ? 1u : 0u);
                    else
                        umma_ss(tmem + C::kColDP, smem_desc_sw128(v_s + koff, 16, 1024),
                                smem_desc_sw128(do_s + koff, 16, 1024), C::kIdescST, kk > 0 ? 1u : 0u);
                }
                umma_commit(bar_s_full);
                // dV and dK for the queries of each pass as soon as the compute warps
                // have written that pass's P^T and dS^T: the first pass's products
                // overlap the second pass's exponentials.  Pass h covers the query
                // blocks 32cb.. with cb = h and 2 + h, i.e. kk = 2h, 2h+1, 2h+4, 2h+5;
                // P^T of queries 16kk.. sits at column 32(kk/2) + 8(kk%2) (dS^T
                // likewise from kColDP).
#pragma unroll 1
                for (int half = 0; half < 2 && ok; ++half) {
                    ok = wait_bounded(bar_p_full(half), (uint32_t)(t & 1), abort_flag, p.wait_limit);
                    if (!ok) break;
                    tc_fence_after();
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4) {   // dV += P^T dO: 16 queries per step
                        const int kk = 4 * (k4 / 2) + 2 * half + (k4 % 2);
                        umma_ts(tmem + C::kColDV, tmem + C::kColS + (uint32_t)(32 * (kk / 2) + 8 * (kk % 2)),
                                smem_desc_sw128(do_s + (uint32_t)(kk * 16 * 128), kSwizzleBoxBytes, 1024),
                                C::kIdescKV, (t > 0 || kk > 0) ? 1u : 0u);
                    }
                    if (half == 1) umma_commit(bar_o_empty(so));   // dO_i is no longer read
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4) {   // dK += dS^T Q
                        const int kk = 4 * (k4 / 2) + 2 * half + (k4 % 2);
                        umma_ts(tmem + C::kColDK, tmem + C::kColDP + (uint32_t)(32 * (kk / 2) + 8 * (kk % 2)),
                                smem_desc_sw128(q_s + (uint32_t)(kk * 16 * 128), kSwizzleBoxBytes, 1024),
                                C::kIdescKV, (t > 0 || kk > 0) ? 1u : 0u);
                    }
                }
                if (!ok) break;
                umma_commit(bar_q_empty(sq));   // Q_i is no longer read
#pragma unroll
                for (int kk = 0; kk < 128 / 16; ++kk) {   // dQ = dS K: 16 keys per step
                    umma_ss(tmem + C::kColS, smem_desc_sw128(ds_s + (uint32_t)(kk * 16 * 128), kSwizzleBoxBytes, 1024),
                            smem_desc_sw128(k_s + (uint32_t)(kk * 16 * 128), kSwizzleBoxBytes, 1024), C::kIdescQ,
                            kk > 0 ? 1u : 0u);
                }
                umma_commit(bar_dq_full);
            }
            // every MMA issued has completed before TMEM is released (also after a
            // give-up; this wait ignores the abort flag and the caller's limit)
            umma_commit(bar_drain);
            (void)wait_own_work(bar_drain, 0);
        }
        __syncwarp();
    } else if (warp >= kBwdComputeWarp0) {
        // ============================================================ P, dS, dQ, and the epilogue
        const int qd = warp & 3;                  // TMEM lane quadrant
        const int g = (warp - kBwdComputeWarp0) >> 2;   // which half of the columns this warp takes
        const int r = qd * 32 + lane;             // key row in the block (S^T lanes) / query row (dQ lanes)
        const uint32_t lane_off = (uint32_t)(qd * 32) << 16;
        const int k = k0 + r;
        const bool key_ok = k < kl;
        const float c = p.scale_log2;
        bool ok = true;
        // query row r of tile t: its LSE and D from global memory (warps of half 0 only),
        // fetched one tile ahead so that the loads' latency overlaps a tile's work
        float lse_next = -INFINITY, d_next = 0.f;
        auto fetch_rows = [&](int t) {
            const int q = (i_lo + t) * 128 + r;
            if (g == 0 && t < n_t && q < p.Nq) {
                lse_next = p.lse[bh * (size_t)p.Nq + q];
                d_next = p.dsum[bh * (size_t)p.Nq + q];
            } else {
                lse_next = -INFINITY;
                d_next = 0.f;
            }
        };
        fetch_rows(0);
        if (C::kKVInTmem && n_t > 0) {
            // key row r of K (warps of half 0) or V (half 1) from the swizzled tile
            // (16-byte chunk c of row r at c ^ (r % 8)) into this lane's TMEM row: column
            // j holds elements 2j and 2j + 1, the A-operand layout of the MMAs
            const bool good = wait_bounded(bar_kv, 0, abort_flag, p.wait_limit);
            if (__all_sync(0xffffffffu, good)) {
                const uint32_t src = base + (g == 0 ? C::kKOff : C::kVOff) + (uint32_t)(r * 128);
                uint32_t w[32];
#pragma unroll
                for (int c4 = 0; c4 < 8; ++c4)
                    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                                 : "=r"(w[4 * c4]), "=r"(w[4 * c4 + 1]), "=r"(w[4 * c4 + 2]), "=r"(w[4 * c4 + 3])
                                 : "r"(src + (uint32_t)((c4 ^ (r & 7)) << 4))
                                 : "memory");
                tmem_st32(tmem + lane_off + (g == 0 ? C::kColK : C::kColV), w);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_kv_tmem);
            } else {
                ok = false;
            }
        }
        for (int t = 0; t < n_t; ++t) {
            const int i0 = (i_lo + t) * 128;
            float* const rb = rows + (t & 1) * 256;
            if (g == 0) {
                // the row's LSE in log2 units (+inf when the row sees no key, or lies
                // past N_q) and D
                rb[r] = (lse_next == -INFINITY) ? INFINITY : lse_next * 1.4426950408889634f;
                rb[128 + r] = d_next;
            }
            fetch_rows(t + 1);
            // all four warps wrote the tile's row data; leave together if any gave up
            if (named_bar_or(kBwdBarCompute, 32 * kBwdComputeWarps, !ok)) break;
            bool good = wait_bounded(bar_s_full, (uint32_t)(t & 1), abort_flag, p.wait_limit);
            if (!__all_sync(0xffffffffu, good)) {
                ok = false;
                continue;
            }
            tc_fence_after();
            // this key row sees every query of the tile (no per-element mask)
            const bool row_full = key_ok && (!p.causal || k <= i0 + off);
            // ... for every row of the warp, and no query row of the tile lies past N_q
            const bool warp_full = __all_sync(0xffffffffu, row_full) && i0 + 128 <= p.Nq;
            // the previous tile's dQ reduce (issued by this warp's lane 0) has read its
            // staging, part of which is the dS^T box written below
            if (lane == 0) bulk_wait_group_read0();
            __syncwarp();
#pragma unroll 1
            for (int pass = 0; pass < 2; ++pass) {
                // queries 32cb .. 32cb+31: each warp stays inside its own 64 queries, so
                // its dS^T goes only to box g, where it alone stages dQ
                const int cb = 2 * g + pass;
                uint32_t su[32], du[32];
                tmem_ld32(tmem + lane_off + C::kColS + 32u * cb, su);
                tmem_ld32(tmem + lane_off + C::kColDP + 32u * cb, du);
                // the 32 queries' LSE (log2 units) and D, same for every lane: 16-byte
                // shared-memory loads while the TMEM loads are in flight
                float lq[32], dq[32];
                {
                    const uint32_t ra = smem_addr(rb + 32 * cb);
#pragma unroll
                    for (int i4 = 0; i4 < 8; ++i4) {
                        ld_shared_v4(ra + 16u * i4, lq[4 * i4], lq[4 * i4 + 1], lq[4 * i4 + 2], lq[4 * i4 + 3]);
                        ld_shared_v4(ra + 512u + 16u * i4, dq[4 * i4], dq[4 * i4 + 1], dq[4 * i4 + 2], dq[4 * i4 + 3]);
                    }
                }
                tmem_wait_ld();
                uint32_t pw[16], dw[16];
                const int qa0 = i0 + 32 * cb;
                // one pair in four of the exponentials on the FMA pipe (MUFU is the
                // busiest unit here), where every score of the warp is visible and
                // finite (2^x is then the same up to rounding and a 2^-125 floor)
                auto body = [&](auto emu_tag) {
                    constexpr bool kEmu = decltype(emu_tag)::value;
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        reg_after_wait(su[e]);
                        reg_after_wait(su[e + 1]);
                        reg_after_wait(du[e]);
                        reg_after_wait(du[e + 1]);
                        // log2-domain score minus LSE, then P = 2^x and dS = P (dP - D)
                        const float2 x = __ffma2_rn(make_float2(__uint_as_float(su[e]), __uint_as_float(su[e + 1])),
                                                    make_float2(c, c), make_float2(-lq[e], -lq[e + 1]));
                        float p0, p1;
                        if (kEmu && (e & 6) == 6) {
                            const float2 pe = exp2_fma2(x);
                            p0 = pe.x;
                            p1 = pe.y;
                        } else {
                            p0 = ex2_approx(x.x);
                            p1 = ex2_approx(x.y);
                        }
                        if (!kEmu && !row_full) {
                            const bool v0 = key_ok && k <= qa0 + e + off;
                            const bool v1 = key_ok && k <= qa0 + e + 1 + off;
                            p0 = v0 ? p0 : 0.f;
                            p1 = v1 ? p1 : 0.f;
                        }
                        const float2 ds =
                            __fmul2_rn(make_float2(p0, p1),
                                       __fadd2_rn(make_float2(__uint_as_float(du[e]), __uint_as_float(du[e + 1])),
                                                  make_float2(-dq[e], -dq[e + 1])));
                        pw[e >> 1] = pack_bf16x2(p0, p1);
                        dw[e >> 1] = pack_bf16x2(ds.x, ds.y);
                    }
                };
                if (warp_full)
                    body(std::true_type{});
                else
                    body(std::false_type{});
                // P^T over the first 16 of the 32 S^T columns this warp has just read
                // (32cb..), dS^T likewise over dP^T's: no other warp reads them
                tmem_st16(tmem + lane_off + C::kColS + 32u * cb, pw);
                tmem_st16(tmem + lane_off + C::kColDP + 32u * cb, dw);
                // dS^T row r into shared memory: box cb/2 holds queries 64(cb/2)..+63 as
                // 128-byte rows, 16-byte chunk cc at swizzled position cc ^ (r % 8)
#pragma unroll
                for (int t4 = 0; t4 < 4; ++t4) {
                    const int cc = (cb & 1) * 4 + t4;
                    const uint32_t a = base + C::kDSOff + (uint32_t)((cb >> 1) * kSwizzleBoxBytes + r * 128 +
                                                                     ((cc ^ (r & 7)) << 4));
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(dw[4 * t4]),
                                 "r"(dw[4 * t4 + 1]), "r"(dw[4 * t4 + 2]), "r"(dw[4 * t4 + 3])
                                 : "memory");
                }
                tmem_wait_st();
                fence_proxy_async_smem();   // dS^T visible to the tensor core
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_p_full(pass));
            }
            // dQ_i (TMEM lane = query row i0 + r) into the fp32 accumulator
            good = wait_bounded(bar_dq_full, (uint32_t)(t & 1), abort_flag, p.wait_limit);
            if (!__all_sync(0xffffffffu, good)) {
                ok = false;
                continue;
            }
            tc_fence_after();
            {
                uint32_t u[D / 2];   // this warp's half of dQ row i0 + r
#pragma unroll
                for (int c2 = 0; c2 < D / 64; ++c2)
                    tmem_ld32(tmem + lane_off + C::kColS + 32u * (uint32_t)(g * (D / 64) + c2),
                              *reinterpret_cast<uint32_t(*)[32]>(&u[32 * c2]));
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < D / 2; ++i) reg_after_wait(u[i]);
                // dQ_i is in registers: the next tile's S^T may take its TMEM columns
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_s_free);
                // stage row r of this warp's boxes (32 fp32 columns each, 128-byte rows,
                // 16-byte chunk cc at cc ^ (r % 8)) and add them into the fp32
                // accumulator with one tensor reduce per box: rows past N_q are outside
                // the tensor and skipped
#pragma unroll
                for (int c2 = 0; c2 < D / 64; ++c2) {
                    const uint32_t box = base + (c2 == 0 ? C::kDSOff : C::kDQ2Off) + (uint32_t)(g * kSwizzleBoxBytes);
#pragma unroll
                    for (int cc = 0; cc < 8; ++cc) {
                        const uint32_t a = box + (uint32_t)(r * 128 + ((cc ^ (r & 7)) << 4));
                        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(u[32 * c2 + 4 * cc]),
                                     "r"(u[32 * c2 + 4 * cc + 1]), "r"(u[32 * c2 + 4 * cc + 2]),
                                     "r"(u[32 * c2 + 4 * cc + 3])
                                     : "memory");
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
#pragma unroll
                    for (int c2 = 0; c2 < D / 64; ++c2) {
                        const uint32_t box =
                            base + (c2 == 0 ? C::kDSOff : C::kDQ2Off) + (uint32_t)(g * kSwizzleBoxBytes);
                        tma_reduce_add_3d(&tm_dq, box + (uint32_t)(qd * 32 * 128), (g * (D / 64) + c2) * 32,
                                          i0 + qd * 32, (int)bh);
                    }
                    bulk_commit_group();
                }
            }
        }
        // every dQ reduce this warp issued has completed before the CTA exits
        if (lane == 0) bulk_wait_group0();
        __syncwarp();
        // ------------------------------------------------------------ dV, dK -> bf16
        bool have = n_t > 0;
        if (have && ok) {
            const bool good = wait_bounded(bar_drain, 0, abort_flag, p.wait_limit);
            ok = __all_sync(0xffffffffu, good);
            if (ok) tc_fence_after();
        }
        // tcgen05.ld is warp-collective: every lane loads (ok is warp-uniform), and
        // only the stores are limited to keys < N_k
        if (ok) {
#pragma unroll 1
            for (int which = 0; which < 2; ++which) {
                __nv_bfloat16* const out = which == 0 ? p.dv : p.dk;
                const uint32_t col = which == 0 ? C::kColDV : C::kColDK;
                const float f = which == 0 ? 1.f : p.scale;
#pragma unroll 1
                for (int c2 = g * (D / 64); c2 < (g + 1) * (D / 64); ++c2) {
                    uint32_t u[32];
                    if (have) {
                        tmem_ld32(tmem + lane_off + col + 32u * c2, u);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i) reg_after_wait(u[i]);
                    } else {
#pragma unroll
                        for (int i = 0; i < 32; ++i) u[i] = 0u;
                    }
                    if (k >= p.Nk) continue;
                    uint4* dst = reinterpret_cast<uint4*>(out + (bh * (size_t)p.Nk + k) * D + 32 * c2);
#pragma unroll
                    for (int v4 = 0; v4 < 4; ++v4) {
                        uint4 w4;
                        w4.x = pack_bf16x2(__uint_as_float(u[8 * v4]) * f, __uint_as_float(u[8 * v4 + 1]) * f);
                        w4.y = pack_bf16x2(__uint_as_float(u[8 * v4 + 2]) * f, __uint_as_float(u[8 * v4 + 3]) * f);
                        w4.z = pack_bf16x2(__uint_as_float(u[8 * v4 + 4]) * f, __uint_as_float(u[8 * v4 + 5]) * f);
                        w4.w = pack_bf16x2(__uint_as_float(u[8 * v4 + 6]) * f, __uint_as_float(u[8 * v4 + 7]) * f);
                        dst[v4] = w4;
                    }
                }
            }
        }
        tc_fence_before();
    }

    __syncthreads();
    if (warp == kBwdMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// D_i = dO_i . O_i (fp32) for every query row, and the dQ accumulator row zeroed.
// One warp per row.
template <int D>
__global__ void __launch_bounds__(256)
    fa_bwd_pre_kernel(const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ dout,
                      float* __restrict__ dsum, float* __restrict__ dq_acc, long long rows) {
    const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    constexpr int kPer = D / 32;   // consecutive columns per lane
    const __nv_bfloat16* po = o + row * D + lane * kPer;
    const __nv_bfloat16* pd = dout + row * D + lane * kPer;
    float acc = 0.f;
#pragma unroll
    for (int i = 0; i < kPer; ++i) acc = fmaf(__bfloat162float(po[i]), __bfloat162float(pd[i]), acc);
#pragma unroll
    for (int sh = 16; sh > 0; sh >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, sh);
    if (lane == 0) dsum[row] = acc;
    float* z = dq_acc + row * D + lane * kPer;
#pragma unroll
    for (int i = 0; i < kPer; ++i) z[i] = 0.f;
}

// dQ = bf16(scale * dQ accumulator), 8 elements per thread.
__global__ void __launch_bounds__(256)
    fa_bwd_post_kernel(const float* __restrict__ dq_acc, __nv_bfloat16* __restrict__ dq, float scale, long long n8) {
    const long long i = (long long)blockIdx.x * 256 + threadIdx.x;
    if (i >= n8) return;
    const float4 a = reinterpret_cast<const float4*>(dq_acc)[2 * i];
    const float4 b2 = reinterpret_cast<const float4*>(dq_acc)[2 * i + 1];
    uint4 w;
    w.x = pack_bf16x2(a.x * scale, a.y * scale);
    w.y = pack_bf16x2(a.z * scale, a.w * scale);
    w.z = pack_bf16x2(b2.x * scale, b2.y * scale);
    w.w = pack_bf16x2(b2.z * scale, b2.w * scale);
    reinterpret_cast<uint4*>(dq)[i] = w;
}

}  // namespace fa
