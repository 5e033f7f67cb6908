// fa_fwd_persist.cuh -- the dense forward as a persistent CTA.
//
// Same computation, roles, barriers and per-tile arithmetic as
// fa_fwd_sm100_kernel (fa_fwd_kernel.cuh) in its dense single-pass mode; the
// difference is the life of a CTA.  The grid is the same (one CTA per (b, h,
// 128-row query block), heaviest causal blocks first), but a running CTA does
// not exit after its block: once it has issued the last K copy of its block it
// asks the hardware scheduler to cancel the launch of a CTA of the grid that
// has not started yet (clusterlaunchcontrol.try_cancel) and takes over that
// CTA's block.  So a CTA pays its setup (barriers, TMEM, the ones boxes) once,
// and the next block's Q and first K/V copies and its first QK^T product
// overlap this block's last tiles and epilogue.  Claiming only near the end of
// a block keeps the assignment close to the hardware's own (the next block goes
// to a CTA that is about to need one); no global counter is involved, so two
// launches in flight never share scheduling state.
//
// What changes against the single-block kernel:
//  * every barrier phase is counted over all the blocks a CTA has taken, not
//    per block;
//  * the next block's Q copy waits until the QK^T products of this block have
//    read Q (q_free, committed by the QK issuer after its last product);
//  * the next block's first PV product (which starts O afresh) waits until the
//    softmax warps have read this block's O and row sums out of TMEM (o_free);
//  * only the PV issuer commits the per-block drain (its last product
//    completing implies every product of the block has);
//  * O is written from registers with plain 16-byte stores (no staging in the
//    Q buffer, which the next block's copy may already be filling);
//  * warp 8's producer lane also runs the scheduler: one cancel request at a
//    time; it decodes the answer into a whole item (FwdItem) and publishes it
//    to the other roles through a two-slot mailbox (item_ready / item_used).
// Every wait is bounded, as in the single-block kernel.
#pragma once

#include "fa_fwd_kernel.cuh"

namespace fa {

// One (b, h, 128-row query block) problem of the dense forward.
struct FwdItem {
    int h, b;
    int m0;     // first query row
    int kl;     // visible key count of sequence b (key_lens clamped)
    int off;    // causal diagonal offset N_k - N_q
    int t0;     // first K/V tile to visit
    int n_kv;   // K/V tiles to visit
};

// The block of blockIdx (bx, by, bz), with the heaviest-first causal order and
// the L2 head groups of the single-block kernel.
__device__ __forceinline__ FwdItem make_fwd_item(const FwdParams& p, int bx, int by, int bz, int num_m) {
    int blk = bx, h = by, b = bz;
    if (p.head_group > 1) {
        const int HB = p.H * p.B;
        const int lin = bx + num_m * (by + p.H * bz);
        const int per_group = num_m * p.head_group;
        const int gi = lin / per_group;
        const int w = lin - gi * per_group;
        const int hcnt = min(p.head_group, HB - gi * p.head_group);
        blk = w / hcnt;
        const int hb = gi * p.head_group + (w - blk * hcnt);
        h = hb % p.H;
        b = hb / p.H;
    }
    FwdItem it;
    it.h = h;
    it.b = b;
    const int m_blk = p.causal ? (num_m - 1 - blk) : blk;
    it.m0 = m_blk * kBlockM;
    int kl = p.Nk;
    if (p.key_lens != nullptr) {
        kl = p.key_lens[b];
        kl = kl < 0 ? 0 : (kl > p.Nk ? p.Nk : kl);
    }
    it.kl = kl;
    it.off = p.Nk - p.Nq;
    const int last_row = min(it.m0 + kBlockM - 1, p.Nq - 1);
    const int n_all = (row_key_limit(last_row, kl, it.off, p.causal) + kBlockN - 1) / kBlockN;
    const int t_lo = min(row_key_start(it.m0, it.off, p.window_left) / kBlockN, n_all);
    it.t0 = t_lo;
    it.n_kv = n_all - t_lo;
    return it;
}

template <int D, bool kF8>
struct PersistCfg {
    using C = Cfg<D, kF8>;
    // after the single-block kernel's shared memory: 10 barriers (q_free, o_free,
    // drain, fin, clc[2] (one in use), item_ready[2], item_used[2]), two 16-byte cancel
    // responses, a two-slot mailbox of whole items (FwdItem + valid), and the epilogue
    // exchange (m, lu [parity][row]) twice, alternating between blocks
    static constexpr int kExtraOff = (C::kSmemUsed - 1024 + 127) / 128 * 128;
    static constexpr int kNumBars = 10;
    static constexpr int kRespOff = kExtraOff + kNumBars * 8;
    static constexpr int kMailOff = kRespOff + 32;
    static constexpr int kEpiOff = kMailOff + 2 * 32;
    static constexpr int kEpiFloats = 2 * kGroups * kBlockM;
    static constexpr int kUsed = kEpiOff + 2 * kEpiFloats * 4 + 1024;   // + alignment slack
    // at least the single-block kernel's reservation: one CTA per SM (it holds
    // all 512 TMEM columns for its whole life)
    static constexpr int kSmemBytes = kUsed > C::kSmemBytes ? kUsed : C::kSmemBytes;
    static_assert(kSmemBytes <= 232448, "dynamic shared memory per CTA on sm_100");
    // s_full is indexed by the block-local tile parity and the score buffer by the
    // CTA-wide tile count; with one score buffer every QK^T waits for the previous
    // tile's S to be read, so s_full(g) never completes twice ahead of group g
    // across a block boundary (two buffers would allow that)
    static_assert(C::kSBufs == 1, "one TMEM score buffer");
};

template <int D, bool kF8 = false, int kBias = kBiasNone>
__global__ void __launch_bounds__(kNumThreads, 1)
    fa_fwd_persist_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
    using C = Cfg<D, kF8>;
    using PC = PersistCfg<D, kF8>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw_base = smem_addr(smem_raw);
    const uint32_t base = (raw_base + 1023u) & ~1023u;
    uint8_t* const base_ptr = smem_raw + (base - raw_base);

    // the single-block kernel's barriers (its drain slot is not used here)
    const uint32_t bar_q_full = base + C::kBarOff;
    auto bar_full = [&](int r, int s) { return base + C::kBarOff + 8u * (1 + r * C::kStagesK + s); };
    auto bar_empty = [&](int r, int s) { return base + C::kBarOff + 8u * (1 + C::kStages + r * C::kStagesK + s); };
    auto bar_s_full = [&](int g) { return base + C::kBarOff + 8u * (1 + 2 * C::kStages + g); };
    auto bar_s_free = [&](int b) { return base + C::kBarOff + 8u * (3 + 2 * C::kStages + b); };
    auto bar_p_full = [&](int b) { return base + C::kBarOff + 8u * (5 + 2 * C::kStages + b); };
    auto bar_pv_done = [&](int b) { return base + C::kBarOff + 8u * (8 + 2 * C::kStages + b); };
    // the persistent kernel's own
    const uint32_t bar_q_free = base + PC::kExtraOff;            // QK^T products of a block have read Q
    const uint32_t bar_o_free = base + PC::kExtraOff + 8;        // O and its row sums read out of TMEM
    const uint32_t bar_drain = base + PC::kExtraOff + 16;        // every product of a block has landed
    const uint32_t bar_fin = base + PC::kExtraOff + 24;          // both issuers' last products (wind-down)
    auto bar_clc = [&](int s) { return base + PC::kExtraOff + 32u + 8u * s; };
    auto bar_item_ready = [&](int s) { return base + PC::kExtraOff + 48u + 8u * s; };
    auto bar_item_used = [&](int s) { return base + PC::kExtraOff + 64u + 8u * s; };
    auto clc_resp = [&](int s) { return base + PC::kRespOff + 16u * s; };
    // [2] {h, b, m0, kl, off, t0, n_kv, valid}: the scheduler decodes the item once
    int* const mailbox = reinterpret_cast<int*>(base_ptr + PC::kMailOff);
    uint32_t* const tmem_holder = reinterpret_cast<uint32_t*>(base_ptr + C::kMiscOff);
    volatile int* const abort_flag = reinterpret_cast<volatile int*>(base_ptr + C::kMiscOff + 4);
    // [parity][row]: {tile over all blocks, reference max} words (wait_tagged_max)
    const uint32_t mref_w = base + C::kMrefOff;
    float* const epi2 = reinterpret_cast<float*>(base_ptr + PC::kEpiOff);     // [block parity][m, lu][parity][row]
    const uint32_t q_tile = base + C::kQOff;
    auto ring_slot = [&](int r, int s) {
        return r == 0 ? base + C::kKOff + (uint32_t)(s * C::kTileBytes)
                      : base + C::kVOff + (uint32_t)(s * C::kVSlotBytes);
    };
    // roles that read the mailbox: V producer, both issuers, 8 softmax warps
    constexpr int kMailReaders = 3 + kSoftmaxWarps;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int num_m = (int)gridDim.x;
    const FwdItem first = make_fwd_item(p, (int)blockIdx.x, (int)blockIdx.y, (int)blockIdx.z, num_m);

    // ---- setup: barriers (producer lane 0), TMEM (MMA warp), ones boxes
    if (warp == kProducerWarp && lane == 0) {
        mbar_init(bar_q_full, 1);
        for (int r2 = 0; r2 < 2; ++r2)
            for (int s = 0; s < (r2 == 0 ? C::kStagesK : C::kStagesV); ++s) {
                mbar_init(bar_full(r2, s), 1);
                mbar_init(bar_empty(r2, s), 1);
            }
        for (int g = 0; g < 2; ++g) {
            mbar_init(bar_s_full(g), 1);
            mbar_init(bar_s_free(g), 4);
        }
        for (int b2 = 0; b2 < C::kPBufs; ++b2) {
            mbar_init(bar_p_full(b2), 4);
            mbar_init(bar_pv_done(b2), 1);
        }
        mbar_init(bar_q_free, 1);
        mbar_init(bar_o_free, kSoftmaxWarps);
        mbar_init(bar_drain, 1);
        mbar_init(bar_fin, 2);
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar_clc(s), 1);
            mbar_init(bar_item_ready(s), 1);
            mbar_init(bar_item_used(s), kMailReaders);
        }
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
    }
    if (warp == kMmaWarp) {
        tmem_alloc(smem_addr(tmem_holder), kTmemCols);
        tmem_relinquish();
        tc_fence_before();
    }
    for (int i = threadIdx.x; i < C::kStagesV * (C::kBoxBytes / 16); i += kNumThreads) {
        const int sl = i / (C::kBoxBytes / 16);
        const uint32_t a = ring_slot(1, sl) + (uint32_t)C::kTileBytes + (uint32_t)(i % (C::kBoxBytes / 16)) * 16u;
        asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(a), "r"(C::kOnesWord) : "memory");
    }
    // no reference max published yet: tag 0xffffffff names no tile
    for (int i = threadIdx.x; i < kGroups * kBlockM; i += kNumThreads)
        st_relaxed_shared_u64(mref_w + 8u * (uint32_t)i, ~0ull);
    fence_proxy_async_smem();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    // The next block of a mailbox reader (k = blocks taken so far): wait for the
    // scheduler's answer for block k+1 and hand the slot back; returns 1 with the
    // item, 0 when the scheduler has none, -1 when the wait ran out.  One lane waits, reads and
    // arrives; with whole_warp the answer is broadcast to the other lanes, so
    // that the warp takes the same branch.  The single-lane roles (producer
    // and issuer lanes) call it with whole_warp = false from their own lane.
    auto next_item = [&](int k, FwdItem& it, bool whole_warp) -> int {
        const int s = k & 1;
        int m[8] = {0, 0, 0, 0, 0, 0, 0, -1};   // m[7]: 1 item, 0 none, -1 the wait ran out
        if (!whole_warp || lane == 0) {
            if (wait_bounded(bar_item_ready(s), (uint32_t)((k >> 1) & 1), abort_flag, p.wait_limit)) {
                const volatile int* mv = mailbox + 8 * s;
#pragma unroll
                for (int i = 0; i < 8; ++i) m[i] = mv[i];
            }
            mbar_arrive(bar_item_used(s));
        }
        if (whole_warp) {
#pragma unroll
            for (int i = 0; i < 8; ++i) m[i] = __shfl_sync(0xffffffffu, m[i], 0);
        }
        if (m[7] <= 0) return m[7];
        it.h = m[0];
        it.b = m[1];
        it.m0 = m[2];
        it.kl = m[3];
        it.off = m[4];
        it.t0 = m[5];
        it.n_kv = m[6];
        return 1;
    };

    if (warp >= kProducerWarp) {
      setmaxnreg_dec<kRegsControl>();
      if (warp == kProducerWarp || warp == kVProducerWarp) {
        // =========================================================== TMA producers (+ scheduler)
        const int rg = (warp == kProducerWarp) ? 0 : 1;
        const CUtensorMap* const tm = (rg == 0) ? &tm_k : &tm_v;
        const int ns = (rg == 0) ? C::kStagesK : C::kStagesV;
        if (lane == 0) {
            const uint64_t pol_kv = policy_evict_last();
            const uint64_t pol_q = policy_evict_first();
            FwdItem it = first;
            int jr = 0;          // ring copies issued over all blocks
            int nq = 0;          // Q copies issued (blocks with K/V tiles)
            int clc_out = 0;     // cancel requests issued
            int clc_done = 0;    // ... and answered
            bool ok = true;
            for (int k = 0; ok; ++k) {
                if (it.n_kv > 0) {
                    if (rg == 0) {
                        // the previous block's QK^T products have read Q
                        if (nq > 0) ok = wait_bounded(bar_q_free, (uint32_t)((nq - 1) & 1), abort_flag, p.wait_limit);
                        if (!ok) break;
                        mbar_arrive_expect_tx(bar_q_full, (uint32_t)C::kTileBytes);
                        for (int bx = 0; bx < C::kBoxes; ++bx)
                            tma_load_4d(q_tile + bx * C::kBoxBytes, &tm_q, bar_q_full, bx * C::kBoxCols, it.m0, it.h,
                                        it.b, pol_q);
                        ++nq;
                    }
                    for (int j = 0; j < it.n_kv && ok; ++j, ++jr) {
                        const int s = jr % ns;
                        ok = wait_bounded(bar_empty(rg, s), (uint32_t)(((jr / ns) & 1) ^ 1), abort_flag, p.wait_limit);
                        if (!ok) break;
                        mbar_arrive_expect_tx(bar_full(rg, s), (uint32_t)C::kTileBytes);
                        for (int bx = 0; bx < C::kBoxes; ++bx)
                            tma_load_4d(ring_slot(rg, s) + bx * C::kBoxBytes, tm, bar_full(rg, s), bx * C::kBoxCols,
                                        (it.t0 + j) * kBlockN, it.h, it.b, pol_kv);
                    }
                    if (!ok) break;
                }
                if (rg == 0) {
                    // scheduler: claim block k+1 now that every K copy of block k is
                    // issued (a few tiles before this block ends), so that blocks go
                    // to the CTAs that are about to need one, close to the order in
                    // which the hardware would have started them
                    mbar_arrive_expect_tx(bar_clc(0), 16u);
                    clc_try_cancel(clc_resp(0), bar_clc(0));
                    clc_out = k + 1;
                    ok = wait_bounded(bar_clc(0), (uint32_t)(k & 1), abort_flag, p.wait_limit);
                    if (!ok) break;
                    clc_done = k + 1;
                    int x = 0, y = 0, z = 0;
                    bool got = clc_query(clc_resp(0), x, y, z);
                    if (got && (x < 0 || x >= (int)gridDim.x || y < 0 || y >= (int)gridDim.y || z < 0 ||
                                z >= (int)gridDim.z)) {
                        // not a block of this grid: take no more work, and say so
                        got = false;
                        atomicExch(&g_fa_status, kStatusTimeout);
                    }
                    if (got) it = make_fwd_item(p, x, y, z, num_m);
                    // mailbox slot s last carried block k-1's successor: every reader must be done with it
                    const int s = k & 1;
                    if (k >= 2) ok = wait_bounded(bar_item_used(s), (uint32_t)(((k - 2) >> 1) & 1), abort_flag,
                                                  p.wait_limit);
                    if (!ok) break;
                    int* const mw = mailbox + 8 * s;
                    mw[0] = it.h;
                    mw[1] = it.b;
                    mw[2] = it.m0;
                    mw[3] = it.kl;
                    mw[4] = it.off;
                    mw[5] = it.t0;
                    mw[6] = it.n_kv;
                    mw[7] = got ? 1 : 0;
                    mbar_arrive(bar_item_ready(s));   // release: the mailbox writes above are visible
                    if (!got) break;
                } else {
                    if (next_item(k, it, false) <= 0) break;
                }
            }
            // wind-down: every copy this producer issued that may still be in
            // flight (the last Q, the newest copy of each slot) and an
            // unanswered cancel request must have landed before the CTA exits
            if (rg == 0 && nq > 0) (void)wait_own_work(bar_q_full, (uint32_t)((nq - 1) & 1));
            for (int c2 = (jr > ns ? jr - ns : 0); c2 < jr; ++c2)
                (void)wait_own_work(bar_full(rg, c2 % ns), (uint32_t)((c2 / ns) & 1));
            for (int c = clc_done; c < clc_out; ++c) (void)wait_own_work(bar_clc(0), (uint32_t)(c & 1));
        }
        __syncwarp();
    } else {
        // =========================================================== MMA issuers
        if (lane == 0) {
            FwdItem it = first;
            bool ok = true;
            int tt = 0;      // tiles over all blocks
            int nq = 0;      // blocks with K/V tiles so far
            for (int k = 0; ok; ++k) {
                if (it.n_kv > 0) {
                    if (warp == kMmaWarp) {
                        ok = wait_bounded(bar_q_full, (uint32_t)(nq & 1), abort_flag, p.wait_limit);
                        for (int i = 0; i < it.n_kv && ok; ++i, ++tt) {
                            const int t = tt - C::kSBufs;   // S(t) must have been read
                            if (t >= 0)
                                ok = wait_bounded(bar_s_free(t % C::kSBufs), (uint32_t)((t / C::kSBufs) & 1),
                                                  abort_flag, p.wait_limit);
                            const int sl = tt % C::kStagesK;
                            if (ok)
                                ok = wait_bounded(bar_full(0, sl), (uint32_t)((tt / C::kStagesK) & 1), abort_flag,
                                                  p.wait_limit);
                            if (!ok) break;
                            tc_fence_after();
                            const uint32_t slot = ring_slot(0, sl);
#pragma unroll
                            for (int kk = 0; kk < D * C::kElemBytes / 32; ++kk) {
                                const uint32_t koff =
                                    (uint32_t)((kk * 32 / C::kSwz) * C::kBoxBytes + (kk * 32) % C::kSwz);
                                const uint64_t a = smem_desc(q_tile + koff, 16, 8 * C::kSwz, C::kSwzMode);
                                const uint64_t bb = smem_desc(slot + koff, 16, 8 * C::kSwz, C::kSwzMode);
                                if constexpr (kF8)
                                    umma_ss_f8(tmem + C::col_s(tt % C::kSBufs), a, bb, C::kIdescQK, kk > 0 ? 1u : 0u);
                                else
                                    umma_ss(tmem + C::col_s(tt % C::kSBufs), a, bb, C::kIdescQK, kk > 0 ? 1u : 0u);
                            }
                            umma_commit(bar_s_full(i & 1));   // the softmax parity of tile i of this block
                            umma_commit(bar_empty(0, sl));
                        }
                        if (!ok) break;
                        umma_commit(bar_q_free);   // this block's products are done with Q once they land
                    } else {
                        // the block's first product starts O afresh: the previous
                        // block's O must have been read out of TMEM
                        if (nq > 0) ok = wait_bounded(bar_o_free, (uint32_t)((nq - 1) & 1), abort_flag, p.wait_limit);
                        for (int j = 0; j < it.n_kv && ok; ++j, ++tt) {
                            const int pb = tt % C::kPBufs;
                            ok = wait_bounded(bar_p_full(pb), (uint32_t)((tt / C::kPBufs) & 1), abort_flag,
                                              p.wait_limit);
                            const int sl = tt % C::kStagesV;
                            if (ok)
                                ok = wait_bounded(bar_full(1, sl), (uint32_t)((tt / C::kStagesV) & 1), abort_flag,
                                                  p.wait_limit);
                            if (!ok) break;
                            tc_fence_after();
                            const uint32_t slot = ring_slot(1, sl);
#pragma unroll
                            for (int kk = 0; kk < kBlockN / C::kKPerMma; ++kk) {
                                const uint32_t a_col = C::col_p(pb) + (uint32_t)(kk * 8);
                                const uint64_t bb = smem_desc(slot + (uint32_t)(kk * C::kKPerMma * C::kSwz),
                                                              C::kBoxBytes, 8 * C::kSwz, C::kSwzMode);
                                if constexpr (kF8)
                                    umma_ts_f8(tmem + C::kColO, tmem + a_col, bb, C::kIdescPV,
                                               (j > 0 || kk > 0) ? 1u : 0u);
                                else
                                    umma_ts(tmem + C::kColO, tmem + a_col, bb, C::kIdescPV, (j > 0 || kk > 0) ? 1u : 0u);
                            }
                            umma_commit(bar_pv_done(pb));
                            umma_commit(bar_empty(1, sl));
                        }
                        if (!ok) break;
                        umma_commit(bar_drain);   // the block's last product, and with it all of them
                    }
                    ++nq;
                }
                if (next_item(k, it, false) <= 0) break;
            }
            // both issuers: every product issued has landed before TMEM is freed
            umma_commit(bar_fin);
            (void)wait_own_work(bar_fin, 0);
        }
        __syncwarp();
      }
    } else {
        setmaxnreg_inc<kRegsSoftmax>();
        // =========================================================== softmax: one thread per row, tiles in turn
        const int qd = warp & 3;
        const int g = warp >> 2;
        const int r = qd * 32 + lane;
        const uint32_t lane_off = (uint32_t)(qd * 32) << 16;
        const float c = p.scale_log2;
        constexpr bool has_bias = kBias != kBiasNone;
        FwdItem it = first;
        int tt0 = 0;                 // tiles of the blocks before this one
        int nq = 0;                  // blocks with K/V tiles so far
        int sf_own = 0;              // completions of s_full(g) before this block
        for (int k = 0;; ++k) {
            const int n_kv = it.n_kv;
            const int h = it.h, b = it.b, m0 = it.m0, off = it.off, t0 = it.t0;
            const int row = m0 + r;
            const int lim = row_key_limit(row, it.kl, off, p.causal);
            const int lo = row_key_start(row, off, p.window_left);
            const float alpha = (kBias == kBiasSlopes) ? p.slopes[h] * 1.4426950408889634f : 0.f;
            const float* const trow = (kBias == kBiasTable)
                                          ? p.bias_table + (size_t)h * (2 * (size_t)p.bias_radius + 1) + p.bias_radius
                                          : nullptr;
            float m_seen = -INFINITY;
            float lu = 0.f;
            bool ok = true;

            for (int j = g; j < n_kv; j += 2) {
                const int tt = tt0 + j;                                       // tile over all blocks
                const uint32_t use = (uint32_t)((sf_own + (j >> 1)) & 1);     // phase of s_full(g)
                bool good = wait_bounded(bar_s_full(g), use, abort_flag, p.wait_limit);
                if (!__all_sync(0xffffffffu, good)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                float s[kBlockN];
                {
                    uint32_t u[kBlockN];
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4)
                        tmem_ld32(tmem + lane_off + C::col_s(tt % C::kSBufs) + 32u * q4,
                                  *reinterpret_cast<uint32_t(*)[32]>(&u[32 * q4]));
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < kBlockN; ++i) {
                        reg_after_wait(u[i]);
                        s[i] = __uint_as_float(u[i]);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_s_free(tt % C::kSBufs));
                const int kbase = (t0 + j) * kBlockN;
                const bool masked = __any_sync(0xffffffffu, kbase + kBlockN > lim || kbase < lo);
                if constexpr (kBias == kBiasSlopes) {
                    const float d0 = (float)(row + off - kbase);
#pragma unroll
                    for (int i = 0; i < kBlockN; ++i) s[i] = fmaf(s[i], c, -alpha * fabsf(d0 - (float)i));
                } else if constexpr (kBias == kBiasTable) {
                    const int R = p.bias_radius;
                    const int r0 = kbase - (row + off);
                    if (__all_sync(0xffffffffu, r0 >= -R && r0 + kBlockN - 1 <= R)) {
#pragma unroll
                        for (int i = 0; i < kBlockN; ++i)
                            s[i] = fmaf(__ldg(trow + r0 + i), 1.4426950408889634f, s[i] * c);
                    } else {
#pragma unroll
                        for (int i = 0; i < kBlockN; ++i)
                            s[i] = fmaf(__ldg(trow + min(max(r0 + i, -R), R)), 1.4426950408889634f, s[i] * c);
                    }
                }
                const float cs = has_bias ? 1.f : c;
                if (masked) {
#pragma unroll
                    for (int i = 0; i < kBlockN; ++i)
                        if (kbase + i >= lim || kbase + i < lo) s[i] = -INFINITY;
                }
                const float mx = fmaxf(fmaxf(chunk_max32(s, 0), chunk_max32(s, 32)),
                                       fmaxf(chunk_max32(s, 64), chunk_max32(s, 96)));
                // the other warp's reference max after tile tt - 1 (same block)
                float m_prev = -INFINITY;
                if (j > 0) {
                    good = wait_tagged_max(mref_w + 8u * (uint32_t)((g ^ 1) * kBlockM + r), (uint32_t)(tt - 1),
                                           m_prev, abort_flag, p.wait_limit);
                    if (!__all_sync(0xffffffffu, good)) {
                        ok = false;
                        break;
                    }
                }
                const float t_max = mx * cs;
                const float m_cur = (t_max > m_prev + kRescaleThreshold) ? t_max : m_prev;
                if (j + 1 < n_kv)
                    st_relaxed_shared_u64(mref_w + 8u * (uint32_t)(g * kBlockM + r),
                                          ((unsigned long long)(uint32_t)tt << 32) | __float_as_uint(m_cur));
                if (m_cur != m_seen) {
                    const float f = ex2_approx(m_seen - m_cur);
                    lu *= f;
                    m_seen = m_cur;
                }
                const float mu = (m_cur == -INFINITY) ? 0.f : m_cur;
                const int pb = tt % C::kPBufs;
                if (tt >= C::kPBufs) {
                    good = wait_bounded(bar_pv_done(pb), (uint32_t)(((tt - C::kPBufs) / C::kPBufs) & 1), abort_flag,
                                        p.wait_limit);
                    if (!__all_sync(0xffffffffu, good)) {
                        ok = false;
                        break;
                    }
                }
                float2 lu2 = make_float2(0.f, 0.f);
                const uint32_t taddr_p = tmem + lane_off + C::col_p(pb);
                if (masked) {
                    exp_store_half<0, 0, kF8>(s, cs, mu, taddr_p, lu2);
                    exp_store_half<0, 1, kF8>(s, cs, mu, taddr_p, lu2);
                } else {
                    exp_store_half<C::kEmuPairs, 0, kF8>(s, cs, mu, taddr_p, lu2);
                    exp_store_half<C::kEmuPairs, 1, kF8>(s, cs, mu, taddr_p, lu2);
                }
                lu += lu2.x + lu2.y;
                const float alpha_o = (m_cur != m_prev) ? ex2_approx(m_prev - m_cur) : 1.f;
                if (j > 0 && __any_sync(0xffffffffu, alpha_o != 1.f)) {
                    good = wait_bounded(bar_pv_done((tt - 1) % C::kPBufs), (uint32_t)(((tt - 1) / C::kPBufs) & 1),
                                        abort_flag, p.wait_limit);
                    if (!__all_sync(0xffffffffu, good)) {
                        tmem_wait_st();
                        ok = false;
                        break;
                    }
                    tc_fence_after();
#pragma unroll
                    for (int q4 = 0; q4 < D / 32 + 1; ++q4) {
                        const uint32_t ocol = tmem + lane_off + C::kColO + 32u * q4;
                        uint32_t u[32];
                        tmem_ld32(ocol, u);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; i += 2) {
                            reg_after_wait(u[i]);
                            reg_after_wait(u[i + 1]);
                            const float2 v = __fmul2_rn(make_float2(__uint_as_float(u[i]), __uint_as_float(u[i + 1])),
                                                        make_float2(alpha_o, alpha_o));
                            u[i] = __float_as_uint(v.x);
                            u[i + 1] = __float_as_uint(v.y);
                        }
                        tmem_st32(ocol, u);
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_p_full(pb));
            }

            // ---------------------------------------------------------- epilogue of this block
            float* const epi = epi2 + (k & 1) * PC::kEpiFloats;
            const bool have_o = n_kv > 0;
            bool good = ok;
            if (good && have_o) {
                good = wait_bounded(bar_drain, (uint32_t)(nq & 1), abort_flag, p.wait_limit);
                good = __all_sync(0xffffffffu, good);
                if (good) tc_fence_after();
            }
            epi[g * kBlockM + r] = m_seen;
            epi[(2 + g) * kBlockM + r] = lu;
            // The next block's item, read before the quadrant's barrier: both warps
            // read the same mailbox slot, and a read whose wait ran out counts as a
            // failure of this block, so the two warps leave together here (a warp
            // left alone at the next block's barrier would wait without a limit).
            const int nxt = next_item(k, it, true);
            good = !named_bar_or(kBarQuadBase + qd, 64, !(good && nxt >= 0));
            const float m0w = epi[r], m1w = epi[kBlockM + r];
            const float m_fin = fmaxf(m0w, m1w);
            const float f0 = (m0w == m_fin) ? 1.f : ex2_approx(m0w - m_fin);
            const float f1 = (m1w == m_fin) ? 1.f : ex2_approx(m1w - m_fin);
            const float lu_row = epi[2 * kBlockM + r] * f0 + epi[3 * kBlockM + r] * f1;
            if (!good) break;   // both warps of the quadrant leave together
            float l_row = 0.f;
            uint32_t u[D / 2];
            if (have_o) {
                uint32_t ul[32];
                tmem_ld32(tmem + lane_off + C::kColL, ul);
#pragma unroll
                for (int q4 = 0; q4 < D / 64; ++q4)
                    tmem_ld32(tmem + lane_off + C::kColO + (uint32_t)(g * (D / 2) + 32 * q4),
                              *reinterpret_cast<uint32_t(*)[32]>(&u[32 * q4]));
                tmem_wait_ld();
                reg_after_wait(ul[0]);
                l_row = __uint_as_float(ul[0]);
#pragma unroll
                for (int i = 0; i < D / 2; ++i) reg_after_wait(u[i]);
                // O and its row sums are out of TMEM: the next block may start O afresh
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_o_free);
            } else {
#pragma unroll
                for (int i = 0; i < D / 2; ++i) u[i] = 0u;
            }
            float inv_l = (l_row > 0.f) ? 1.f / l_row : 0.f;
            if constexpr (kF8) inv_l *= p.o_scale;
            if (row < p.Nq) {
                uint4* dst = reinterpret_cast<uint4*>(p.o_out + (((size_t)b * p.H + h) * (size_t)p.Nq + row) * D +
                                                      g * (D / 2));
#pragma unroll
                for (int v4 = 0; v4 < D / 16; ++v4) {
                    uint4 w4;
                    w4.x = pack_bf16x2(__uint_as_float(u[8 * v4]) * inv_l, __uint_as_float(u[8 * v4 + 1]) * inv_l);
                    w4.y = pack_bf16x2(__uint_as_float(u[8 * v4 + 2]) * inv_l, __uint_as_float(u[8 * v4 + 3]) * inv_l);
                    w4.z = pack_bf16x2(__uint_as_float(u[8 * v4 + 4]) * inv_l, __uint_as_float(u[8 * v4 + 5]) * inv_l);
                    w4.w = pack_bf16x2(__uint_as_float(u[8 * v4 + 6]) * inv_l, __uint_as_float(u[8 * v4 + 7]) * inv_l);
                    dst[v4] = w4;
                }
                if (g == 0) {
                    const float lse =
                        (lu_row > 0.f) ? (m_fin + lg2_approx(lu_row)) * 0.69314718055994531f : -INFINITY;
                    p.lse[((size_t)b * p.H + h) * (size_t)p.Nq + row] = lse;
                }
            }
            // the counters of the blocks taken so far
            if (n_kv > 0) {
                tt0 += n_kv;
                // group 0 takes the even tiles, group 1 the odd ones
                sf_own += (g == 0) ? (n_kv + 1) / 2 : n_kv / 2;
                ++nq;
            }
            if (nxt <= 0) break;   // the same answer in both warps (same mailbox slot)
        }
        tc_fence_before();
    }

    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace fa
