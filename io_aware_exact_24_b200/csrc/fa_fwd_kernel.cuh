// fa_fwd_kernel.cuh -- exact attention forward for sm_100a (B200).
//
// What it computes: O = softmax(scale * Q K^T + mask) V and the per-row
// log-sum-exp, the tiled way described in "FlashAttention 与边缘设备上的注意力
// 内存瓶颈" (section 3.1 tiling, 3.2 online softmax) and "FlashAttention：把
// 注意力从公式写成数据流" (section "分块与在线 softmax": for each Q tile walk the
// K/V tiles, update running max, exp-sum and output accumulator; the score
// matrix is never stored).  The pages' kernels target A100/RTX 3090/T4 and
// Hopper; this one is laid out for Blackwell:
//
//  * one CTA = one (b, h) and two 128-row Q tiles (256 query rows) that share
//    every K/V tile loaded into shared memory;
//  * warp 8 (one elected lane) streams Q once and then K_j, V_j through a ring
//    of shared-memory slots with TMA (128B-swizzled boxes of 64 columns x 128
//    rows), one mbarrier pair (full/empty) per slot -- the double buffering
//    that "FlashAttention：把注意力从公式写成数据流" (section "端侧与专用加速器")
//    names for hiding loads;
//  * warp 9 (one elected lane) issues tcgen05 MMAs: S_t = Q_t K_j^T into TMEM
//    (fp32, 128 lanes x 128 columns) and O_t += P_t V_j with P_t read from
//    TMEM and V_j from shared memory; completions are signalled with
//    tcgen05.commit onto mbarriers;
//  * warps 0-3 own Q tile 0 and warps 4-7 own Q tile 1 (one thread per query
//    row, because TMEM lane i is row i): load the S row from TMEM, mask it on
//    boundary tiles only, update the running max m and sum l in the exp2
//    domain, write P back to TMEM as bf16, and rescale their O row in TMEM
//    when the max moved by more than 2^8 (exact: m, l and O always share one
//    reference max);
//  * while one tile's rows are in softmax the tensor core works on the other
//    tile, so the MMAs of tile 1 overlap the exponentials of tile 0 and back;
//  * epilogue: O / l -> bf16 into the (now idle) Q buffer, TMA store clipped at
//    N_q; LSE = ln2 * (m + log2 l); rows without a visible key give O = 0 and
//    LSE = -inf ("FlashAttention：把注意力从公式写成数据流", section "精度、掩码和
//    边界情况": masked positions never enter the normaliser).
//
// Every mbarrier wait is bounded; a wait that runs out records
// FA_ERR_DEVICE_TIMEOUT in g_fa_status and the CTA winds down instead of
// hanging.
#pragma once

#include <cmath>
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "sm100_ptx.cuh"

namespace fa {

constexpr int kBlockM = 128;        // query rows per Q tile (= TMEM lanes)
constexpr int kBlockN = 128;        // keys per K/V tile
constexpr int kTilesPerCta = 2;     // Q tiles sharing one K/V stream
constexpr int kNumThreads = 320;    // 8 softmax warps + producer warp + MMA warp
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kTmemCols = 512;
constexpr int kSwizzleBoxBytes = 128 * 128;  // one 64-column x 128-row bf16 box
constexpr float kRescaleThreshold = 8.0f;    // log2 units: rescale only if max grows > 2^8
constexpr int kStatusTimeout = -6;           // FA_ERR_DEVICE_TIMEOUT

struct FwdParams {
    float* lse;                 // [B,H,Nq]
    const int32_t* key_lens;    // [B] or nullptr
    int B, H, Nq, Nk;
    float scale_log2;           // scale * log2(e), > 0
    int causal;
    unsigned long long wait_limit;  // clock64 cycles per wait before giving up
};

template <int D>
struct Cfg {
    static_assert(D == 64 || D == 128, "head dim");
    static constexpr int kBoxes = D / 64;                        // 64-column boxes per row
    static constexpr int kTileBytes = kBlockM * D * 2;           // one Q / K / V tile
    static constexpr int kStages = (D == 64) ? 8 : 4;            // K/V ring slots
    static constexpr int kQOff = 0;
    static constexpr int kKvOff = kTilesPerCta * kTileBytes;
    static constexpr int kBarOff = kKvOff + kStages * kTileBytes;
    // barriers: q_full, kv_full[S], kv_empty[S], s_full[2], p_full[2], o_full[2], drain
    static constexpr int kNumBars = 8 + 2 * kStages;
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;
    static constexpr int kSmemBytes = kMiscOff + 16 + 1024;      // + alignment slack
    // TMEM columns
    static constexpr uint32_t kColS0 = 0;
    static constexpr uint32_t kColO0 = 256;
    __host__ __device__ static constexpr uint32_t col_s(int t) { return kColS0 + 128u * t; }
    __host__ __device__ static constexpr uint32_t col_o(int t) { return kColO0 + (uint32_t)D * t; }
    // P (bf16, 64 columns): separate columns when they fit, else over the first
    // half of the tile's own S columns (S is fully read before P is written).
    __host__ __device__ static constexpr uint32_t col_p(int t) { return D == 64 ? 384u + 64u * t : col_s(t); }
    // Instruction descriptors (kind::f16): D=f32, A=B=bf16, M=128.
    //   QK^T: A=Q K-major, B=K K-major, N=128.  PV: A=P (TMEM, K-major), B=V MN-major, N=D.
    static constexpr uint32_t kIdescQK = (1u << 4) | (1u << 7) | (1u << 10) | (0u << 15) |
                                         (0u << 16) | ((uint32_t)(kBlockN >> 3) << 17) |
                                         ((uint32_t)(kBlockM >> 4) << 24);
    static constexpr uint32_t kIdescPV = (1u << 4) | (1u << 7) | (1u << 10) | (0u << 15) |
                                         (1u << 16) | ((uint32_t)(D >> 3) << 17) |
                                         ((uint32_t)(kBlockM >> 4) << 24);
};

// Shared-memory matrix descriptor, 128-byte swizzle, sm_100 version bits.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((addr & 0x3FFFFu) >> 4);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;   // descriptor version for tcgen05
    d |= (uint64_t)2 << 61;   // SWIZZLE_128B
    return d;
}

__device__ int g_fa_status;

// Bounded mbarrier wait.  Returns false (and raises the CTA's abort flag and
// the device status word) if the phase did not complete within the limit, or
// if another role of this CTA already gave up.
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                             unsigned long long limit) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if ((unsigned long long)(clock64() - t0) > limit) {
            *abort_flag = 1;
            atomicExch(&g_fa_status, kStatusTimeout);
            return false;
        }
    }
}

// Number of keys (prefix length) a query row may see.
__device__ __forceinline__ int row_key_limit(int row, int kl, int off, int causal) {
    if (!causal) return kl;
    long long c = (long long)row + off + 1;
    c = c < 0 ? 0 : c;
    return c < kl ? (int)c : kl;
}

template <int D>
__global__ void __launch_bounds__(kNumThreads, 1)
    fa_fwd_sm100_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                        const FwdParams p) {
    using C = Cfg<D>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw_base = smem_addr(smem_raw);
    const uint32_t base = (raw_base + 1023u) & ~1023u;
    uint8_t* const base_ptr = smem_raw + (base - raw_base);

    const uint32_t bar_q_full = base + C::kBarOff;
    auto bar_kv_full = [&](int s) { return base + C::kBarOff + 8u * (1 + s); };
    auto bar_kv_empty = [&](int s) { return base + C::kBarOff + 8u * (1 + C::kStages + s); };
    auto bar_s_full = [&](int t) { return base + C::kBarOff + 8u * (1 + 2 * C::kStages + t); };
    auto bar_p_full = [&](int t) { return base + C::kBarOff + 8u * (3 + 2 * C::kStages + t); };
    auto bar_o_full = [&](int t) { return base + C::kBarOff + 8u * (5 + 2 * C::kStages + t); };
    const uint32_t bar_drain = base + C::kBarOff + 8u * (7 + 2 * C::kStages);
    uint32_t* const tmem_holder = reinterpret_cast<uint32_t*>(base_ptr + C::kMiscOff);
    volatile int* const abort_flag = reinterpret_cast<volatile int*>(base_ptr + C::kMiscOff + 4);
    auto q_tile = [&](int t) { return base + C::kQOff + (uint32_t)(t * C::kTileBytes); };
    auto kv_slot = [&](int s) { return base + C::kKvOff + (uint32_t)(s * C::kTileBytes); };

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // ---- work item: (b, h, 256-row block); heavy causal blocks launch first
    const int num_m = (int)gridDim.x;
    const int m_blk = p.causal ? (num_m - 1 - (int)blockIdx.x) : (int)blockIdx.x;
    const int h = blockIdx.y;
    const int b = blockIdx.z;
    const int m0 = m_blk * (kTilesPerCta * kBlockM);
    int kl = p.Nk;
    if (p.key_lens != nullptr) {
        kl = p.key_lens[b];
        kl = kl < 0 ? 0 : (kl > p.Nk ? p.Nk : kl);
    }
    const int off = p.Nk - p.Nq;  // causal diagonal offset (bottom-right aligned)
    // K/V tiles each Q tile must visit (0 for a tile with no query row).
    int n_tiles[kTilesPerCta];
#pragma unroll
    for (int t = 0; t < kTilesPerCta; ++t) {
        const int first = m0 + t * kBlockM;
        if (first >= p.Nq) {
            n_tiles[t] = 0;
            continue;
        }
        const int last = min(first + kBlockM - 1, p.Nq - 1);
        const int n_end = row_key_limit(last, kl, off, p.causal);
        n_tiles[t] = (n_end + kBlockN - 1) / kBlockN;
    }
    const int n_kv = max(n_tiles[0], n_tiles[1]);

    // ---- setup: barriers (producer lane 0), TMEM (MMA warp)
    if (warp == kProducerWarp && lane == 0) {
        mbar_init(bar_q_full, 1);
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(bar_kv_full(s), 1);
            mbar_init(bar_kv_empty(s), 1);
        }
        for (int t = 0; t < kTilesPerCta; ++t) {
            mbar_init(bar_s_full(t), 1);
            mbar_init(bar_p_full(t), kBlockM);
            mbar_init(bar_o_full(t), 1);
        }
        mbar_init(bar_drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
        prefetch_tensormap(&tm_o);
    }
    if (warp == kMmaWarp) {
        tmem_alloc(smem_addr(tmem_holder), kTmemCols);
        tmem_relinquish();
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    if (warp == kProducerWarp) {
        // =========================================================== TMA producer
        if (lane == 0 && n_kv > 0) {
            const uint64_t pol_kv = policy_evict_last();
            const uint64_t pol_q = policy_evict_first();
            // only tiles with work are loaded: a tile that sees no key writes its
            // zeros through the same buffer, which must not have a copy in flight
            int q_tiles = 0;
            for (int t = 0; t < kTilesPerCta; ++t) q_tiles += (n_tiles[t] > 0) ? 1 : 0;
            mbar_arrive_expect_tx(bar_q_full, (uint32_t)(q_tiles * C::kTileBytes));
            for (int t = 0; t < kTilesPerCta; ++t) {
                if (n_tiles[t] == 0) continue;
                for (int bx = 0; bx < C::kBoxes; ++bx)
                    tma_load_4d(q_tile(t) + bx * kSwizzleBoxBytes, &tm_q, bar_q_full, bx * 64,
                                m0 + t * kBlockM, h, b, pol_q);
            }
            int issued[C::kStages];
            for (int s = 0; s < C::kStages; ++s) issued[s] = -1;
            bool ok = true;
            for (int j = 0; j < n_kv && ok; ++j) {
                for (int which = 0; which < 2 && ok; ++which) {
                    const int n = 2 * j + which;
                    const int s = n % C::kStages;
                    const uint32_t round = (uint32_t)(n / C::kStages);
                    if (!wait_bounded(bar_kv_empty(s), (round & 1u) ^ 1u, abort_flag, p.wait_limit)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(bar_kv_full(s), (uint32_t)C::kTileBytes);
                    const CUtensorMap* m = which == 0 ? &tm_k : &tm_v;
                    for (int bx = 0; bx < C::kBoxes; ++bx)
                        tma_load_4d(kv_slot(s) + bx * kSwizzleBoxBytes, m, bar_kv_full(s), bx * 64,
                                    j * kBlockN, h, b, pol_kv);
                    issued[s] = n;
                }
            }
            if (!ok) {
                // wind down: let every copy already issued land before the CTA exits
                for (int s = 0; s < C::kStages; ++s)
                    if (issued[s] >= 0)
                        (void)wait_bounded(bar_kv_full(s), (uint32_t)((issued[s] / C::kStages) & 1), abort_flag,
                                           p.wait_limit);
            }
        }
        __syncwarp();
    } else if (warp == kMmaWarp) {
        // =========================================================== MMA issuer
        if (lane == 0 && n_kv > 0) {
            bool ok = wait_bounded(bar_q_full, 0, abort_flag, p.wait_limit);
            auto mma_qk = [&](int t, int slot) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t koff = (uint32_t)((kk / 4) * kSwizzleBoxBytes + (kk % 4) * 32);
                    const uint64_t a = smem_desc_sw128(q_tile(t) + koff, 16, 1024);
                    const uint64_t bb = smem_desc_sw128(kv_slot(slot) + koff, 16, 1024);
                    umma_ss(tmem + C::col_s(t), a, bb, C::kIdescQK, kk > 0 ? 1u : 0u);
                }
            };
            auto mma_pv = [&](int t, int slot, bool accumulate) {
#pragma unroll
                for (int kk = 0; kk < kBlockN / 16; ++kk) {
                    const uint64_t bb =
                        smem_desc_sw128(kv_slot(slot) + (uint32_t)(kk * 16 * 128), kSwizzleBoxBytes, 1024);
                    umma_ts(tmem + C::col_o(t), tmem + C::col_p(t) + (uint32_t)(kk * 8), bb, C::kIdescPV,
                            (accumulate || kk > 0) ? 1u : 0u);
                }
            };
            auto kv_wait = [&](int n) {
                const int s = n % C::kStages;
                return wait_bounded(bar_kv_full(s), (uint32_t)((n / C::kStages) & 1), abort_flag, p.wait_limit);
            };
            for (int j = 0; j < n_kv && ok; ++j) {
                const int sK = (2 * j) % C::kStages;
                const int sV = (2 * j - 1 + 2 * C::kStages) % C::kStages;  // slot of V_{j-1}
                ok = kv_wait(2 * j);
                if (ok && j > 0) ok = kv_wait(2 * j - 1);
                if (!ok) break;
                tc_fence_after();
                for (int t = 0; t < kTilesPerCta && ok; ++t) {
                    if (j < n_tiles[t]) {
                        if (j > 0) {
                            ok = wait_bounded(bar_p_full(t), (uint32_t)((j - 1) & 1), abort_flag, p.wait_limit);
                            if (!ok) break;
                            tc_fence_after();
                            mma_pv(t, sV, j - 1 > 0);
                        }
                        mma_qk(t, sK);
                        umma_commit(bar_s_full(t));
                    } else if (j == n_tiles[t] && j > 0) {
                        ok = wait_bounded(bar_p_full(t), (uint32_t)((j - 1) & 1), abort_flag, p.wait_limit);
                        if (!ok) break;
                        tc_fence_after();
                        mma_pv(t, sV, j - 1 > 0);
                        umma_commit(bar_o_full(t));
                    }
                }
                if (!ok) break;
                umma_commit(bar_kv_empty(sK));
                if (j > 0) umma_commit(bar_kv_empty(sV));
            }
            if (ok) {
                const int j = n_kv;
                const int sV = (2 * j - 1) % C::kStages;
                ok = kv_wait(2 * j - 1);
                if (ok) tc_fence_after();
                for (int t = 0; t < kTilesPerCta && ok; ++t) {
                    if (n_tiles[t] != n_kv) continue;
                    ok = wait_bounded(bar_p_full(t), (uint32_t)((j - 1) & 1), abort_flag, p.wait_limit);
                    if (!ok) break;
                    tc_fence_after();
                    mma_pv(t, sV, j - 1 > 0);
                    umma_commit(bar_o_full(t));
                }
                if (ok) umma_commit(bar_kv_empty(sV));
            }
            // drain: every MMA and commit of this CTA has landed before TMEM is freed
            umma_commit(bar_drain);
            (void)wait_bounded(bar_drain, 0, abort_flag, p.wait_limit);
        }
        __syncwarp();
    } else {
        // =========================================================== softmax, one row per thread
        const int t = warp >> 2;                       // Q tile of this warpgroup
        const int r = threadIdx.x & (kBlockM - 1);     // row inside the tile == TMEM lane
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const int row = m0 + t * kBlockM + r;
        const int nt = n_tiles[t];
        const bool tile_has_rows = (m0 + t * kBlockM) < p.Nq;
        const int lim = row_key_limit(row, kl, off, p.causal);
        const float c = p.scale_log2;
        float m_ref = -INFINITY;   // reference max (log2 units) shared by l and O
        float l = 0.f;
        bool ok = true;

        for (int j = 0; j < nt; ++j) {
            if (!wait_bounded(bar_s_full(t), (uint32_t)(j & 1), abort_flag, p.wait_limit)) {
                ok = false;
                break;
            }
            tc_fence_after();
            float s[kBlockN];
            {
                uint32_t u[kBlockN];
#pragma unroll
                for (int q4 = 0; q4 < kBlockN / 32; ++q4)
                    tmem_ld32(tmem + lane_off + C::col_s(t) + 32u * q4,
                              *reinterpret_cast<uint32_t(*)[32]>(&u[32 * q4]));
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < kBlockN; ++i) {
                    reg_after_wait(u[i]);
                    s[i] = __uint_as_float(u[i]);
                }
            }
            const int kbase = j * kBlockN;
            if (kbase + kBlockN > lim) {
#pragma unroll
                for (int i = 0; i < kBlockN; ++i)
                    if (kbase + i >= lim) s[i] = -INFINITY;
            }
            float mx0 = s[0], mx1 = s[1], mx2 = s[2], mx3 = s[3];
#pragma unroll
            for (int i = 4; i < kBlockN; i += 4) {
                mx0 = fmaxf(mx0, s[i]);
                mx1 = fmaxf(mx1, s[i + 1]);
                mx2 = fmaxf(mx2, s[i + 2]);
                mx3 = fmaxf(mx3, s[i + 3]);
            }
            const float mx = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3));
            const float t_max = mx * c;   // c > 0, so -inf stays -inf
            const float m_new = fmaxf(m_ref, t_max);
            float alpha = 1.f;
            if (m_new > m_ref + kRescaleThreshold) {
                alpha = ex2_approx(m_ref - m_new);  // 0 when m_ref is -inf
                l *= alpha;
                m_ref = m_new;
            }
            const float mu = (m_ref == -INFINITY) ? 0.f : m_ref;
            float l0 = 0.f, l1 = 0.f;
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
                // 64 probabilities -> 32 packed bf16 pairs -> TMEM columns of P
                uint32_t w[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const float e0 = ex2_approx(fmaf(s[64 * h2 + 2 * i], c, -mu));
                    const float e1 = ex2_approx(fmaf(s[64 * h2 + 2 * i + 1], c, -mu));
                    l0 += e0;
                    l1 += e1;
                    w[i] = pack_bf16x2(e0, e1);
                }
                tmem_st32(tmem + lane_off + C::col_p(t) + 32u * h2, w);
            }
            l += l0 + l1;
            // O still holds the sum over tiles < j, relative to the old max.
            if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
                for (int q4 = 0; q4 < D / 32; ++q4) {
                    uint32_t u[32];
                    tmem_ld32(tmem + lane_off + C::col_o(t) + 32u * q4, u);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        reg_after_wait(u[i]);
                        u[i] = __float_as_uint(__uint_as_float(u[i]) * alpha);
                    }
                    tmem_st32(tmem + lane_off + C::col_o(t) + 32u * q4, u);
                }
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar_p_full(t));
        }

        // ---------------------------------------------------------- epilogue
        if (ok && tile_has_rows) {
            bool have_o = nt > 0;
            if (have_o) {
                if (!wait_bounded(bar_o_full(t), 0, abort_flag, p.wait_limit)) {
                    ok = false;
                    have_o = false;
                }
                tc_fence_after();
            }
            if (ok) {
                const float inv_l = (l > 0.f) ? 1.f / l : 0.f;
                const uint32_t stage = q_tile(t);
#pragma unroll
                for (int q4 = 0; q4 < D / 32; ++q4) {
                    uint32_t u[32];
                    if (have_o) {
                        tmem_ld32(tmem + lane_off + C::col_o(t) + 32u * q4, u);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i) reg_after_wait(u[i]);
                    } else {
#pragma unroll
                        for (int i = 0; i < 32; ++i) u[i] = 0u;
                    }
                    uint32_t pkd[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        pkd[i] = pack_bf16x2(__uint_as_float(u[2 * i]) * inv_l,
                                             __uint_as_float(u[2 * i + 1]) * inv_l);
                    // 4 x 16-byte chunks of row r; chunk cc of the row lives in box cc/8,
                    // swizzled position (cc%8) ^ (r%8) inside the row's 128 bytes.
#pragma unroll
                    for (int v4 = 0; v4 < 4; ++v4) {
                        const int cc = q4 * 4 + v4;
                        const uint32_t addr = stage + (uint32_t)((cc >> 3) * kSwizzleBoxBytes + r * 128 +
                                                                 (((cc & 7) ^ (r & 7)) << 4));
                        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr),
                                     "r"(pkd[4 * v4]), "r"(pkd[4 * v4 + 1]), "r"(pkd[4 * v4 + 2]),
                                     "r"(pkd[4 * v4 + 3])
                                     : "memory");
                    }
                }
                if (row < p.Nq) {
                    const float lse = (l > 0.f) ? (m_ref + lg2_approx(l)) * 0.69314718055994531f : -INFINITY;
                    p.lse[((size_t)b * p.H + h) * (size_t)p.Nq + row] = lse;
                }
                fence_proxy_async_smem();
                named_bar_sync(1 + t, kBlockM);
                if (r == 0) {
                    for (int bx = 0; bx < C::kBoxes; ++bx)
                        tma_store_4d(&tm_o, stage + bx * kSwizzleBoxBytes, bx * 64, m0 + t * kBlockM, h, b);
                    bulk_commit_group();
                    bulk_wait_group_read0();
                }
            }
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
