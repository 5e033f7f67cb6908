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
//  * one CTA = one (b, h) and one 128-row Q tile (TMEM lane i = query row i);
//  * warp 8 (one elected lane) loads Q once and then streams K and V tiles
//    (128 keys) through a ring of shared-memory slots with TMA (128B-swizzled
//    boxes of 64 columns x 128 rows), one full/empty mbarrier pair per slot --
//    the double buffering "FlashAttention：把注意力从公式写成数据流" (section
//    "端侧与专用加速器") names for hiding loads;
//  * warp 9 (one elected lane) issues the tcgen05 MMAs.  S is double-buffered
//    in TMEM: S(j+2) = Q K_{j+2}^T is issued right after O += P(j) V_j, so the
//    score tile the softmax needs next is computed while it works on the
//    current one and the softmax never waits on the tensor core;
//  * warps 0-7 do the online softmax, one thread per query row and tile:
//    warps q and q+4 both own TMEM lanes 32q..32q+31 and take the K/V tiles
//    in turn (even / odd), so one warp's exponentials overlap the other's
//    loads and maxima.  Only the running reference max passes between them
//    (shared memory + an mbarrier); each keeps its own partial row sum.
//    Exponentials are taken in the exp2 domain, some on MUFU and some with a
//    polynomial on the FMA pipe; P goes back to TMEM as bf16 over the first
//    half of the tile's S buffer and feeds the PV MMA from there;
//  * the reference max moves only when the row max grows by more than 2^8;
//    O is then rescaled in TMEM (exact: m, l and O always share one max);
//  * epilogue: O / l -> bf16 -> shared memory (128B-swizzled) -> TMA store
//    clipped at N_q; LSE = ln2 * (m + log2 l); rows without a visible key give
//    O = 0 and LSE = -inf ("FlashAttention：把注意力从公式写成数据流", section
//    "精度、掩码和边界情况": masked positions never enter the normaliser).
//
// Every mbarrier wait is bounded; a wait that runs out records
// FA_ERR_DEVICE_TIMEOUT in g_fa_status and the CTA winds down instead of
// hanging.
#pragma once

#include <cmath>
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "exp2_poly.cuh"
#include "sm100_ptx.cuh"

namespace fa {

constexpr int kBlockM = 128;        // query rows per CTA (= TMEM lanes)
constexpr int kBlockN = 128;        // keys per K/V tile
constexpr int kNumThreads = 384;    // 8 softmax warps, producer, MMA, 2 spare
constexpr int kSoftmaxWarps = 8;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kTmemCols = 512;
// Registers are allocated per warpgroup: 384 threads x 168 at launch, then the
// softmax warpgroups take 216 and the producer/MMA warpgroup keeps 72
// (2*128*216 + 128*72 = 384*168).
constexpr uint32_t kRegsSoftmax = 216;
constexpr uint32_t kRegsControl = 72;
constexpr int kSwizzleBoxBytes = 128 * 128;  // one 64-column x 128-row bf16 box
constexpr float kRescaleThreshold = 8.0f;    // log2 units: rescale only if max grows > 2^8
constexpr int kStatusTimeout = -6;           // FA_ERR_DEVICE_TIMEOUT
// named barriers (epilogue only): 1..4 pair the two warps of a lane quadrant, 5 spans all softmax warps
constexpr uint32_t kBarQuadBase = 1;
constexpr uint32_t kBarSoftmaxAll = 5;

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
    static constexpr int kStages = (D == 64) ? 10 : 5;           // K/V ring slots
    // Of every 8 pairs of probabilities, this many are computed on the FMA pipe
    // (exp2_fma2) and the rest on MUFU, so neither unit is the lone bottleneck.
#ifdef FA_EMU_PAIRS_D64
    static constexpr int kEmuPairs = (D == 64) ? FA_EMU_PAIRS_D64 : FA_EMU_PAIRS_D128;
#else
    static constexpr int kEmuPairs = 2;
#endif
    static constexpr int kQOff = 0;
    static constexpr int kKvOff = kTileBytes;
    static constexpr int kBarOff = kKvOff + kStages * kTileBytes;
    // barriers: q_full, kv_full[S], kv_empty[S], s_full[2], p_full[2], o_done[2],
    // m_ready[4 quadrants][2 parities], drain
    static constexpr int kNumBars = 16 + 2 * kStages;
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;      // tmem base, abort flag
    static constexpr int kMrefOff = kMiscOff + 16;               // published reference max [parity][row]
    static constexpr int kEpiOff = kMrefOff + 2 * kBlockM * 4;   // epilogue exchange: m [2][row], l [2][row]
    static constexpr int kSmemBytes = kEpiOff + 4 * kBlockM * 4 + 1024;  // + alignment slack
    // TMEM columns: S buffers at 0 and 128 (P of a tile over the first 64
    // columns of its S buffer), O at 256.
    __host__ __device__ static constexpr uint32_t col_s(int b) { return 128u * b; }
    static constexpr uint32_t kColO = 256;
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
        // sleeps until the phase completes (or 0.1 ms passes): a waiting warp
        // leaves its issue slots to the warps that are computing
        if (mbar_try_wait_sleep(bar, parity, 100000u)) return true;
        if (*abort_flag) return false;
        if ((unsigned long long)(clock64() - t0) > limit) {
            *abort_flag = 1;
            atomicExch(&g_fa_status, kStatusTimeout);
            return false;
        }
    }
}

// 2^x for two finite x on the FMA pipe: x = n + r with n = rint(x) (added into the
// exponent field) and 2^r, r in [-1/2, 1/2], from the fitted cubic in exp2_poly.cuh.
// x is clamped at -125 so 2^n stays a normal number; callers never pass -inf.
__device__ __forceinline__ float2 exp2_fma2(float2 x) {
    x.x = fmaxf(x.x, -125.f);
    x.y = fmaxf(x.y, -125.f);
    const float2 t = __fadd2_rn(x, make_float2(12582912.f, 12582912.f));  // 1.5*2^23: rint in the low bits
    const float2 n = __fadd2_rn(t, make_float2(-12582912.f, -12582912.f));
    const float2 r = __ffma2_rn(n, make_float2(-1.f, -1.f), x);
    float2 q = __ffma2_rn(r, make_float2(kExp2C3, kExp2C3), make_float2(kExp2C2, kExp2C2));
    q = __ffma2_rn(q, r, make_float2(kExp2C1, kExp2C1));
    q = __ffma2_rn(q, r, make_float2(kExp2C0, kExp2C0));
    float2 e;
    e.x = __uint_as_float(__float_as_uint(q.x) + (__float_as_uint(t.x) << 23));
    e.y = __uint_as_float(__float_as_uint(q.y) + (__float_as_uint(t.y) << 23));
    return e;
}

// p = 2^(s*c - mu) for keys 64*h2 .. 64*h2+63 of the thread's row, packed to
// bf16 pairs and stored to its TMEM lane at taddr_p + 32*h2; the fp32 p are
// summed into (l0, l1).  kEmu of every 8 pairs go through exp2_fma2, the rest
// through MUFU ex2 (which maps -inf to 0, so masked tiles use kEmu = 0).
template <int kEmu, int h2>
__device__ __forceinline__ void exp_store_half(const float (&s)[kBlockN], float c, float mu, uint32_t taddr_p,
                                               float2& l0, float2& l1) {
    const float2 c2 = make_float2(c, c);
    const float2 nmu = make_float2(-mu, -mu);
    uint32_t w[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        const int pi = 32 * h2 + i;
        const float2 x = __ffma2_rn(make_float2(s[2 * pi], s[2 * pi + 1]), c2, nmu);
        float2 e;
        if ((i & 7) < kEmu) {
            e = exp2_fma2(x);
        } else {
            e.x = ex2_approx(x.x);
            e.y = ex2_approx(x.y);
        }
        if (i & 1)
            l1 = __fadd2_rn(l1, e);
        else
            l0 = __fadd2_rn(l0, e);
        w[i] = pack_bf16x2(e.x, e.y);
    }
    tmem_st32(taddr_p + 32u * h2, w);
}

// Maximum of s[o .. o+31] as a tree of three-input max (depth 4).
__device__ __forceinline__ float chunk_max32(const float (&s)[kBlockN], int o) {
    float a[11];
#pragma unroll
    for (int i = 0; i < 10; ++i) a[i] = max3f(s[o + 3 * i], s[o + 3 * i + 1], s[o + 3 * i + 2]);
    a[10] = fmaxf(s[o + 30], s[o + 31]);
    const float b0 = max3f(a[0], a[1], a[2]), b1 = max3f(a[3], a[4], a[5]), b2 = max3f(a[6], a[7], a[8]);
    return max3f(max3f(b0, b1, b2), a[9], a[10]);
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
    auto bar_s_full = [&](int b) { return base + C::kBarOff + 8u * (1 + 2 * C::kStages + b); };
    auto bar_p_full = [&](int b) { return base + C::kBarOff + 8u * (3 + 2 * C::kStages + b); };
    auto bar_o_done = [&](int b) { return base + C::kBarOff + 8u * (5 + 2 * C::kStages + b); };
    auto bar_m_ready = [&](int qd, int b) { return base + C::kBarOff + 8u * (7 + 2 * C::kStages + 2 * qd + b); };
    const uint32_t bar_drain = base + C::kBarOff + 8u * (15 + 2 * C::kStages);
    uint32_t* const tmem_holder = reinterpret_cast<uint32_t*>(base_ptr + C::kMiscOff);
    volatile int* const abort_flag = reinterpret_cast<volatile int*>(base_ptr + C::kMiscOff + 4);
    float* const mref = reinterpret_cast<float*>(base_ptr + C::kMrefOff);     // [parity][row]
    float* const epi = reinterpret_cast<float*>(base_ptr + C::kEpiOff);       // m [2][row], l [2][row]
    const uint32_t q_tile = base + C::kQOff;
    auto kv_slot = [&](int s) { return base + C::kKvOff + (uint32_t)(s * C::kTileBytes); };

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // ---- work item: (b, h, 128-row block); heavy causal blocks launch first
    const int num_m = (int)gridDim.x;
    const int m_blk = p.causal ? (num_m - 1 - (int)blockIdx.x) : (int)blockIdx.x;
    const int h = blockIdx.y;
    const int b = blockIdx.z;
    const int m0 = m_blk * kBlockM;
    int kl = p.Nk;
    if (p.key_lens != nullptr) {
        kl = p.key_lens[b];
        kl = kl < 0 ? 0 : (kl > p.Nk ? p.Nk : kl);
    }
    const int off = p.Nk - p.Nq;  // causal diagonal offset (bottom-right aligned)
    // K/V tiles this Q tile must visit: enough for its last real row.
    const int last_row = min(m0 + kBlockM - 1, p.Nq - 1);
    const int n_kv = (row_key_limit(last_row, kl, off, p.causal) + kBlockN - 1) / kBlockN;

    // ---- setup: barriers (producer lane 0), TMEM (MMA warp)
    if (warp == kProducerWarp && lane == 0) {
        mbar_init(bar_q_full, 1);
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(bar_kv_full(s), 1);
            mbar_init(bar_kv_empty(s), 1);
        }
        mbar_init(bar_s_full(0), 1);
        mbar_init(bar_s_full(1), 1);
        for (int b2 = 0; b2 < 2; ++b2) {
            mbar_init(bar_p_full(b2), kSoftmaxWarps / 2);
            mbar_init(bar_o_done(b2), 1);
        }
        for (int i = 0; i < 8; ++i) mbar_init(bar_m_ready(i >> 1, i & 1), 1);
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

    // The K/V load order, shared by producer and MMA issuer: K0, K1, then for
    // every j: V_j followed by K_{j+2} -- the order the MMAs consume them in.
    if (warp >= kProducerWarp) {
      setmaxnreg_dec<kRegsControl>();   // whole warpgroup 2, one instruction
      if (warp == kProducerWarp) {
        // =========================================================== TMA producer
        if (lane == 0 && n_kv > 0) {
            const uint64_t pol_kv = policy_evict_last();
            const uint64_t pol_q = policy_evict_first();
            mbar_arrive_expect_tx(bar_q_full, (uint32_t)C::kTileBytes);
            for (int bx = 0; bx < C::kBoxes; ++bx)
                tma_load_4d(q_tile + bx * kSwizzleBoxBytes, &tm_q, bar_q_full, bx * 64, m0, h, b, pol_q);
            int cnt = 0;
            int issued[C::kStages];
            for (int s = 0; s < C::kStages; ++s) issued[s] = -1;
            auto load = [&](const CUtensorMap* m, int j) {
                const int s = cnt % C::kStages;
                const uint32_t round = (uint32_t)(cnt / C::kStages);
                if (!wait_bounded(bar_kv_empty(s), (round & 1u) ^ 1u, abort_flag, p.wait_limit)) return false;
                mbar_arrive_expect_tx(bar_kv_full(s), (uint32_t)C::kTileBytes);
                for (int bx = 0; bx < C::kBoxes; ++bx)
                    tma_load_4d(kv_slot(s) + bx * kSwizzleBoxBytes, m, bar_kv_full(s), bx * 64, j * kBlockN, h,
                                b, pol_kv);
                issued[s] = cnt;
                ++cnt;
                return true;
            };
            bool ok = load(&tm_k, 0);
            if (ok && n_kv > 1) ok = load(&tm_k, 1);
            for (int j = 0; j < n_kv && ok; ++j) {
                ok = load(&tm_v, j);
                if (ok && j + 2 < n_kv) ok = load(&tm_k, j + 2);
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
            int cnt = 0;
            auto next_slot = [&](int& s) {
                s = cnt % C::kStages;
                const bool r = wait_bounded(bar_kv_full(s), (uint32_t)((cnt / C::kStages) & 1), abort_flag,
                                            p.wait_limit);
                ++cnt;
                return r;
            };
            auto mma_qk = [&](int buf, int slot) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t koff = (uint32_t)((kk / 4) * kSwizzleBoxBytes + (kk % 4) * 32);
                    const uint64_t a = smem_desc_sw128(q_tile + koff, 16, 1024);
                    const uint64_t bb = smem_desc_sw128(kv_slot(slot) + koff, 16, 1024);
                    umma_ss(tmem + C::col_s(buf), a, bb, C::kIdescQK, kk > 0 ? 1u : 0u);
                }
            };
            auto mma_pv = [&](int buf, int slot, bool accumulate) {
#pragma unroll
                for (int kk = 0; kk < kBlockN / 16; ++kk) {
                    // keys 16kk..16kk+15 of P: 8 bf16-pair columns per step
                    const uint32_t a_col = C::col_s(buf) + (uint32_t)(kk * 8);
                    const uint64_t bb =
                        smem_desc_sw128(kv_slot(slot) + (uint32_t)(kk * 16 * 128), kSwizzleBoxBytes, 1024);
                    umma_ts(tmem + C::kColO, tmem + a_col, bb, C::kIdescPV, (accumulate || kk > 0) ? 1u : 0u);
                }
            };
            int s = 0;
            for (int j = 0; j < 2 && j < n_kv && ok; ++j) {
                ok = next_slot(s);
                if (!ok) break;
                tc_fence_after();
                mma_qk(j, s);
                umma_commit(bar_s_full(j));
                umma_commit(bar_kv_empty(s));
            }
            for (int j = 0; j < n_kv && ok; ++j) {
                ok = next_slot(s);  // V_j
                if (ok) ok = wait_bounded(bar_p_full(j & 1), (uint32_t)((j >> 1) & 1), abort_flag, p.wait_limit);
                if (!ok) break;
                tc_fence_after();
                mma_pv(j & 1, s, j > 0);
                umma_commit(bar_o_done(j & 1));
                umma_commit(bar_kv_empty(s));
                if (j + 2 < n_kv) {
                    ok = next_slot(s);  // K_{j+2}
                    if (!ok) break;
                    tc_fence_after();
                    // overwrites S(j) and P(j): issued after the PV that reads P(j)
                    mma_qk(j & 1, s);
                    umma_commit(bar_s_full(j & 1));
                    umma_commit(bar_kv_empty(s));
                }
            }
            // drain: every MMA and commit of this CTA has landed before TMEM is freed
            umma_commit(bar_drain);
            (void)wait_bounded(bar_drain, 0, abort_flag, p.wait_limit);
        }
        __syncwarp();
      }
    } else {
        setmaxnreg_inc<kRegsSoftmax>();   // warpgroups 0 and 1
        // =========================================================== softmax: one thread per row, alternate tiles
        const int qd = warp & 3;                     // TMEM lane quadrant
        const int par = warp >> 2;                   // this warp takes the tiles j with j % 2 == par
        const int r = qd * 32 + lane;                // row inside the tile == TMEM lane
        const uint32_t lane_off = (uint32_t)(qd * 32) << 16;
        const int row = m0 + r;
        const int lim = row_key_limit(row, kl, off, p.causal);
        const float c = p.scale_log2;
        float m_seen = -INFINITY;  // newest reference max this thread knows (log2 units)
        float l = 0.f;             // sum of this warp's probabilities, relative to m_seen
        bool ok = true;

        for (int j = par; j < n_kv; j += 2) {
            const int buf = j & 1;
            bool good = wait_bounded(bar_s_full(buf), (uint32_t)((j >> 1) & 1), abort_flag, p.wait_limit);
            if (!__all_sync(0xffffffffu, good)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const int kbase = j * kBlockN;
            // warp-uniform: the element mask runs only on tiles that cross a row's key limit
            const bool masked = __any_sync(0xffffffffu, kbase + kBlockN > lim);
            float s[kBlockN];
            {
                uint32_t u[kBlockN];
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4)
                    tmem_ld32(tmem + lane_off + C::col_s(buf) + 32u * q4,
                              *reinterpret_cast<uint32_t(*)[32]>(&u[32 * q4]));
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < kBlockN; ++i) {
                    reg_after_wait(u[i]);
                    s[i] = __uint_as_float(u[i]);
                }
            }
            if (masked) {
#pragma unroll
                for (int i = 0; i < kBlockN; ++i)
                    if (kbase + i >= lim) s[i] = -INFINITY;
            }
            const float mx = fmaxf(fmaxf(chunk_max32(s, 0), chunk_max32(s, 32)),
                                   fmaxf(chunk_max32(s, 64), chunk_max32(s, 96)));
            // reference max after tile j-1, published by the partner warp
            float m_prev = -INFINITY;
            if (j > 0) {
                good = wait_bounded(bar_m_ready(qd, (j - 1) & 1), (uint32_t)(((j - 1) >> 1) & 1), abort_flag,
                                    p.wait_limit);
                if (!__all_sync(0xffffffffu, good)) {
                    ok = false;
                    break;
                }
                m_prev = mref[((j - 1) & 1) * kBlockM + r];
            }
            const float t_max = mx * c;   // c > 0, so -inf stays -inf
            const float m_cur = (t_max > m_prev + kRescaleThreshold) ? t_max : m_prev;
            if (j + 1 < n_kv) {
                mref[buf * kBlockM + r] = m_cur;
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_m_ready(qd, buf));
            }
            if (m_cur != m_seen) {
                l *= ex2_approx(m_seen - m_cur);  // 0 while m_seen is -inf
                m_seen = m_cur;
            }
            const float mu = (m_cur == -INFINITY) ? 0.f : m_cur;
            float2 l0 = make_float2(0.f, 0.f), l1 = make_float2(0.f, 0.f);
            const uint32_t taddr_p = tmem + lane_off + C::col_s(buf);
            if (masked) {
                exp_store_half<0, 0>(s, c, mu, taddr_p, l0, l1);
                exp_store_half<0, 1>(s, c, mu, taddr_p, l0, l1);
            } else {
                exp_store_half<C::kEmuPairs, 0>(s, c, mu, taddr_p, l0, l1);
                exp_store_half<C::kEmuPairs, 1>(s, c, mu, taddr_p, l0, l1);
            }
            l += (l0.x + l0.y) + (l1.x + l1.y);
            if (j > 0) {
                // O holds tiles < j relative to m_prev once the PV of tile j-1 is done
                good = wait_bounded(bar_o_done((j - 1) & 1), (uint32_t)(((j - 1) >> 1) & 1), abort_flag,
                                    p.wait_limit);
                if (!__all_sync(0xffffffffu, good)) {
                    tmem_wait_st();
                    ok = false;
                    break;
                }
                tc_fence_after();
                const float alpha = (m_cur != m_prev) ? ex2_approx(m_prev - m_cur) : 1.f;
                if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
                    for (int q4 = 0; q4 < D / 32; ++q4) {
                        const uint32_t ocol = tmem + lane_off + C::kColO + 32u * q4;
                        uint32_t u[32];
                        tmem_ld32(ocol, u);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; i += 2) {
                            reg_after_wait(u[i]);
                            reg_after_wait(u[i + 1]);
                            const float2 v = __fmul2_rn(
                                make_float2(__uint_as_float(u[i]), __uint_as_float(u[i + 1])),
                                make_float2(alpha, alpha));
                            u[i] = __float_as_uint(v.x);
                            u[i + 1] = __float_as_uint(v.y);
                        }
                        tmem_st32(ocol, u);
                    }
                }
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_p_full(buf));
        }

        // ---------------------------------------------------------- epilogue
        // Exits and skipped stores are decided jointly (bar.red.or), so a wait
        // that ran out never leaves another warp stuck at a named barrier.
        const bool have_o = n_kv > 0;
        bool good = ok;
        if (good && have_o) {
            good = wait_bounded(bar_o_done((n_kv - 1) & 1), (uint32_t)(((n_kv - 1) >> 1) & 1), abort_flag,
                                p.wait_limit);
            good = __all_sync(0xffffffffu, good);
            if (good) tc_fence_after();
        }
        epi[par * kBlockM + r] = m_seen;
        epi[(2 + par) * kBlockM + r] = l;
        good = !named_bar_or(kBarQuadBase + qd, 64, !good);
        // both warps' sums, brought to the final (largest) reference max
        const float m_oth = epi[(par ^ 1) * kBlockM + r];
        const float l_oth = epi[(2 + (par ^ 1)) * kBlockM + r];
        const float m_fin = fmaxf(m_seen, m_oth);
        const float l_row = (m_seen == m_fin ? l : l * ex2_approx(m_seen - m_fin)) +
                            (m_oth == m_fin ? l_oth : l_oth * ex2_approx(m_oth - m_fin));
        if (good) {
            const float inv_l = (l_row > 0.f) ? 1.f / l_row : 0.f;
#pragma unroll
            for (int q4 = 0; q4 < D / 64; ++q4) {
                const int col0 = par * (D / 2) + 32 * q4;   // first O column of this chunk
                uint32_t u[32];
                if (have_o) {
                    tmem_ld32(tmem + lane_off + C::kColO + (uint32_t)col0, u);
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
                    pkd[i] = pack_bf16x2(__uint_as_float(u[2 * i]) * inv_l, __uint_as_float(u[2 * i + 1]) * inv_l);
                // 4 x 16-byte chunks of row r; chunk cc of the row lives in box cc/8,
                // swizzled position (cc%8) ^ (r%8) inside the row's 128 bytes.
#pragma unroll
                for (int v4 = 0; v4 < 4; ++v4) {
                    const int cc = col0 / 8 + v4;
                    const uint32_t addr = q_tile + (uint32_t)((cc >> 3) * kSwizzleBoxBytes + r * 128 +
                                                              (((cc & 7) ^ (r & 7)) << 4));
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(pkd[4 * v4]),
                                 "r"(pkd[4 * v4 + 1]), "r"(pkd[4 * v4 + 2]), "r"(pkd[4 * v4 + 3])
                                 : "memory");
                }
            }
            if (par == 0 && row < p.Nq) {
                const float lse = (l_row > 0.f) ? (m_fin + lg2_approx(l_row)) * 0.69314718055994531f : -INFINITY;
                p.lse[((size_t)b * p.H + h) * (size_t)p.Nq + row] = lse;
            }
        }
        fence_proxy_async_smem();
        const bool any_bad = named_bar_or(kBarSoftmaxAll, kSoftmaxWarps * 32, !good);
        if (!any_bad && threadIdx.x == 0) {
            for (int bx = 0; bx < C::kBoxes; ++bx)
                tma_store_4d(&tm_o, q_tile + bx * kSwizzleBoxBytes, bx * 64, m0, h, b);
            bulk_commit_group();
            bulk_wait_group_read0();
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
