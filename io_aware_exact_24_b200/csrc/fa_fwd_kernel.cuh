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
//  * warp 8 (one elected lane) loads Q once and then streams the K tiles (128
//    keys), warp 10 the V tiles, each through its own ring of shared-memory
//    slots with TMA (128B-swizzled boxes of 64 columns x 128 rows), one
//    full/empty mbarrier pair per slot -- the double buffering
//    "FlashAttention：把注意力从公式写成数据流" (section "端侧与专用加速器") names
//    for hiding loads;
//  * two warps (one elected lane each) issue the tcgen05 MMAs: warp 9 the
//    S(i) = Q K_i^T products into the TMEM score buffer(s), warp 11 the
//    O += P(j) V_j products.  The two streams touch disjoint TMEM and
//    separate rings, so neither waits for the other and the tensor core is
//    fed by one while the other waits on a barrier;
//  * P is written to its own TMEM buffers (three, 64 columns of bf16 pairs
//    each), never over the scores: a PV product followed by a QK^T product
//    into the columns it has just read is a write-after-read on TMEM that the
//    tensor core resolves by draining.  Scores are read out within a few
//    hundred cycles of landing, so one score buffer (two at d = 64, where
//    TMEM has room) keeps the QK^T stream going;
//  * warps 0-7 do the online softmax, one thread per query row: warps q and
//    q+4 both own TMEM lanes 32q..32q+31 and take the K/V tiles in turn (even
//    / odd), each holding a whole 128-key row in registers.  A score buffer
//    is handed back as soon as it has been read, so the next QK^T product
//    overlaps the exponentials.  Only the running reference max passes
//    between the two warps (shared memory + an mbarrier); each keeps its own
//    partial row sums.  Exponentials are taken in the exp2 domain, some on
//    MUFU and some with a polynomial on the FMA pipe;
//  * V is extended by a column block of ones, so the PV product also
//    accumulates the row sums of the bf16 P it uses (next to O, in TMEM, and
//    rescaled with it); the softmax keeps only the unrounded sum for the LSE;
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
constexpr int kGroups = 2;          // softmax warps per TMEM lane quadrant (tiles taken in turn)
constexpr int kSoftmaxWarps = 4 * kGroups;
constexpr int kNumThreads = 384;    // 8 softmax warps, 2 TMA producers, 2 MMA issuers
constexpr int kProducerWarp = 8;    // Q and the K tiles
constexpr int kMmaWarp = 9;         // issues the QK^T products (and owns the TMEM allocation)
constexpr int kVProducerWarp = 10;  // the V tiles
constexpr int kPvWarp = 11;         // issues the PV products
constexpr int kTmemCols = 512;
// Registers are allocated per warpgroup: 384 threads x 168 at launch, then the
// two softmax warpgroups take 200 and the producer/MMA warpgroup keeps 104
// (2*128*200 + 128*104 <= 384*168).
constexpr uint32_t kRegsSoftmax = 200;
constexpr uint32_t kRegsControl = 104;
constexpr int kSwizzleBoxBytes = 128 * 128;  // one 64-column x 128-row bf16 box
constexpr float kRescaleThreshold = 8.0f;    // log2 units: rescale only if max grows > 2^8
constexpr int kStatusTimeout = -6;           // FA_ERR_DEVICE_TIMEOUT
// additive score bias of the kernel instantiation
constexpr int kBiasNone = 0;     // plain scores
constexpr int kBiasSlopes = 1;   // -slope_h * |i + off - j|
constexpr int kBiasTable = 2;    // a per-head table indexed by the clamped relative position
// named barriers (epilogue only): 1..4 join the warps of a lane quadrant, 5 spans all softmax warps
constexpr uint32_t kBarQuadBase = 1;
constexpr uint32_t kBarSoftmaxAll = 5;

struct FwdParams {
    float* lse;                 // [B,H,Nq]
    const int32_t* key_lens;    // [B] or nullptr
    int B, H, Nq, Nk;
    float scale_log2;           // scale * log2(e), > 0
    int causal;
    int window_left;            // sliding window: keys before i+off-window_left are masked; < 0: none
    const float* slopes;        // [H] additive positional bias -slopes[h]*|i+off-j| (kBias == kBiasSlopes)
    // custom positional bias (kBias == kBiasTable): fp32 [H, 2*bias_radius+1];
    // key j of query i gets bias_table[h][clamp(j - (i+off), -R, R) + R]
    const float* bias_table;
    int bias_radius;
    // packed variable-length mode only: sequence b holds query tokens
    // cu_q[b] .. cu_q[b+1]-1 and key tokens cu_k[b] .. cu_k[b+1]-1; Nq / Nk
    // are then the token totals, Q/O are [Nq, H, D], K/V [Nk, H, D], LSE [Nq, H]
    const int32_t* cu_q;
    const int32_t* cu_k;
    __nv_bfloat16* o_packed;    // O of the packed mode (written with plain stores)
    unsigned long long wait_limit;  // clock64 cycles per wait before giving up
    // split-KV mode only: each Q tile's K/V tiles are cut into num_splits
    // contiguous ranges, one CTA each, writing a partial result per range
    int num_splits;
    float* o_part;              // [num_splits, B, H, Nq, D] fp32, O of the range / its own l
    float* lse_part;            // [num_splits, B, H, Nq] fp32, LSE of the range (-inf if empty)
    // arrival words per (query block, h, b), [B, H, num query blocks], any initial
    // contents: (ticket << 16) | arrivals of the call whose ticket is split_ticket;
    // the last CTA of a query block to arrive merges its ranges into o_out / lse
    unsigned long long* split_counter;
    unsigned long long split_ticket;   // 48 bits, different for every call
    __nv_bfloat16* o_out;       // final O [B,H,Nq,D] of the split-KV mode
    // dense single-pass mode: > 1 reorders the CTAs' work (see the kernel); 0 or 1 keeps
    // blockIdx = (query block, h, b)
    int head_group;
    // E4M3 mode only: the V descale, applied to O in the epilogue
    float o_scale;
};

// kF8 = false: bf16 Q, K, V and P (kind::f16 MMAs).  kF8 = true: E4M3 Q, K, V
// with per-tensor descales, P rounded to E4M3 (kind::f8f6f4 MMAs, K = 32 per
// instruction).  Shared-memory tiles are 128-row boxes whose rows are one
// swizzle span wide: 128 bytes (128B swizzle) whenever a Q/K/V row has at
// least 128 bytes, else 64 bytes (64B swizzle: E4M3 at d = 64).
template <int D, bool kF8 = false>
struct Cfg {
    static_assert(D == 64 || D == 128, "head dim");
    static constexpr int kElemBytes = kF8 ? 1 : 2;
    static constexpr int kRowBytes = D * kElemBytes;             // one Q / K / V row
    static constexpr int kSwz = kRowBytes < 128 ? kRowBytes : 128;   // swizzle span (bytes)
    static constexpr uint32_t kSwzMode = kSwz == 128 ? 2u : 4u;  // descriptor layout: 128B / 64B swizzle
    static constexpr int kBoxBytes = kBlockM * kSwz;             // one box: 128 rows x one span
    static constexpr int kBoxCols = kSwz / kElemBytes;           // elements per box row
    static constexpr int kBoxes = kRowBytes / kSwz;              // boxes per Q / K / V row
    static constexpr int kOBoxes = D / 64;                       // 128B-swizzled boxes per bf16 O row
    static constexpr int kTileBytes = kBlockM * kRowBytes;       // one Q / K / V tile
    static constexpr int kKPerMma = 32 / kElemBytes;             // K extent of one MMA (32 bytes)
    static constexpr int kStagesK = (kTileBytes <= 16384) ? 4 : 2;   // K ring slots
    static constexpr int kStagesV = (kTileBytes <= 16384) ? 4 : 2;   // V ring slots
    // A V slot holds the tile (kBoxes boxes) followed by one box of ones: the
    // PV product runs with N = D + 16 and its last 16 output columns
    // accumulate the row sums of the rounded P it multiplies.
    static constexpr int kVSlotBytes = kTileBytes + kBoxBytes;
    static constexpr uint32_t kOnesWord = kF8 ? 0x38383838u : 0x3F803F80u;   // 1.0 in E4M3 / bf16
    static constexpr int kNPV = D + 16;
    static constexpr int kStages = kStagesK + kStagesV;
    // Of every 8 pairs of probabilities, this many are computed on the FMA pipe
    // (exp2_fma2) and the rest on MUFU, so neither unit is the lone bottleneck.
#ifdef FA_EMU_PAIRS_D64
    static constexpr int kEmuPairs = (D == 64 || kF8) ? FA_EMU_PAIRS_D64 : FA_EMU_PAIRS_D128;
#else
    static constexpr int kEmuPairs = (D == 64 || kF8) ? 2 : 0;   // measured best on B200
#endif
    static constexpr int kQOff = 0;
    static constexpr int kKOff = kTileBytes;
    static constexpr int kVOff = kKOff + kStagesK * kTileBytes;
    static constexpr int kBarOff = kVOff + kStagesV * kVSlotBytes;
    static constexpr int kSBufs = 1;                             // TMEM score buffers
    static constexpr int kPBufs = 3;                             // TMEM probability buffers
    // barriers: q_full, k_full[S], k_empty[S], v_full[S], v_empty[S],
    // s_full[2 (per softmax warp)], s_free[2], p_full[3], pv_done[3],
    // 8 unused slots (the reference max now travels in tagged words), drain
    static constexpr int kNumBars = 1 + 2 * kStages + 2 + 2 + 3 + 3 + 8 + 1;
    static_assert(kSBufs <= 2 && kPBufs <= 3, "barrier slots");
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;      // tmem base, abort flag
    static constexpr int kMrefOff = kMiscOff + 16;               // published reference max [group][row], 8 B each
    static constexpr int kEpiOff = kMrefOff + kGroups * kBlockM * 8;  // epilogue exchange: m, lu [2][row] each
    static constexpr int kSmemUsed = kEpiOff + 2 * kGroups * kBlockM * 4 + 1024;  // + alignment slack
    // One CTA per SM either way (it holds all 512 TMEM columns), so the smaller
    // E4M3 layouts reserve as much shared memory as the bf16 d = 64 one.
    static constexpr int kSmemBytes = kSmemUsed < 200 * 1024 ? 200 * 1024 : kSmemUsed;
    static_assert(kSmemBytes <= 232448, "dynamic shared memory per CTA on sm_100");
    // The bf16 O tile is staged for its TMA store from the start of the Q
    // buffer on; with 8-bit inputs it also covers the first K slot(s) (idle by then).
    static_assert(kOBoxes * kSwizzleBoxBytes <= kVOff, "O staging area");
    // TMEM columns: the S buffer at 0..127, the P buffers (kPCols each: bf16
    // pairs or E4M3 quads) after it, then O (D columns) and its row-sum
    // columns; the O rescale also touches the 16 unused columns after those.
    static constexpr uint32_t kPCols = kBlockN * kElemBytes / 4;
    __host__ __device__ static constexpr uint32_t col_s(int b) { return 128u * b; }
    __host__ __device__ static constexpr uint32_t col_p(int b) { return 128u * kSBufs + kPCols * b; }
    static constexpr uint32_t kColO = 128u * kSBufs + kPCols * kPBufs;
    static constexpr uint32_t kColL = kColO + D;                 // row sum of the rounded P
    static_assert(kColO + D + 32 <= 512, "TMEM columns");
    // Instruction descriptors: D = f32, M = 128; A/B format 1 = bf16 (kind::f16)
    // or 0 = E4M3 (kind::f8f6f4).
    //   QK^T: A=Q K-major, B=K K-major, N=128.
    //   PV: A=P (TMEM, K-major), B=[V | ones] MN-major, N=D+16.
    static constexpr uint32_t kFmt = kF8 ? 0u : 1u;
    static constexpr uint32_t kIdescQK = (1u << 4) | (kFmt << 7) | (kFmt << 10) | (0u << 15) |
                                         (0u << 16) | ((uint32_t)(kBlockN >> 3) << 17) |
                                         ((uint32_t)(kBlockM >> 4) << 24);
    static constexpr uint32_t kIdescPV = (1u << 4) | (kFmt << 7) | (kFmt << 10) | (0u << 15) |
                                         (1u << 16) | ((uint32_t)(kNPV >> 3) << 17) |
                                         ((uint32_t)(kBlockM >> 4) << 24);
};

// Shared-memory matrix descriptor with sm_100 version bits; `mode` is the
// layout field: 2 = 128-byte swizzle, 4 = 64-byte swizzle.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo, uint32_t mode) {
    uint64_t d = 0;
    d |= (uint64_t)((addr & 0x3FFFFu) >> 4);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;   // descriptor version for tcgen05
    d |= (uint64_t)(mode & 7u) << 61;
    return d;
}
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    return smem_desc(addr, lbo, sbo, 2u);
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
        // plain try_wait: an explicit suspend-time hint wakes the waiter
        // noticeably later after the phase completes
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if ((unsigned long long)(clock64() - t0) > limit) {
            *abort_flag = 1;
            atomicExch(&g_fa_status, kStatusTimeout);
            return false;
        }
    }
}

// The reference max one softmax warp hands to the other warp of its lane quadrant,
// per row: one 64-bit shared word {tile index (high half), max bits (low half)},
// written and read in single accesses, so a reader that sees the tile it waits for
// also sees that tile's max.  The reader polls until the word names its tile (the
// writer cannot move on to a later tile before it has read this reader's next word).
__device__ __forceinline__ unsigned long long ld_relaxed_shared_u64(uint32_t addr) {
    unsigned long long v;
    asm volatile("ld.relaxed.cta.shared.b64 %0, [%1];" : "=l"(v) : "r"(addr) : "memory");
    return v;
}
__device__ __forceinline__ void st_relaxed_shared_u64(uint32_t addr, unsigned long long v) {
    asm volatile("st.relaxed.cta.shared.b64 [%0], %1;" ::"r"(addr), "l"(v) : "memory");
}
__device__ __forceinline__ bool wait_tagged_max(uint32_t addr, uint32_t tag, float& m, volatile int* abort_flag,
                                                unsigned long long limit) {
    unsigned long long v = ld_relaxed_shared_u64(addr);
    if ((uint32_t)(v >> 32) != tag) {
        const long long t0 = clock64();
        while (true) {
            v = ld_relaxed_shared_u64(addr);
            if ((uint32_t)(v >> 32) == tag) break;
            if (*abort_flag) return false;
            if ((unsigned long long)(clock64() - t0) > limit) {
                *abort_flag = 1;
                atomicExch(&g_fa_status, kStatusTimeout);
                return false;
            }
        }
    }
    m = __uint_as_float((uint32_t)v);
    return true;
}

// Bounded wait for this thread's own asynchronous work (a TMA copy it issued, or
// the commit of its MMAs) when winding down: unlike wait_bounded it does not
// give up when another role of the CTA has raised the abort flag, because
// shared memory and TMEM must not be released while that work may still land.
// The limit is the default one (about a second), not a caller's shorter limit.
constexpr unsigned long long kDrainWaitLimit = 1ull << 31;
__device__ __forceinline__ bool wait_own_work(uint32_t bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((unsigned long long)(clock64() - t0) > kDrainWaitLimit) {
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

// p = 2^(s*c - mu) for keys 64*h2 .. 64*h2+63 of the thread's row, rounded
// to bf16 pairs (kF8 = false) or E4M3 quads (kF8 = true) and stored to its
// TMEM lane: 32 (or 16) columns from taddr_p + 32*h2 (or 16*h2).  lu sums the
// unrounded p (for the log-sum-exp; the sum of the rounded p, which
// normalises O, comes out of the PV product).  kEmu of every 8 pairs go
// through exp2_fma2, the rest through MUFU ex2 (which maps -inf to 0, so masked
// tiles use kEmu = 0).  p <= 2^8 (the reference-max threshold), inside E4M3's
// range.
template <int kEmu, int h2, bool kF8 = false>
__device__ __forceinline__ void exp_store_half(const float (&s)[kBlockN], float c, float mu, uint32_t taddr_p,
                                               float2& lu) {
    const float2 c2 = make_float2(c, c);
    const float2 nmu = make_float2(-mu, -mu);
    uint32_t w[kF8 ? 16 : 32];
    float2 prev = make_float2(0.f, 0.f);
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
        if constexpr (kF8) {
            if (i & 1)
                w[i >> 1] = pack_e4m3x4(prev.x, prev.y, e.x, e.y);
            else
                prev = e;
        } else {
            w[i] = pack_bf16x2(e.x, e.y);
        }
        lu = __fadd2_rn(lu, e);
    }
    if constexpr (kF8)
        tmem_st16(taddr_p + 16u * h2, w);
    else
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

// First key a query row may see: the sliding-window start (0 without a window).
__device__ __forceinline__ int row_key_start(int row, int off, int window_left) {
    if (window_left < 0) return 0;
    const long long c = (long long)row + off - window_left;
    return c < 0 ? 0 : (c > 0x7fffffffLL ? 0x7fffffff : (int)c);
}

// Number of keys (prefix length) a query row may see.
__device__ __forceinline__ int row_key_limit(int row, int kl, int off, int causal) {
    if (!causal) return kl;
    long long c = (long long)row + off + 1;
    c = c < 0 ? 0 : c;
    return c < kl ? (int)c : kl;
}

// Counts one arrival of this call's CTAs of a query block and tells whether it
// was the last of n.  The word holds (ticket << 16) | count.  An arrival that
// finds another ticket there (an earlier call, or whatever the workspace held)
// tries once to claim the word with (ticket << 16) | 0: the first claim wins,
// and every later claim fails because the word has changed, so it needs no
// retry; then each arrival adds 1 (one atomic, no retry loop however many
// ranges arrive at once).  Every add lands on a word that already carries this
// call's ticket, so the words need no reset between calls; two calls share a
// word only if their 48-bit tickets are equal.
__device__ __forceinline__ bool split_arrive_last(unsigned long long* word, unsigned long long ticket, int n) {
    const unsigned long long cur = atomicAdd(word, 0ull);
    if ((cur >> 16) != ticket) atomicCAS(word, cur, ticket << 16);
    const unsigned long long old = atomicAdd(word, 1ull);
    return (int)(old & 0xffffull) + 1 == n;
}

// Split-KV merge, run by the 256 softmax threads of a CTA once its partial
// (O_s, LSE_s) is in global memory: the CTA counts its arrival for its query
// block, and the last of the block's num_splits CTAs to arrive merges every
// range of the block's rows.  With M = max_s LSE_s and w_s = e^(LSE_s - M):
//   O = sum_s w_s O_s / sum_s w_s,   LSE = M + ln sum_s w_s
// (each O_s is normalised by its own range's sum, so w_s carries that sum;
// this is the online softmax's running-max rule applied to whole ranges).  A
// row whose ranges are all empty (M = -inf) gets O = 0, LSE = -inf; an empty
// range has LSE_s = -inf, so w_s = 0 and its O_s (zeros) adds nothing.  Work
// items are (row, 4 columns), spread over the 256 threads, so a decode block
// with one row still loads its ranges' partials in parallel.  The arrival
// words need no reset (split_arrive_last).
template <int D>
__device__ __forceinline__ void split_merge(const FwdParams& p, uint8_t* flag_smem, int n_split, int num_m, int m_blk,
                                            int m0, int h, int b) {
    volatile int* const flag = reinterpret_cast<volatile int*>(flag_smem);
    const size_t grp = ((size_t)b * p.H + h) * (size_t)num_m + (size_t)m_blk;
    if (threadIdx.x == 0) {
        // every softmax thread fenced its own partial stores before the barrier
        // that preceded this arrival
        *flag = split_arrive_last(p.split_counter + grp, p.split_ticket, n_split) ? 1 : 0;
    }
    named_bar_sync(kBarSoftmaxAll, kSoftmaxWarps * 32);
    if (!*flag) return;
    __threadfence();   // the other ranges' partials, published before their arrivals
    constexpr int kC4 = D / 4;
    const int rows = min(kBlockM, p.Nq - m0);
    const size_t rows_total = (size_t)p.B * p.H * (size_t)p.Nq;
    const size_t row0 = ((size_t)b * p.H + h) * (size_t)p.Nq + (size_t)m0;
    for (int it = threadIdx.x; it < rows * kC4; it += kSoftmaxWarps * 32) {
        const int rr = it / kC4, c4 = it - rr * kC4;
        const size_t rg = row0 + (size_t)rr;
        float mx = -INFINITY;
#pragma unroll 4
        for (int sp = 0; sp < n_split; ++sp) mx = fmaxf(mx, __ldcg(p.lse_part + sp * rows_total + rg));
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        float wsum = 0.f;
        if (mx != -INFINITY) {
#pragma unroll 4
            for (int sp = 0; sp < n_split; ++sp) {
                const float ls = __ldcg(p.lse_part + sp * rows_total + rg);
                const float4 v = __ldcg(reinterpret_cast<const float4*>(p.o_part + (sp * rows_total + rg) * D) + c4);
                const float w = (ls == -INFINITY) ? 0.f : expf(ls - mx);
                acc.x = fmaf(w, v.x, acc.x);
                acc.y = fmaf(w, v.y, acc.y);
                acc.z = fmaf(w, v.z, acc.z);
                acc.w = fmaf(w, v.w, acc.w);
                wsum += w;
            }
        }
        const float inv = (wsum > 0.f) ? 1.f / wsum : 0.f;
        uint2 pk;
        pk.x = pack_bf16x2(acc.x * inv, acc.y * inv);
        pk.y = pack_bf16x2(acc.z * inv, acc.w * inv);
        *reinterpret_cast<uint2*>(p.o_out + rg * D + 4 * c4) = pk;
        if (c4 == 0) p.lse[rg] = (wsum > 0.f) ? mx + logf(wsum) : -INFINITY;
    }
}

// kSplit = false: the whole forward (O and LSE).  kSplit = true: the split-KV
// forward ("FlashAttention：把注意力从公式写成数据流", section "端侧与专用加速器",
// and "[2205.14135] FlashAttention: Fast and Memory-Efficient Exact Attention
// with IO-Awareness", its note on the decode case): partial (O, LSE) for one
// contiguous range of K/V tiles, merged by the block's last CTA (split_merge).
// kVarlen = true: packed variable-length batches (FwdParams::cu_q / cu_k);
// the TMA maps then view [tokens, H, D] as (D, H, tokens, 1).
// kF8 = true: E4M3 inputs (see Cfg); O is still bf16 and FwdParams::o_scale
// (the V descale) multiplies it in the epilogue.
// kBias: kBiasNone, or an additive positional bias on the scores
// ("FlashAttention：把注意力从公式写成数据流", section "精度、掩码和边界情况":
// positional biases are among the mask variants): kBiasSlopes, a linear
// distance penalty per head, or kBiasTable, any per-head function of the
// relative position j - (i + off) given as a table, clamped at +-R.
template <int D, bool kSplit = false, bool kVarlen = false, bool kF8 = false, int kBias = kBiasNone>
__global__ void __launch_bounds__(kNumThreads, 1)
    fa_fwd_sm100_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                        const FwdParams p) {
    using C = Cfg<D, kF8>;
    static_assert(!kF8 || (!kSplit && !kVarlen), "E4M3 inputs: dense single-pass mode");
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw_base = smem_addr(smem_raw);
    const uint32_t base = (raw_base + 1023u) & ~1023u;
    uint8_t* const base_ptr = smem_raw + (base - raw_base);

    const uint32_t bar_q_full = base + C::kBarOff;
    // ring r = 0 (K, kStagesK slots) or 1 (V, kStagesV slots): full barriers
    // of both rings, then the empty ones
    auto bar_full = [&](int r, int s) { return base + C::kBarOff + 8u * (1 + r * C::kStagesK + s); };
    auto bar_empty = [&](int r, int s) { return base + C::kBarOff + 8u * (1 + C::kStages + r * C::kStagesK + s); };
    auto bar_s_full = [&](int g) { return base + C::kBarOff + 8u * (1 + 2 * C::kStages + g); };
    auto bar_s_free = [&](int b) { return base + C::kBarOff + 8u * (3 + 2 * C::kStages + b); };
    auto bar_p_full = [&](int b) { return base + C::kBarOff + 8u * (5 + 2 * C::kStages + b); };
    auto bar_pv_done = [&](int b) { return base + C::kBarOff + 8u * (8 + 2 * C::kStages + b); };
    const uint32_t bar_drain = base + C::kBarOff + 8u * (19 + 2 * C::kStages);
    uint32_t* const tmem_holder = reinterpret_cast<uint32_t*>(base_ptr + C::kMiscOff);
    volatile int* const abort_flag = reinterpret_cast<volatile int*>(base_ptr + C::kMiscOff + 4);
    // [group][row]: {tile, reference max} words (wait_tagged_max)
    const uint32_t mref_w = base + C::kMrefOff;
    float* const epi = reinterpret_cast<float*>(base_ptr + C::kEpiOff);       // m, l, lu [group][row] each
    const uint32_t q_tile = base + C::kQOff;
    auto ring_slot = [&](int r, int s) {
        return r == 0 ? base + C::kKOff + (uint32_t)(s * C::kTileBytes)
                      : base + C::kVOff + (uint32_t)(s * C::kVSlotBytes);
    };

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // ---- work item: (b, h, 128-row block[, K/V range]); heavy causal blocks launch first
    const int n_split = kSplit ? p.num_splits : 1;
    const int split = kSplit ? (int)blockIdx.x % n_split : 0;
    int blk = kSplit ? (int)blockIdx.x / n_split : (int)blockIdx.x;
    const int num_m = (int)gridDim.x / n_split;
    int h = blockIdx.y;
    int b = blockIdx.z;
    if constexpr (!kSplit && !kVarlen) {
        if (p.head_group > 1) {
            // CTAs start in linear order.  Walk the (b, h) problems in groups of
            // head_group, and inside a group take every problem's block of rank 0
            // (the heaviest, when causal), then rank 1, ...: the blocks running at
            // any time share few K/V tensors (they stay in L2), and the light
            // blocks of a group come last, where they fill the tail.
            const int HB = p.H * p.B;
            const int lin = (int)blockIdx.x + num_m * ((int)blockIdx.y + p.H * (int)blockIdx.z);
            const int per_group = num_m * p.head_group;
            const int gi = lin / per_group;
            const int w = lin - gi * per_group;
            const int hcnt = min(p.head_group, HB - gi * p.head_group);
            blk = w / hcnt;
            const int hb = gi * p.head_group + (w - blk * hcnt);
            h = hb % p.H;
            b = hb / p.H;
        }
    }
    const int m_blk = p.causal ? (num_m - 1 - blk) : blk;
    const int m0 = m_blk * kBlockM;
    // this (b, h) problem's sizes, and where its rows start in the tensors
    int Nq_b = p.Nq, Nk_b = p.Nk, q_base = 0, k_base = 0;
    if constexpr (kVarlen) {
        q_base = p.cu_q[b];
        k_base = p.cu_k[b];
        Nq_b = p.cu_q[b + 1] - q_base;
        Nk_b = p.cu_k[b + 1] - k_base;
        // offsets outside the packed tensors make the sequence empty (nothing is written)
        if (q_base < 0 || Nq_b < 0 || q_base > p.Nq - Nq_b) Nq_b = 0;
        if (k_base < 0 || Nk_b < 0 || k_base > p.Nk - Nk_b) Nk_b = 0;
        if (m0 >= Nq_b) return;   // the whole CTA, before any setup
    }
    int kl = Nk_b;
    if (p.key_lens != nullptr) {
        kl = p.key_lens[b];
        kl = kl < 0 ? 0 : (kl > Nk_b ? Nk_b : kl);
    }
    const int off = Nk_b - Nq_b;  // causal diagonal offset (bottom-right aligned)
    // TMA coordinates of a 128-row tile starting at row `r0` of this problem:
    // (column, row, head, batch) dense, (column, head, token, 0) packed
    auto tile_coords = [&](int base_tok, int r0, int& c1, int& c2, int& c3) {
        if constexpr (kVarlen) {
            c1 = h;
            c2 = base_tok + r0;
            c3 = 0;
        } else {
            c1 = r0;
            c2 = h;
            c3 = b;
        }
    };
    // K/V tiles this Q tile must visit: enough for its last real row; in
    // split-KV mode this CTA takes tiles t0 .. t0+n_kv-1 of them.
    const int last_row = min(m0 + kBlockM - 1, Nq_b - 1);
    const int n_all = (row_key_limit(last_row, kl, off, p.causal) + kBlockN - 1) / kBlockN;
    // With a sliding window the first row's window start bounds the tiles from below.
    const int t_lo = min(row_key_start(m0, off, p.window_left) / kBlockN, n_all);
    const int n_span = n_all - t_lo;
    const int t0 = t_lo + (kSplit ? (int)((long long)split * n_span / n_split) : 0);
    const int n_kv = kSplit ? t_lo + (int)((long long)(split + 1) * n_span / n_split) - t0 : n_span;

    // ---- setup: barriers (producer lane 0), TMEM (MMA warp)
    if (warp == kProducerWarp && lane == 0) {
        mbar_init(bar_q_full, 1);
        for (int r2 = 0; r2 < 2; ++r2)
            for (int s = 0; s < (r2 == 0 ? C::kStagesK : C::kStagesV); ++s) {
                mbar_init(bar_full(r2, s), 1);
                mbar_init(bar_empty(r2, s), 1);
            }
        for (int g = 0; g < 2; ++g) {
            mbar_init(bar_s_full(g), 1);
            mbar_init(bar_s_free(g), 4);    // one arrival per lane quadrant
        }
        for (int b2 = 0; b2 < C::kPBufs; ++b2) {
            mbar_init(bar_p_full(b2), 4);   // one arrival per lane quadrant
            mbar_init(bar_pv_done(b2), 1);
        }
        mbar_init(bar_drain, 2);   // one commit from each MMA issuer
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
        prefetch_tensormap(&tm_o);
    }
    // no reference max published yet: tag 0xffffffff names no tile
    for (int i = threadIdx.x; i < kGroups * kBlockM; i += kNumThreads)
        st_relaxed_shared_u64(mref_w + 8u * (uint32_t)i, ~0ull);
    if (warp == kMmaWarp) {
        tmem_alloc(smem_addr(tmem_holder), kTmemCols);
        tmem_relinquish();
        tc_fence_before();
    }
    // the ones box of every V slot (TMA writes only the boxes before it)
    for (int i = threadIdx.x; i < C::kStagesV * (C::kBoxBytes / 16); i += kNumThreads) {
        const int sl = i / (C::kBoxBytes / 16);
        const uint32_t a = ring_slot(1, sl) + (uint32_t)C::kTileBytes + (uint32_t)(i % (C::kBoxBytes / 16)) * 16u;
        asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(a), "r"(C::kOnesWord) : "memory");
    }
    fence_proxy_async_smem();   // visible to the tensor core's reads
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    if (warp >= kProducerWarp) {
      setmaxnreg_dec<kRegsControl>();   // whole warpgroup 2, one instruction
      if (warp == kProducerWarp || warp == kVProducerWarp) {
        // =========================================================== TMA producers
        // Each streams its own tensor, tiles 0 .. n_kv-1 in order, through its
        // own ring; warp 8 also loads the Q tile first.
        const int rg = (warp == kProducerWarp) ? 0 : 1;
        const CUtensorMap* const tm = (rg == 0) ? &tm_k : &tm_v;
        const int ns = (rg == 0) ? C::kStagesK : C::kStagesV;
        if (lane == 0 && n_kv > 0) {
            const uint64_t pol_kv = policy_evict_last();
            if (rg == 0) {
                mbar_arrive_expect_tx(bar_q_full, (uint32_t)C::kTileBytes);
                int qc1, qc2, qc3;
                tile_coords(q_base, m0, qc1, qc2, qc3);
                for (int bx = 0; bx < C::kBoxes; ++bx)
                    tma_load_4d(q_tile + bx * C::kBoxBytes, &tm_q, bar_q_full, bx * C::kBoxCols, qc1, qc2, qc3,
                                policy_evict_first());
            }
            bool ok = true;
            int j = 0;
            for (; j < n_kv && ok; ++j) {
                const int s = j % ns;
                const uint32_t round = (uint32_t)(j / ns);
                ok = wait_bounded(bar_empty(rg, s), (round & 1u) ^ 1u, abort_flag, p.wait_limit);
                if (!ok) break;
                mbar_arrive_expect_tx(bar_full(rg, s), (uint32_t)C::kTileBytes);
                int kc1, kc2, kc3;
                tile_coords(k_base, (t0 + j) * kBlockN, kc1, kc2, kc3);
                for (int bx = 0; bx < C::kBoxes; ++bx)
                    tma_load_4d(ring_slot(rg, s) + bx * C::kBoxBytes, tm, bar_full(rg, s), bx * C::kBoxCols, kc1, kc2,
                                kc3, pol_kv);
            }
            // Before the CTA can exit, every copy this producer issued that may
            // still be in flight (Q, and at most one per slot, the newest ones)
            // must have landed.  On the normal path the consumers have waited for
            // them already (or are about to); after a timeout anywhere in the CTA
            // they may not have, so this wait ignores the abort flag.
            if (rg == 0) (void)wait_own_work(bar_q_full, 0);
            for (int c2 = (j > ns ? j - ns : 0); c2 < j; ++c2)
                (void)wait_own_work(bar_full(rg, c2 % ns), (uint32_t)((c2 / ns) & 1));
        }
        __syncwarp();
    } else {
        // =========================================================== MMA issuers
        if (lane == 0 && n_kv > 0) {
            bool ok = true;
            if (warp == kMmaWarp) {
                ok = wait_bounded(bar_q_full, 0, abort_flag, p.wait_limit);
                for (int i = 0; i < n_kv && ok; ++i) {
                    // S(i - kSBufs) has been read into registers (first tiles: free buffer)
                    const int t = i - C::kSBufs;
                    if (t >= 0)
                        ok = wait_bounded(bar_s_free(t % C::kSBufs), (uint32_t)((t / C::kSBufs) & 1), abort_flag,
                                          p.wait_limit);
                    const int sl = i % C::kStagesK;
                    if (ok) ok = wait_bounded(bar_full(0, sl), (uint32_t)((i / C::kStagesK) & 1), abort_flag,
                                              p.wait_limit);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t slot = ring_slot(0, sl);
#pragma unroll
                    for (int kk = 0; kk < D * C::kElemBytes / 32; ++kk) {
                        // 32 bytes of every row per MMA, kSwz / 32 steps per box
                        const uint32_t koff =
                            (uint32_t)((kk * 32 / C::kSwz) * C::kBoxBytes + (kk * 32) % C::kSwz);
                        const uint64_t a = smem_desc(q_tile + koff, 16, 8 * C::kSwz, C::kSwzMode);
                        const uint64_t bb = smem_desc(slot + koff, 16, 8 * C::kSwz, C::kSwzMode);
                        if constexpr (kF8)
                            umma_ss_f8(tmem + C::col_s(i % C::kSBufs), a, bb, C::kIdescQK, kk > 0 ? 1u : 0u);
                        else
                            umma_ss(tmem + C::col_s(i % C::kSBufs), a, bb, C::kIdescQK, kk > 0 ? 1u : 0u);
                    }
                    umma_commit(bar_s_full(i & 1));   // per softmax warp: tiles i, i+2, ...
                    umma_commit(bar_empty(0, sl));
                }
            } else {
                for (int j = 0; j < n_kv && ok; ++j) {
                    // P(j) is in TMEM, and V_j has landed
                    const int pb = j % C::kPBufs;
                    ok = wait_bounded(bar_p_full(pb), (uint32_t)((j / C::kPBufs) & 1), abort_flag, p.wait_limit);
                    const int sl = j % C::kStagesV;
                    if (ok) ok = wait_bounded(bar_full(1, sl), (uint32_t)((j / C::kStagesV) & 1), abort_flag,
                                              p.wait_limit);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t slot = ring_slot(1, sl);
#pragma unroll
                    for (int kk = 0; kk < kBlockN / C::kKPerMma; ++kk) {
                        // keys kK*kk .. kK*kk+kK-1 of P (kK = 16 bf16 or 32 E4M3): 8 TMEM
                        // columns of P, kK rows (one swizzle span each) of the V slot per step
                        const uint32_t a_col = C::col_p(pb) + (uint32_t)(kk * 8);
                        const uint64_t bb =
                            smem_desc(slot + (uint32_t)(kk * C::kKPerMma * C::kSwz), C::kBoxBytes, 8 * C::kSwz,
                                      C::kSwzMode);
                        if constexpr (kF8)
                            umma_ts_f8(tmem + C::kColO, tmem + a_col, bb, C::kIdescPV, (j > 0 || kk > 0) ? 1u : 0u);
                        else
                            umma_ts(tmem + C::kColO, tmem + a_col, bb, C::kIdescPV, (j > 0 || kk > 0) ? 1u : 0u);
                    }
                    umma_commit(bar_pv_done(pb));
                    umma_commit(bar_empty(1, sl));
                }
            }
            // drain: every MMA and commit of this CTA has landed before TMEM is
            // freed (the barrier completes once both issuers have committed);
            // this wait ignores the abort flag, so a wound-down CTA drains too
            umma_commit(bar_drain);
            (void)wait_own_work(bar_drain, 0);
        }
        __syncwarp();
      }
    } else {
        setmaxnreg_inc<kRegsSoftmax>();   // warpgroups 0 and 1
        // =========================================================== softmax: one thread per row, tiles in turn
        const int qd = warp & 3;                     // TMEM lane quadrant
        const int g = warp >> 2;                     // this warp takes the tiles j with j % 2 == g
        const int r = qd * 32 + lane;                // row inside the tile == TMEM lane
        const uint32_t lane_off = (uint32_t)(qd * 32) << 16;
        const int row = m0 + r;
        const int lim = row_key_limit(row, kl, off, p.causal);
        const int lo = row_key_start(row, off, p.window_left);   // 0 without a window
        // additive positional bias, in log2 units per unit of distance (warp-uniform switch)
        constexpr bool has_bias = kBias != kBiasNone;
        const float alpha = (kBias == kBiasSlopes) ? p.slopes[h] * 1.4426950408889634f : 0.f;
        const float* const trow =
            (kBias == kBiasTable) ? p.bias_table + (size_t)h * (2 * (size_t)p.bias_radius + 1) + p.bias_radius : nullptr;
        const float c = p.scale_log2;
        float m_seen = -INFINITY;  // newest reference max this thread knows (log2 units)
        float lu = 0.f;            // the same sum before rounding (for the LSE)
        bool ok = true;

        for (int j = g; j < n_kv; j += 2) {
            const uint32_t use = (uint32_t)((j >> 1) & 1);   // phase parity of this tile in buffers g
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
                    tmem_ld32(tmem + lane_off + C::col_s(j % C::kSBufs) + 32u * q4,
                              *reinterpret_cast<uint32_t(*)[32]>(&u[32 * q4]));
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < kBlockN; ++i) {
                    reg_after_wait(u[i]);
                    s[i] = __uint_as_float(u[i]);
                }
            }
            // the score buffer is free for S(j + kSBufs)
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_s_free(j % C::kSBufs));
            const int kbase = (t0 + j) * kBlockN;
            // warp-uniform: the element mask runs only on tiles that cross a row's key limit
            const bool masked = __any_sync(0xffffffffu, kbase + kBlockN > lim || kbase < lo);
            if constexpr (kBias == kBiasSlopes) {
                // t_i = s_i * c - alpha * |row + off - (kbase + i)|; from here on the
                // scores are in log2 units already (scale factor 1)
                const float d0 = (float)(row + off - kbase);
#pragma unroll
                for (int i = 0; i < kBlockN; ++i) s[i] = fmaf(s[i], c, -alpha * fabsf(d0 - (float)i));
            } else if constexpr (kBias == kBiasTable) {
                // t_i = s_i * c + log2(e) * table[clamp(r0 + i, -R, R)], r0 the relative
                // position of the tile's first key; tiles inside [-R, R] for the whole
                // warp skip the clamp.  Masked keys are overwritten with -inf below.
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
            // reference max after tile j-1, published by the other warp of the quadrant
            float m_prev = -INFINITY;
            if (j > 0) {
                good = wait_tagged_max(mref_w + 8u * (uint32_t)((g ^ 1) * kBlockM + r), (uint32_t)(j - 1), m_prev,
                                       abort_flag, p.wait_limit);
                if (!__all_sync(0xffffffffu, good)) {
                    ok = false;
                    break;
                }
            }
            const float t_max = mx * cs;  // cs > 0, so -inf stays -inf
            const float m_cur = (t_max > m_prev + kRescaleThreshold) ? t_max : m_prev;
            if (j + 1 < n_kv)
                st_relaxed_shared_u64(mref_w + 8u * (uint32_t)(g * kBlockM + r),
                                      ((unsigned long long)(uint32_t)j << 32) | __float_as_uint(m_cur));
            if (m_cur != m_seen) {
                const float f = ex2_approx(m_seen - m_cur);  // 0 while m_seen is -inf
                lu *= f;
                m_seen = m_cur;
            }
            const float mu = (m_cur == -INFINITY) ? 0.f : m_cur;
            // P buffer j % 3 was last read by PV(j-3)
            const int pb = j % C::kPBufs;
            if (j >= C::kPBufs) {
                good = wait_bounded(bar_pv_done(pb), (uint32_t)(((j - C::kPBufs) / C::kPBufs) & 1), abort_flag,
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
            // O holds tiles < j relative to m_prev.  Only when some row of this
            // warp moved its reference max does O have to be rescaled, and only
            // then must PV(j-1) be complete first; PV(j) waits for this warp's
            // P-ready arrival, so it cannot have started.
            const float alpha = (m_cur != m_prev) ? ex2_approx(m_prev - m_cur) : 1.f;
            if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
                good = wait_bounded(bar_pv_done((j - 1) % C::kPBufs), (uint32_t)(((j - 1) / C::kPBufs) & 1),
                                    abort_flag, p.wait_limit);
                if (!__all_sync(0xffffffffu, good)) {
                    tmem_wait_st();
                    ok = false;
                    break;
                }
                tc_fence_after();
#pragma unroll
                for (int q4 = 0; q4 < D / 32 + 1; ++q4) {   // O and its row-sum columns
                    const uint32_t ocol = tmem + lane_off + C::kColO + 32u * q4;
                    uint32_t u[32];
                    tmem_ld32(ocol, u);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; i += 2) {
                        reg_after_wait(u[i]);
                        reg_after_wait(u[i + 1]);
                        const float2 v = __fmul2_rn(make_float2(__uint_as_float(u[i]), __uint_as_float(u[i + 1])),
                                                    make_float2(alpha, alpha));
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

        // ---------------------------------------------------------- epilogue
        // Exits and skipped stores are decided jointly (bar.red.or), so a wait
        // that ran out never leaves another warp stuck at a named barrier.
        const bool have_o = n_kv > 0;
        bool good = ok;
        if (good && have_o) {
            // every MMA of the CTA is done: the drain commit completes its only phase
            good = wait_bounded(bar_drain, 0, abort_flag, p.wait_limit);
            good = __all_sync(0xffffffffu, good);
            if (good) tc_fence_after();
        }
        epi[g * kBlockM + r] = m_seen;
        epi[(2 + g) * kBlockM + r] = lu;
        good = !named_bar_or(kBarQuadBase + qd, 64, !good);
        // both warps' sums, brought to the final (largest) reference max, in a
        // fixed order so both warps get the same bits
        const float m0w = epi[r], m1w = epi[kBlockM + r];
        const float m_fin = fmaxf(m0w, m1w);
        const float f0 = (m0w == m_fin) ? 1.f : ex2_approx(m0w - m_fin);
        const float f1 = (m1w == m_fin) ? 1.f : ex2_approx(m1w - m_fin);
        const float lu_row = epi[2 * kBlockM + r] * f0 + epi[3 * kBlockM + r] * f1;   // gives the LSE
        if (good) {
            // O and the sum of the bf16 P it was built from share every rescale,
            // so O / l needs no reference max
            float l_row = 0.f;
            if (have_o) {
                uint32_t u[32];
                tmem_ld32(tmem + lane_off + C::kColL, u);
                tmem_wait_ld();
                reg_after_wait(u[0]);
                l_row = __uint_as_float(u[0]);
            }
            float inv_l = (l_row > 0.f) ? 1.f / l_row : 0.f;
            if constexpr (kF8) inv_l *= p.o_scale;
#pragma unroll
            for (int q4 = 0; q4 < D / 64; ++q4) {
                const int col0 = g * (D / 2) + 32 * q4;   // first O column of this chunk
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
                if constexpr (kVarlen) {
                    // packed O: plain 16-byte stores of this row's chunk (a TMA
                    // store would also write rows of the next sequence)
                    if (row < Nq_b) {
                        uint4* dst = reinterpret_cast<uint4*>(
                            p.o_packed + ((size_t)(q_base + row) * p.H + h) * D + col0);
#pragma unroll
                        for (int v4 = 0; v4 < 4; ++v4) {
                            uint4 w4;
                            w4.x = pack_bf16x2(__uint_as_float(u[8 * v4]) * inv_l, __uint_as_float(u[8 * v4 + 1]) * inv_l);
                            w4.y = pack_bf16x2(__uint_as_float(u[8 * v4 + 2]) * inv_l,
                                               __uint_as_float(u[8 * v4 + 3]) * inv_l);
                            w4.z = pack_bf16x2(__uint_as_float(u[8 * v4 + 4]) * inv_l,
                                               __uint_as_float(u[8 * v4 + 5]) * inv_l);
                            w4.w = pack_bf16x2(__uint_as_float(u[8 * v4 + 6]) * inv_l,
                                               __uint_as_float(u[8 * v4 + 7]) * inv_l);
                            dst[v4] = w4;
                        }
                    }
                } else if constexpr (kSplit) {
                    // partial O of this K/V range, fp32, straight to global memory
                    if (row < p.Nq) {
                        float4* dst = reinterpret_cast<float4*>(
                            p.o_part + ((((size_t)split * p.B + b) * p.H + h) * (size_t)p.Nq + row) * D + col0);
#pragma unroll
                        for (int v4 = 0; v4 < 8; ++v4)
                            dst[v4] = make_float4(__uint_as_float(u[4 * v4]) * inv_l, __uint_as_float(u[4 * v4 + 1]) * inv_l,
                                                  __uint_as_float(u[4 * v4 + 2]) * inv_l,
                                                  __uint_as_float(u[4 * v4 + 3]) * inv_l);
                    }
                } else {
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
            }
            if (g == 0 && row < Nq_b) {
                const float lse = (lu_row > 0.f) ? (m_fin + lg2_approx(lu_row)) * 0.69314718055994531f : -INFINITY;
                if constexpr (kVarlen)
                    p.lse[(size_t)(q_base + row) * p.H + h] = lse;
                else if constexpr (kSplit)
                    p.lse_part[(((size_t)split * p.B + b) * p.H + h) * (size_t)p.Nq + row] = lse;
                else
                    p.lse[((size_t)b * p.H + h) * (size_t)p.Nq + row] = lse;
            }
        } else if constexpr (kSplit) {
            // a wait ran out (the device status records it): leave an empty
            // range (O = 0, LSE = -inf) rather than whatever the workspace held,
            // so the merge adds nothing stale from an earlier call
            if (row < p.Nq) {
                float4* dst = reinterpret_cast<float4*>(
                    p.o_part + ((((size_t)split * p.B + b) * p.H + h) * (size_t)p.Nq + row) * D + g * (D / 2));
#pragma unroll
                for (int v4 = 0; v4 < D / 8; ++v4) dst[v4] = make_float4(0.f, 0.f, 0.f, 0.f);
                if (g == 0) p.lse_part[(((size_t)split * p.B + b) * p.H + h) * (size_t)p.Nq + row] = -INFINITY;
            }
        }
        fence_proxy_async_smem();
        if constexpr (kSplit) __threadfence();   // this CTA's partials, before its arrival below
        const bool any_bad = named_bar_or(kBarSoftmaxAll, kSoftmaxWarps * 32, !good);
        if (!kSplit && !kVarlen && !any_bad && threadIdx.x == 0) {
            for (int bx = 0; bx < C::kOBoxes; ++bx)
                tma_store_4d(&tm_o, q_tile + bx * kSwizzleBoxBytes, bx * 64, m0, h, b);
            bulk_commit_group();
            bulk_wait_group_read0();
        }
        if constexpr (kSplit) split_merge<D>(p, base_ptr + C::kMiscOff + 8, n_split, num_m, m_blk, m0, h, b);
        tc_fence_before();
    }

    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}


}  // namespace fa
