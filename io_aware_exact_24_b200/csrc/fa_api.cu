// fa_api.cu -- host side of the C ABI declared in include/fa.h.
//
// Validates arguments (before any CUDA call), encodes the TMA tensor maps
// for Q, K, V and O, and launches the sm_100a kernel.  No allocation, no
// per-call state: the only caches are the driver's tensor-map encoder entry
// point and a per-device "kernel attributes set" flag.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <chrono>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>

#include <utility>

#include "fa.h"
#include "fa_bwd_kernel.cuh"
#include "fa_fwd_kernel.cuh"
#include "fa_fwd_persist.cuh"
#include "fa_decode_kernel.cuh"

// Dense forward launches use the persistent kernel (fa_fwd_persist.cuh); 0 keeps
// one CTA per query block to the end (the split-KV and packed modes always do).
#ifndef FA_PERSISTENT
#define FA_PERSISTENT 1
#endif

namespace {

constexpr int kVersion = 10000;  // 1.0.0

// Last FA_ERR_CUDA cause on this thread (what fa_last_error returns).
thread_local char t_last_error[256] = "";

int cuda_fail(const char* what, cudaError_t e) {
    snprintf(t_last_error, sizeof t_last_error, "%s: %s (%d)", what, cudaGetErrorString(e), (int)e);
    return FA_ERR_CUDA;
}
constexpr unsigned long long kWaitLimitCycles = 1ull << 31;  // ~1 s at B200 clocks
#ifndef FA_HEAD_GROUP_MB
#define FA_HEAD_GROUP_MB 48
#endif
// share of the 126 MB L2 that the K/V of the (b, h) problems in flight may take
constexpr long long kHeadGroupL2Bytes = (long long)FA_HEAD_GROUP_MB << 20;
// below this many query blocks per (b, h) the per-CTA fixed cost dominates and
// the plain order measured faster (GPT-2-sized causal problems, N = 1024)
constexpr unsigned kHeadGroupMinBlocks = 32;
// Longest K/V walk (tiles of 128 keys) for which the dense forward uses persistent CTAs.
constexpr int kPersistMaxTiles = 16;
constexpr int kMaxDevices = 64;
// fa_fwd_host pipelines its copies in chunks of heads: about this many chunks,
// at most kHostChunksMax
constexpr int kHostChunksTarget = 8;
constexpr int kHostChunksMax = 64;
// largest relative-position radius of a bias table (2^30: the table's
// 2R+1 entries and every clamped index stay within int range)
constexpr int kMaxBiasRadius = 1 << 30;

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encoder() {
    static std::once_flag once;
    static EncodeTiledFn fn = nullptr;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

struct DeviceState {
    std::once_flag once;
    int status = FA_OK;
    int num_sms = 148;   // multiProcessorCount, read once
};
DeviceState g_dev[kMaxDevices];

// Shared-memory limit of the persistent dense kernels of one head dim and input type.
template <int D, bool kF8>
cudaError_t set_persist_smem() {
    const int bytes = fa::PersistCfg<D, kF8>::kSmemBytes;
    cudaError_t e = cudaFuncSetAttribute(fa::fa_fwd_persist_kernel<D, kF8, fa::kBiasNone>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (!kF8) {
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(fa::fa_fwd_persist_kernel<D, kF8, fa::kBiasSlopes>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(fa::fa_fwd_persist_kernel<D, kF8, fa::kBiasTable>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    }
    return e;
}

// Per device, once: check the architecture and raise the kernels' shared-memory limit.
int prepare_device(int dev) {
    if (dev < 0 || dev >= kMaxDevices) return FA_ERR_UNSUPPORTED;
    DeviceState& st = g_dev[dev];
    std::call_once(st.once, [&] {
        int major = 0, minor = 0;
        cudaError_t e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
        if (e == cudaSuccess) e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
        if (e != cudaSuccess) {
            st.status = cuda_fail("cudaDeviceGetAttribute", e);
            return;
        }
        if (major != 10 || minor != 0) {  // built for sm_100a only
            st.status = FA_ERR_UNSUPPORTED;
            return;
        }
        int sms = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && sms > 0)
            st.num_sms = sms;
        e = cudaFuncSetAttribute(fa::fa_fwd_sm100_kernel<64, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 fa::Cfg<64>::kSmemBytes);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(fa::fa_fwd_sm100_kernel<128, false>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, fa::Cfg<128>::kSmemBytes);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(fa::fa_fwd_sm100_kernel<64, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     fa::Cfg<64>::kSmemBytes);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(fa::fa_fwd_sm100_kernel<128, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     fa::Cfg<128>::kSmemBytes);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(fa::fa_fwd_sm100_kernel<64, false, true>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, fa::Cfg<64>::kSmemBytes);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(fa::fa_fwd_sm100_kernel<128, false, true>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, fa::Cfg<128>::kSmemBytes);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(fa::fa_fwd_sm100_kernel<128, false, false, true>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, fa::Cfg<128, true>::kSmemBytes);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(fa::fa_fwd_sm100_kernel<64, false, false, true>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, fa::Cfg<64, true>::kSmemBytes);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(fa::fa_fwd_sm100_kernel<64, false, false, false, fa::kBiasSlopes>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, fa::Cfg<64>::kSmemBytes);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(fa::fa_fwd_sm100_kernel<128, false, false, false, fa::kBiasSlopes>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, fa::Cfg<128>::kSmemBytes);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(fa::fa_fwd_sm100_kernel<64, false, false, false, fa::kBiasTable>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, fa::Cfg<64>::kSmemBytes);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(fa::fa_fwd_sm100_kernel<128, false, false, false, fa::kBiasTable>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, fa::Cfg<128>::kSmemBytes);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(fa::fa_decode_splitkv_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     fa::DecCfg<64>::kSmemBytes);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(fa::fa_decode_splitkv_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     fa::DecCfg<128>::kSmemBytes);
#if FA_PERSISTENT
        if (e == cudaSuccess) e = set_persist_smem<64, false>();
        if (e == cudaSuccess) e = set_persist_smem<128, false>();
        if (e == cudaSuccess) e = set_persist_smem<64, true>();
        if (e == cudaSuccess) e = set_persist_smem<128, true>();
#endif
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(fa::fa_bwd_sm100_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     fa::BwdCfg<64>::kSmemBytes);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(fa::fa_bwd_sm100_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     fa::BwdCfg<128>::kSmemBytes);
        if (e != cudaSuccess) {
            st.status = cuda_fail("cudaFuncSetAttribute(MaxDynamicSharedMemorySize)", e);
            return;
        }
        st.status = FA_OK;
    });
    return st.status;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// Argument checks shared by fa_fwd and fa_fwd_host (no CUDA calls).
int validate(const void* q, const void* k, const void* v, const void* o, const void* lse, int B, int H,
             int N_q, int N_k, int d, float scale, const void* key_lens, bool* empty) {
    if (B < 0 || H < 0 || N_q < 0 || N_k < 0) return FA_ERR_INVALID_ARG;
    if (!std::isfinite(scale) || !(scale > 0.f)) return FA_ERR_INVALID_ARG;
    if (!(scale * 1.4426950408889634f > 0.f) || !std::isfinite(scale * 1.4426950408889634f))
        return FA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
    *empty = (B == 0 || H == 0 || N_q == 0);
    if (*empty) return FA_OK;
    if (B > 65535 || H > 65535) return FA_ERR_UNSUPPORTED;
    // TMA: global strides must stay below 2^40 bytes.
    const unsigned long long head_bytes_q = (unsigned long long)N_q * d * 2;
    const unsigned long long head_bytes_k = (unsigned long long)N_k * d * 2;
    if ((unsigned long long)H * head_bytes_q >= (1ull << 40) || (unsigned long long)H * head_bytes_k >= (1ull << 40))
        return FA_ERR_UNSUPPORTED;
    if (q == nullptr || o == nullptr || lse == nullptr) return FA_ERR_INVALID_ARG;
    if (N_k > 0 && (k == nullptr || v == nullptr)) return FA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(o, 16) || !aligned(lse, 4)) return FA_ERR_MISALIGNED;
    if (N_k > 0 && (!aligned(k, 16) || !aligned(v, 16))) return FA_ERR_MISALIGNED;
    if (key_lens != nullptr && !aligned(key_lens, 4)) return FA_ERR_MISALIGNED;
    return FA_OK;
}

// [B,H,N,d] viewed as a 4-D tensor (d, N, H, B), box of one swizzle span x 128
// rows: 128B swizzle with 64 bf16 or 128 one-byte (e4m3) columns, or, for rows of
// 64 one-byte elements, 64B swizzle with 64 columns (the kernel's Cfg geometry).
bool encode_bhnd(CUtensorMap* map, const void* ptr, int B, int H, int N, int d, bool e4m3 = false) {
    EncodeTiledFn enc = encoder();
    if (enc == nullptr) return false;
    const cuuint64_t eb = e4m3 ? 1 : 2;
    const cuuint64_t span = (cuuint64_t)d * eb < 128 ? (cuuint64_t)d * eb : 128;
    const cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)N, (cuuint64_t)H, (cuuint64_t)B};
    const cuuint64_t strides[3] = {(cuuint64_t)d * eb, (cuuint64_t)N * d * eb, (cuuint64_t)H * N * d * eb};
    const cuuint32_t box[4] = {(cuuint32_t)(span / eb), (cuuint32_t)fa::kBlockM, 1, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(map, e4m3 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4,
               const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               span == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The backward's fp32 dQ accumulator [B*H, N, d] as a 3-D tensor for tensor reduces:
// boxes of 32 columns x 32 rows (one warp's rows), 128-byte swizzle; rows past N
// (a ragged last query tile) lie outside the tensor and are skipped.
bool encode_dq_acc(CUtensorMap* map, float* ptr, int BH, int N, int d) {
    EncodeTiledFn enc = encoder();
    if (enc == nullptr) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)N, (cuuint64_t)BH};
    const cuuint64_t strides[2] = {(cuuint64_t)d * 4, (cuuint64_t)N * d * 4};
    const cuuint32_t box[3] = {32, 32, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, ptr, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A 48-bit ticket for each split-KV call: the arrival words in the workspace
// carry it, so they need no reset between calls (see split_arrive_last).  The
// sequence starts at a value taken from the clock, so a workspace left by
// another process is unlikely to hold a current ticket.
unsigned long long next_split_ticket() {
    static std::atomic<unsigned long long> seq{(unsigned long long)std::chrono::steady_clock::now()
                                                   .time_since_epoch()
                                                   .count() *
                                               0x9E3779B97F4A7C15ull};
    return (seq.fetch_add(1, std::memory_order_relaxed) + 1) & ((1ull << 48) - 1);
}

// Split-KV: partial results and per-block arrival words in the workspace.
struct SplitParts {
    int num_splits;   // 0: plain forward
    float* o_part;
    float* lse_part;
    unsigned long long* counter;   // arrival words [B, H, query blocks]
};

// Packed [T, H, d] bf16 viewed as (d, H, T, 1), box 64 x 1 x 128 x 1: the same
// 128-token x 64-column shared-memory tile as the dense map, for one head.
bool encode_thd(CUtensorMap* map, const void* ptr, int T, int H, int d) {
    EncodeTiledFn enc = encoder();
    if (enc == nullptr) return false;
    const cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)T, 1};
    const cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)H * d * 2, (cuuint64_t)T * H * d * 2};
    const cuuint32_t box[4] = {64, 1, (cuuint32_t)fa::kBlockM, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
int launch_varlen(const void* q, const void* k, const void* v, void* o, float* lse, const int32_t* cu_q,
                  const int32_t* cu_k, int B, int H, int T_q, int T_k, int max_q, float scale, int causal,
                  cudaStream_t stream) {
    CUtensorMap tq, tk, tv;
    const void* kp = T_k > 0 ? k : q;
    const void* vp = T_k > 0 ? v : q;
    const int tk_map = T_k > 0 ? T_k : 1;
    if (!encode_thd(&tq, q, T_q, H, D) || !encode_thd(&tk, kp, tk_map, H, D) || !encode_thd(&tv, vp, tk_map, H, D)) {
        snprintf(t_last_error, sizeof t_last_error, "cuTensorMapEncodeTiled failed");
        return FA_ERR_CUDA;
    }
    fa::FwdParams p{};
    p.lse = lse;
    p.key_lens = nullptr;
    p.B = B;
    p.H = H;
    p.Nq = T_q;
    p.Nk = T_k;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.causal = causal ? 1 : 0;
    p.window_left = -1;
    p.slopes = nullptr;
    p.cu_q = cu_q;
    p.cu_k = cu_k;
    p.o_packed = reinterpret_cast<__nv_bfloat16*>(o);
    p.wait_limit = kWaitLimitCycles;
    p.num_splits = 1;
    dim3 grid((unsigned)((max_q + fa::kBlockM - 1) / fa::kBlockM), (unsigned)H, (unsigned)B);
    // the O map is never used in this mode; any valid map will do
    fa::fa_fwd_sm100_kernel<D, false, true><<<grid, fa::kNumThreads, fa::Cfg<D>::kSmemBytes, stream>>>(tq, tk, tv,
                                                                                                     tq, p);
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? FA_OK : cuda_fail("kernel launch (packed variable-length)", e);
}

// Additive positional bias of a launch: none, per-head slopes, or a per-head table.
struct BiasArgs {
    int mode;             // fa::kBiasNone / kBiasSlopes / kBiasTable
    const float* ptr;     // slopes [H] or table [H, 2*radius+1]
    int radius;
};

// kF8: E4M3 Q, K, V (plain single-pass path only); o_scale multiplies O.
template <int D, bool kF8 = false>
int launch(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N_q, int N_k,
           float scale, int causal, const int32_t* key_lens, cudaStream_t stream, SplitParts sp = {0, nullptr, nullptr, nullptr},
           int window_left = -1, BiasArgs bias = {fa::kBiasNone, nullptr, 0}, float o_scale = 1.f,
           unsigned long long wait_limit = kWaitLimitCycles) {
    CUtensorMap tq, tk, tv, to;
    // With no keys the K/V maps are never read; give them a valid 1-row shape.
    const void* kp = N_k > 0 ? k : q;
    const void* vp = N_k > 0 ? v : q;
    const int nk_map = N_k > 0 ? N_k : 1;
    const int b_kv = N_k > 0 ? B : 1, h_kv = N_k > 0 ? H : 1;
    if (!encode_bhnd(&tq, q, B, H, N_q, D, kF8) || !encode_bhnd(&tk, kp, b_kv, h_kv, nk_map, D, kF8) ||
        !encode_bhnd(&tv, vp, b_kv, h_kv, nk_map, D, kF8) || !encode_bhnd(&to, o, B, H, N_q, D)) {
        snprintf(t_last_error, sizeof t_last_error, "cuTensorMapEncodeTiled failed");
        return FA_ERR_CUDA;
    }
    fa::FwdParams p{};
    p.lse = lse;
    p.key_lens = key_lens;
    p.B = B;
    p.H = H;
    p.Nq = N_q;
    p.Nk = N_k;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.causal = causal ? 1 : 0;
    p.window_left = window_left;
    p.slopes = bias.mode == fa::kBiasSlopes ? bias.ptr : nullptr;
    p.bias_table = bias.mode == fa::kBiasTable ? bias.ptr : nullptr;
    p.bias_radius = bias.radius;
    p.wait_limit = wait_limit;
    p.num_splits = sp.num_splits > 0 ? sp.num_splits : 1;
    p.o_part = sp.o_part;
    p.lse_part = sp.lse_part;
    p.split_counter = sp.counter;
    p.split_ticket = sp.num_splits > 0 ? next_split_ticket() : 0;
    p.o_out = reinterpret_cast<__nv_bfloat16*>(o);
    p.o_scale = o_scale;
    const int rows_per_cta = fa::kBlockM;
    const unsigned num_m = (unsigned)((N_q + rows_per_cta - 1) / rows_per_cta);
    if (sp.num_splits <= 0 && causal && num_m >= kHeadGroupMinBlocks) {
        // causal blocks differ in cost: order the CTAs heaviest first inside groups
        // of (b, h) problems whose K and V together fit in a share of the L2
        const long long kv_head = 4LL * N_k * D;
        long long hg = kHeadGroupL2Bytes / (kv_head > 0 ? kv_head : 1);
        const long long hb = (long long)H * B;
        p.head_group = (int)(hg < 1 ? 1 : (hg > hb ? hb : hg));
    }
#if FA_PERSISTENT
    // Dense launches with more query blocks than SMs and at most
    // kPersistMaxTiles K/V tiles per block run persistent CTAs that take over the
    // blocks not yet started: a block then costs about 1 us less of fixed time
    // (next Q and first S prefetched under this block's tail, no CTA start), but
    // the steady state is about 5 % slower per tile, so long blocks keep one CTA
    // per block (measured: padded 16x16x512 d64 +13 %, causal 8x12x1024 d64 +2 %,
    // 1x16x16384 d64 -4 %, causal 2x32x8000 d128 -5 %).
    int dev = 0;
    const bool persist = sp.num_splits <= 0 && cudaGetDevice(&dev) == cudaSuccess && dev >= 0 &&
                         dev < kMaxDevices && (long long)num_m * H * B > g_dev[dev].num_sms &&
                         (N_k + fa::kBlockN - 1) / fa::kBlockN <= kPersistMaxTiles;
    if (persist) {
        dim3 grid(num_m, (unsigned)H, (unsigned)B);
        const int smem = fa::PersistCfg<D, kF8>::kSmemBytes;
        if (bias.mode == fa::kBiasSlopes)
            fa::fa_fwd_persist_kernel<D, kF8, fa::kBiasSlopes><<<grid, fa::kNumThreads, smem, stream>>>(tq, tk, tv, p);
        else if (bias.mode == fa::kBiasTable)
            fa::fa_fwd_persist_kernel<D, kF8, fa::kBiasTable><<<grid, fa::kNumThreads, smem, stream>>>(tq, tk, tv, p);
        else
            fa::fa_fwd_persist_kernel<D, kF8, fa::kBiasNone><<<grid, fa::kNumThreads, smem, stream>>>(tq, tk, tv, p);
        const cudaError_t e = cudaGetLastError();
        return e == cudaSuccess ? FA_OK : cuda_fail("kernel launch (persistent)", e);
    }
#endif
    if constexpr (kF8) {
        dim3 grid(num_m, (unsigned)H, (unsigned)B);
        fa::fa_fwd_sm100_kernel<D, false, false, true>
            <<<grid, fa::kNumThreads, fa::Cfg<D, true>::kSmemBytes, stream>>>(tq, tk, tv, to, p);
        const cudaError_t e = cudaGetLastError();
        return e == cudaSuccess ? FA_OK : cuda_fail("kernel launch (e4m3)", e);
    } else {
    if (sp.num_splits <= 0) {
        dim3 grid(num_m, (unsigned)H, (unsigned)B);
        if (bias.mode == fa::kBiasSlopes)
            fa::fa_fwd_sm100_kernel<D, false, false, false, fa::kBiasSlopes>
                <<<grid, fa::kNumThreads, fa::Cfg<D>::kSmemBytes, stream>>>(tq, tk, tv, to, p);
        else if (bias.mode == fa::kBiasTable)
            fa::fa_fwd_sm100_kernel<D, false, false, false, fa::kBiasTable>
                <<<grid, fa::kNumThreads, fa::Cfg<D>::kSmemBytes, stream>>>(tq, tk, tv, to, p);
        else
            fa::fa_fwd_sm100_kernel<D, false><<<grid, fa::kNumThreads, fa::Cfg<D>::kSmemBytes, stream>>>(tq, tk, tv,
                                                                                                       to, p);
        const cudaError_t e = cudaGetLastError();
        return e == cudaSuccess ? FA_OK : cuda_fail("kernel launch", e);
    }
    // the arrival words need no reset: each call's arrivals carry its own ticket
    cudaError_t e;
    if (N_q == 1) {
        // one query row: matrix-vector products, streamed on the CUDA cores
        dim3 grid((unsigned)sp.num_splits, (unsigned)H, (unsigned)B);
        fa::fa_decode_splitkv_kernel<D><<<grid, fa::kDecThreads, fa::DecCfg<D>::kSmemBytes, stream>>>(
            tk, tv, reinterpret_cast<const __nv_bfloat16*>(q), p);
        e = cudaGetLastError();
        return e == cudaSuccess ? FA_OK : cuda_fail("kernel launch (decode)", e);
    }
    dim3 grid(num_m * (unsigned)sp.num_splits, (unsigned)H, (unsigned)B);
    fa::fa_fwd_sm100_kernel<D, true><<<grid, fa::kNumThreads, fa::Cfg<D>::kSmemBytes, stream>>>(tq, tk, tv, to, p);
    e = cudaGetLastError();
    return e == cudaSuccess ? FA_OK : cuda_fail("kernel launch (split-KV)", e);
    }
}

constexpr int kMaxSplits = 256;
constexpr int kDefaultNumSms = 148;   // B200, when no device can be queried

// Streaming multiprocessors of the current device (kDefaultNumSms without one).
int current_num_sms() {
    int ndev = 0, dev = -1, n = 0;
    if (cudaGetDeviceCount(&ndev) != cudaSuccess || ndev == 0 || cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
        cudaGetLastError();
        return kDefaultNumSms;
    }
    return n;
}

// Workspace of the split-KV forward: O partials, LSE partials, then one
// 64-bit arrival word per (query block, head, batch), each part 256-byte aligned.
struct SplitLayout {
    size_t o_part, lse_part, counter, total;
};
SplitLayout split_layout(int B, int H, int N_q, int d, int num_splits) {
    const size_t rows = (size_t)num_splits * B * H * N_q;
    const size_t blocks = (size_t)((N_q + fa::kBlockM - 1) / fa::kBlockM) * B * H;
    SplitLayout L{};
    L.o_part = 0;
    L.lse_part = (rows * d * 4 + 255) / 256 * 256;
    L.counter = L.lse_part + (rows * 4 + 255) / 256 * 256;
    L.total = L.counter + (blocks * 8 + 255) / 256 * 256;
    return L;
}

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct HostLayout {
    size_t q, k, v, o, lse, kl, total;
};
HostLayout host_layout(int B, int H, int N_q, int N_k, int d, int has_key_lens) {
    HostLayout L{};
    const size_t bh = (size_t)B * H;
    size_t off = 0;
    L.q = off;
    off = round_up(off + bh * N_q * d * 2, 256);
    L.k = off;
    off = round_up(off + bh * N_k * d * 2, 256);
    L.v = off;
    off = round_up(off + bh * N_k * d * 2, 256);
    L.o = off;
    off = round_up(off + bh * N_q * d * 2, 256);
    L.lse = off;
    off = round_up(off + bh * N_q * 4, 256);
    L.kl = off;
    off = round_up(off + (has_key_lens ? (size_t)B * 4 : 0), 256);
    L.total = off;
    return L;
}

// Workspace of the backward pass: D = rowsum(dO * O) [B,H,N_q] fp32, then the
// fp32 dQ accumulator [B,H,N_q,d], each 256-byte aligned.
struct BwdLayout {
    size_t dsum, dq_acc, total;
};
BwdLayout bwd_layout(int B, int H, int N_q, int d) {
    const size_t rows = (size_t)B * H * N_q;
    BwdLayout L{};
    L.dsum = 0;
    L.dq_acc = round_up(rows * 4, 256);
    L.total = L.dq_acc + round_up(rows * d * 4, 256);
    return L;
}

template <int D>
int launch_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout,
               void* dq, void* dk, void* dv, int B, int H, int N_q, int N_k, float scale, int causal,
               const int32_t* key_lens, uint8_t* ws, cudaStream_t stream,
               unsigned long long wait_limit = kWaitLimitCycles) {
    const BwdLayout L = bwd_layout(B, H, N_q, D);
    float* dsum = reinterpret_cast<float*>(ws + L.dsum);
    float* dq_acc = reinterpret_cast<float*>(ws + L.dq_acc);
    const long long rows = (long long)B * H * N_q;
    cudaError_t e;
    if (rows > 0) {
        fa::fa_bwd_pre_kernel<D><<<(unsigned)((rows + 7) / 8), 256, 0, stream>>>(
            reinterpret_cast<const __nv_bfloat16*>(o), reinterpret_cast<const __nv_bfloat16*>(dout), dsum, dq_acc,
            rows);
        e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail("kernel launch (backward preprocessing)", e);
    }
    const size_t kv_bytes = (size_t)B * H * N_k * D * 2;
    if (N_k > 0 && N_q == 0) {
        // no query: no gradient reaches K or V
        e = cudaMemsetAsync(dk, 0, kv_bytes, stream);
        if (e == cudaSuccess) e = cudaMemsetAsync(dv, 0, kv_bytes, stream);
        if (e != cudaSuccess) return cuda_fail("cudaMemsetAsync", e);
    }
    if (N_k > 0 && N_q > 0) {
        CUtensorMap tq, tk, tv, tdo, tdq;
        if (!encode_bhnd(&tq, q, B, H, N_q, D) || !encode_bhnd(&tk, k, B, H, N_k, D) ||
            !encode_bhnd(&tv, v, B, H, N_k, D) || !encode_bhnd(&tdo, dout, B, H, N_q, D) ||
            !encode_dq_acc(&tdq, dq_acc, B * H, N_q, D)) {
            snprintf(t_last_error, sizeof t_last_error, "cuTensorMapEncodeTiled failed");
            return FA_ERR_CUDA;
        }
        fa::BwdParams p{};
        p.lse = lse;
        p.dsum = dsum;
        p.dq_acc = dq_acc;
        p.dk = reinterpret_cast<__nv_bfloat16*>(dk);
        p.dv = reinterpret_cast<__nv_bfloat16*>(dv);
        p.key_lens = key_lens;
        p.B = B;
        p.H = H;
        p.Nq = N_q;
        p.Nk = N_k;
        p.scale = scale;
        p.scale_log2 = scale * 1.4426950408889634f;
        p.causal = causal ? 1 : 0;
        p.wait_limit = wait_limit;
        dim3 grid((unsigned)((N_k + 127) / 128), (unsigned)H, (unsigned)B);
        fa::fa_bwd_sm100_kernel<D><<<grid, fa::kBwdThreads, fa::BwdCfg<D>::kSmemBytes, stream>>>(tq, tk, tv, tdo, tdq, p);
        e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail("kernel launch (backward)", e);
    }
    if (rows > 0) {
        const long long n8 = rows * D / 8;
        fa::fa_bwd_post_kernel<<<(unsigned)((n8 + 255) / 256), 256, 0, stream>>>(
            dq_acc, reinterpret_cast<__nv_bfloat16*>(dq), scale, n8);
        e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail("kernel launch (backward dQ)", e);
    }
    return FA_OK;
}

__global__ void selftest_wait_kernel(unsigned long long limit) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        fa::mbar_init(fa::smem_addr(&bar), 1);
        abort_flag = 0;
        fa::fence_mbar_init();
    }
    __syncthreads();
    // Nothing ever arrives on this barrier: the wait must give up and record a timeout.
    (void)fa::wait_bounded(fa::smem_addr(&bar), 0, &abort_flag, limit);
    __syncthreads();
}

}  // namespace

extern "C" {

int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N_q, int N_k, int d,
           float scale, int causal, const int32_t* key_lens, fa_stream_t stream) {
    bool empty = false;
    int st = validate(q, k, v, o, lse, B, H, N_q, N_k, d, scale, key_lens, &empty);
    if (st != FA_OK || empty) return st;
    int dev = -1;
    int ndev = 0;
    if (cudaGetDeviceCount(&ndev) != cudaSuccess || ndev == 0) {
        cudaGetLastError();
        return FA_ERR_NO_DEVICE;
    }
    const cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail("cudaGetDevice", e);
    st = prepare_device(dev);
    if (st != FA_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (d == 64) return launch<64>(q, k, v, o, lse, B, H, N_q, N_k, scale, causal, key_lens, s);
    return launch<128>(q, k, v, o, lse, B, H, N_q, N_k, scale, causal, key_lens, s);
}

int fa_splitkv_num_splits(int B, int H, int N_q, int N_k) {
    if (B <= 0 || H <= 0 || N_q <= 0 || N_k <= 0) return 1;
    const long long ctas = (long long)((N_q + fa::kBlockM - 1) / fa::kBlockM) * B * H;
    const int tiles = (N_k + fa::kBlockN - 1) / fa::kBlockN;
    // One CTA fits per SM.  Once the plain grid covers most of the SMs the
    // K/V stream already runs at HBM speed and splitting only adds the merge;
    // below that, split into as many ranges as still fit in one wave, with at
    // least two K/V tiles per range.
    const int num_sms = current_num_sms();
    if (ctas >= num_sms * 4 / 5) return 1;
    long long s = num_sms / ctas;
    const long long cap = tiles / 2 > 1 ? tiles / 2 : 1;
    if (s > cap) s = cap;
    if (s > kMaxSplits) s = kMaxSplits;
    return s < 1 ? 1 : (int)s;
}

size_t fa_fwd_splitkv_workspace_size(int B, int H, int N_q, int d, int num_splits) {
    if (B < 0 || H < 0 || N_q < 0 || (d != 64 && d != 128) || num_splits < 1 || num_splits > kMaxSplits) return 0;
    return split_layout(B, H, N_q, d, num_splits).total;
}

int fa_fwd_splitkv(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N_q, int N_k,
                   int d, float scale, int causal, const int32_t* key_lens, int num_splits, void* workspace,
                   size_t workspace_bytes, fa_stream_t stream) {
    bool empty = false;
    int st = validate(q, k, v, o, lse, B, H, N_q, N_k, d, scale, key_lens, &empty);
    if (st != FA_OK) return st;
    if (num_splits < 1 || num_splits > kMaxSplits) return FA_ERR_INVALID_ARG;
    if (empty) return FA_OK;
    const SplitLayout L = split_layout(B, H, N_q, d, num_splits);
    if (workspace == nullptr || workspace_bytes < L.total) return FA_ERR_INVALID_ARG;
    if (!aligned(workspace, 256)) return FA_ERR_MISALIGNED;
    if ((unsigned long long)((N_q + fa::kBlockM - 1) / fa::kBlockM) * num_splits > 0x7fffffffull)
        return FA_ERR_UNSUPPORTED;
    int dev = -1;
    int ndev = 0;
    if (cudaGetDeviceCount(&ndev) != cudaSuccess || ndev == 0) {
        cudaGetLastError();
        return FA_ERR_NO_DEVICE;
    }
    const cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail("cudaGetDevice", e);
    st = prepare_device(dev);
    if (st != FA_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    const SplitParts sp{num_splits, reinterpret_cast<float*>(ws + L.o_part), reinterpret_cast<float*>(ws + L.lse_part),
                        reinterpret_cast<unsigned long long*>(ws + L.counter)};
    if (d == 64) return launch<64>(q, k, v, o, lse, B, H, N_q, N_k, scale, causal, key_lens, s, sp);
    return launch<128>(q, k, v, o, lse, B, H, N_q, N_k, scale, causal, key_lens, s, sp);
}

}  // extern "C"

namespace {

// Scratch of fa_fwd_splitkv_noalloc: one file-scope device array per process
// and device, sized once at module load (no allocation call at any time).
constexpr size_t kNoAllocScratchBytes = 16u << 20;
static __device__ __align__(256) unsigned char g_splitkv_scratch[kNoAllocScratchBytes];

struct ScratchState {
    std::once_flag once;
    int status = FA_OK;
    void* ptr = nullptr;
};
ScratchState g_scratch[kMaxDevices];

// Device address of the scratch array on `dev`, looked up once per device.
int scratch_address(int dev, void** out) {
    if (dev < 0 || dev >= kMaxDevices) return FA_ERR_UNSUPPORTED;
    ScratchState& st = g_scratch[dev];
    std::call_once(st.once, [&] {
        void* p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_splitkv_scratch);
        if (e != cudaSuccess) {
            st.status = cuda_fail("cudaGetSymbolAddress(split-KV scratch)", e);
            return;
        }
        st.ptr = p;
        st.status = FA_OK;
    });
    *out = st.ptr;
    return st.status;
}

}  // namespace

extern "C" {

int fa_fwd_splitkv_noalloc(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N_q,
                           int N_k, int d, float scale, int causal, const int32_t* key_lens, int num_splits,
                           fa_stream_t stream) {
    bool empty = false;
    int st = validate(q, k, v, o, lse, B, H, N_q, N_k, d, scale, key_lens, &empty);
    if (st != FA_OK) return st;
    if (num_splits < 1 || num_splits > kMaxSplits) return FA_ERR_INVALID_ARG;
    if (empty) return FA_OK;
    const SplitLayout L = split_layout(B, H, N_q, d, num_splits);
    if (L.total > kNoAllocScratchBytes) return FA_ERR_UNSUPPORTED;
    if ((unsigned long long)((N_q + fa::kBlockM - 1) / fa::kBlockM) * num_splits > 0x7fffffffull)
        return FA_ERR_UNSUPPORTED;
    int dev = -1;
    int ndev = 0;
    if (cudaGetDeviceCount(&ndev) != cudaSuccess || ndev == 0) {
        cudaGetLastError();
        return FA_ERR_NO_DEVICE;
    }
    const cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail("cudaGetDevice", e);
    st = prepare_device(dev);
    if (st != FA_OK) return st;
    void* scratch = nullptr;
    st = scratch_address(dev, &scratch);
    if (st != FA_OK) return st;
    // Every partial the merge reads is written first, and the arrival words carry
    // each call's own ticket, so nothing in the scratch has to start at zero.
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(scratch);
    const SplitParts sp{num_splits, reinterpret_cast<float*>(ws + L.o_part), reinterpret_cast<float*>(ws + L.lse_part),
                        reinterpret_cast<unsigned long long*>(ws + L.counter)};
    if (d == 64) return launch<64>(q, k, v, o, lse, B, H, N_q, N_k, scale, causal, key_lens, s, sp);
    return launch<128>(q, k, v, o, lse, B, H, N_q, N_k, scale, causal, key_lens, s, sp);
}

int fa_fwd_window(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N_q, int N_k,
                  int d, float scale, int causal, const int32_t* key_lens, int window_left, fa_stream_t stream) {
    bool empty = false;
    int st = validate(q, k, v, o, lse, B, H, N_q, N_k, d, scale, key_lens, &empty);
    if (st != FA_OK) return st;
    if (window_left < 0) return FA_ERR_INVALID_ARG;
    if (empty) return FA_OK;
    int dev = -1;
    int ndev = 0;
    if (cudaGetDeviceCount(&ndev) != cudaSuccess || ndev == 0) {
        cudaGetLastError();
        return FA_ERR_NO_DEVICE;
    }
    const cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail("cudaGetDevice", e);
    st = prepare_device(dev);
    if (st != FA_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const SplitParts none{0, nullptr, nullptr, nullptr};
    if (d == 64) return launch<64>(q, k, v, o, lse, B, H, N_q, N_k, scale, causal, key_lens, s, none, window_left);
    return launch<128>(q, k, v, o, lse, B, H, N_q, N_k, scale, causal, key_lens, s, none, window_left);
}

int fa_fwd_fp8(const void* q8, const void* k8, const void* v8, void* o, float* lse, int B, int H, int N_q, int N_k,
               int d, float scale, float q_descale, float k_descale, float v_descale, int causal,
               const int32_t* key_lens, fa_stream_t stream) {
    bool empty = false;
    int st = validate(q8, k8, v8, o, lse, B, H, N_q, N_k, d, scale, key_lens, &empty);
    if (st != FA_OK) return st;
    for (const float x : {q_descale, k_descale, v_descale})
        if (!std::isfinite(x) || !(x > 0.f)) return FA_ERR_INVALID_ARG;
    // the scores' three factors, folded into the one scale the kernel applies
    const float c = scale * q_descale * k_descale;
    if (!(c * 1.4426950408889634f > 0.f) || !std::isfinite(c * 1.4426950408889634f)) return FA_ERR_INVALID_ARG;
    if (empty) return FA_OK;
    int dev = -1;
    int ndev = 0;
    if (cudaGetDeviceCount(&ndev) != cudaSuccess || ndev == 0) {
        cudaGetLastError();
        return FA_ERR_NO_DEVICE;
    }
    const cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail("cudaGetDevice", e);
    st = prepare_device(dev);
    if (st != FA_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const SplitParts none{0, nullptr, nullptr, nullptr};
    const BiasArgs nob{fa::kBiasNone, nullptr, 0};
    if (d == 64) return launch<64, true>(q8, k8, v8, o, lse, B, H, N_q, N_k, c, causal, key_lens, s, none, -1, nob,
                                         v_descale);
    return launch<128, true>(q8, k8, v8, o, lse, B, H, N_q, N_k, c, causal, key_lens, s, none, -1, nob, v_descale);
}

size_t fa_bwd_workspace_size(int B, int H, int N_q, int d) {
    if (B < 0 || H < 0 || N_q < 0 || (d != 64 && d != 128)) return 0;
    return bwd_layout(B, H, N_q, d).total;
}

// fa_bwd's argument checks and launch; wait_limit bounds every pipeline wait of the
// main kernel (the default outside the self test).
static int bwd_entry(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout,
                     void* dq, void* dk, void* dv, int B, int H, int N_q, int N_k, int d, float scale, int causal,
                     const int32_t* key_lens, void* workspace, size_t workspace_bytes, fa_stream_t stream,
                     unsigned long long wait_limit) {
    bool empty = false;
    int st = validate(q, k, v, o, lse, B, H, N_q, N_k, d, scale, key_lens, &empty);
    if (st != FA_OK) return st;
    if (B == 0 || H == 0) return FA_OK;
    // with N_q = 0 only dK = dV = 0 are written; validate() stopped before the pointers
    if (N_k > 0 && (k == nullptr || v == nullptr || dk == nullptr || dv == nullptr)) return FA_ERR_INVALID_ARG;
    if (N_q > 0 && (q == nullptr || o == nullptr || lse == nullptr || dout == nullptr || dq == nullptr))
        return FA_ERR_INVALID_ARG;
    if (!aligned(dout, 16) || !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16)) return FA_ERR_MISALIGNED;
    if (N_k > 0 && (!aligned(k, 16) || !aligned(v, 16))) return FA_ERR_MISALIGNED;
    if (key_lens != nullptr && !aligned(key_lens, 4)) return FA_ERR_MISALIGNED;
    const BwdLayout L = bwd_layout(B, H, N_q, d);
    if (workspace == nullptr || workspace_bytes < L.total) return FA_ERR_INVALID_ARG;
    if (!aligned(workspace, 256)) return FA_ERR_MISALIGNED;
    int dev = -1;
    int ndev = 0;
    if (cudaGetDeviceCount(&ndev) != cudaSuccess || ndev == 0) {
        cudaGetLastError();
        return FA_ERR_NO_DEVICE;
    }
    const cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail("cudaGetDevice", e);
    st = prepare_device(dev);
    if (st != FA_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    if (d == 64)
        return launch_bwd<64>(q, k, v, o, lse, dout, dq, dk, dv, B, H, N_q, N_k, scale, causal, key_lens, ws, s,
                              wait_limit);
    return launch_bwd<128>(q, k, v, o, lse, dout, dq, dk, dv, B, H, N_q, N_k, scale, causal, key_lens, ws, s,
                           wait_limit);
}

int fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout, void* dq,
           void* dk, void* dv, int B, int H, int N_q, int N_k, int d, float scale, int causal,
           const int32_t* key_lens, void* workspace, size_t workspace_bytes, fa_stream_t stream) {
    return bwd_entry(q, k, v, o, lse, dout, dq, dk, dv, B, H, N_q, N_k, d, scale, causal, key_lens, workspace,
                     workspace_bytes, stream, kWaitLimitCycles);
}

int fa_fwd_bias(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N_q, int N_k,
                int d, float scale, int causal, const int32_t* key_lens, const float* slopes, int window_left,
                fa_stream_t stream) {
    bool empty = false;
    int st = validate(q, k, v, o, lse, B, H, N_q, N_k, d, scale, key_lens, &empty);
    if (st != FA_OK) return st;
    if (empty) return FA_OK;
    if (slopes == nullptr) return FA_ERR_INVALID_ARG;
    if (!aligned(slopes, 4)) return FA_ERR_MISALIGNED;
    int dev = -1;
    int ndev = 0;
    if (cudaGetDeviceCount(&ndev) != cudaSuccess || ndev == 0) {
        cudaGetLastError();
        return FA_ERR_NO_DEVICE;
    }
    const cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail("cudaGetDevice", e);
    st = prepare_device(dev);
    if (st != FA_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const SplitParts none{0, nullptr, nullptr, nullptr};
    const int wl = window_left < 0 ? -1 : window_left;
    const BiasArgs bias{fa::kBiasSlopes, slopes, 0};
    if (d == 64) return launch<64>(q, k, v, o, lse, B, H, N_q, N_k, scale, causal, key_lens, s, none, wl, bias);
    return launch<128>(q, k, v, o, lse, B, H, N_q, N_k, scale, causal, key_lens, s, none, wl, bias);
}

int fa_fwd_bias_table(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N_q,
                      int N_k, int d, float scale, int causal, const int32_t* key_lens, const float* table,
                      int radius, int window_left, fa_stream_t stream) {
    bool empty = false;
    int st = validate(q, k, v, o, lse, B, H, N_q, N_k, d, scale, key_lens, &empty);
    if (st != FA_OK) return st;
    if (radius < 0 || radius > kMaxBiasRadius) return FA_ERR_INVALID_ARG;
    if (empty) return FA_OK;
    if (table == nullptr) return FA_ERR_INVALID_ARG;
    if (!aligned(table, 4)) return FA_ERR_MISALIGNED;
    int dev = -1;
    int ndev = 0;
    if (cudaGetDeviceCount(&ndev) != cudaSuccess || ndev == 0) {
        cudaGetLastError();
        return FA_ERR_NO_DEVICE;
    }
    const cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail("cudaGetDevice", e);
    st = prepare_device(dev);
    if (st != FA_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const SplitParts none{0, nullptr, nullptr, nullptr};
    const int wl = window_left < 0 ? -1 : window_left;
    const BiasArgs bias{fa::kBiasTable, table, radius};
    if (d == 64) return launch<64>(q, k, v, o, lse, B, H, N_q, N_k, scale, causal, key_lens, s, none, wl, bias);
    return launch<128>(q, k, v, o, lse, B, H, N_q, N_k, scale, causal, key_lens, s, none, wl, bias);
}

int fa_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse, const int32_t* cu_seqlens_q,
                  const int32_t* cu_seqlens_k, int B, int H, int total_q, int total_k, int max_seqlen_q, int d,
                  float scale, int causal, fa_stream_t stream) {
    if (B < 0 || H < 0 || total_q < 0 || total_k < 0 || max_seqlen_q < 0) return FA_ERR_INVALID_ARG;
    if (!std::isfinite(scale) || !(scale > 0.f)) return FA_ERR_INVALID_ARG;
    if (!(scale * 1.4426950408889634f > 0.f) || !std::isfinite(scale * 1.4426950408889634f))
        return FA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
    if (B == 0 || H == 0 || total_q == 0 || max_seqlen_q == 0) return FA_OK;
    if (B > 65535 || H > 65535) return FA_ERR_UNSUPPORTED;
    if ((unsigned long long)total_q * H * d * 2 >= (1ull << 40) || (unsigned long long)total_k * H * d * 2 >= (1ull << 40))
        return FA_ERR_UNSUPPORTED;
    if (q == nullptr || o == nullptr || lse == nullptr || cu_seqlens_q == nullptr || cu_seqlens_k == nullptr)
        return FA_ERR_INVALID_ARG;
    if (total_k > 0 && (k == nullptr || v == nullptr)) return FA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(o, 16) || !aligned(lse, 4) || !aligned(cu_seqlens_q, 4) ||
        !aligned(cu_seqlens_k, 4))
        return FA_ERR_MISALIGNED;
    if (total_k > 0 && (!aligned(k, 16) || !aligned(v, 16))) return FA_ERR_MISALIGNED;
    int dev = -1;
    int ndev = 0;
    if (cudaGetDeviceCount(&ndev) != cudaSuccess || ndev == 0) {
        cudaGetLastError();
        return FA_ERR_NO_DEVICE;
    }
    const cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail("cudaGetDevice", e);
    int st = prepare_device(dev);
    if (st != FA_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (d == 64)
        return launch_varlen<64>(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, B, H, total_q, total_k, max_seqlen_q,
                                 scale, causal, s);
    return launch_varlen<128>(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, B, H, total_q, total_k, max_seqlen_q,
                              scale, causal, s);
}

size_t fa_fwd_host_workspace_size(int B, int H, int N_q, int N_k, int d, int has_key_lens) {
    if (B < 0 || H < 0 || N_q < 0 || N_k < 0 || (d != 64 && d != 128)) return 0;
    return host_layout(B, H, N_q, N_k, d, has_key_lens).total;
}

// Copy streams and events of fa_fwd_host, per device, created on first use.
// Calls on one device are serialised (they are synchronous anyway).
struct HostPipe {
    std::once_flag once;
    std::mutex mu;
    cudaError_t status = cudaSuccess;
    cudaStream_t h2d = nullptr, d2h = nullptr;
    cudaEvent_t start = nullptr, last_out = nullptr;
    cudaEvent_t in_done[kHostChunksMax] = {};
    cudaEvent_t fwd_done[kHostChunksMax] = {};
};
HostPipe g_host_pipe[kMaxDevices];

HostPipe* host_pipe(int dev) {
    HostPipe& hp = g_host_pipe[dev];
    std::call_once(hp.once, [&] {
        cudaError_t e = cudaStreamCreateWithFlags(&hp.h2d, cudaStreamNonBlocking);
        if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&hp.d2h, cudaStreamNonBlocking);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&hp.start, cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&hp.last_out, cudaEventDisableTiming);
        for (int i = 0; i < kHostChunksMax && e == cudaSuccess; ++i) {
            e = cudaEventCreateWithFlags(&hp.in_done[i], cudaEventDisableTiming);
            if (e == cudaSuccess) e = cudaEventCreateWithFlags(&hp.fwd_done[i], cudaEventDisableTiming);
        }
        hp.status = e;
    });
    return &hp;
}

int fa_fwd_host(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N_q, int N_k,
                int d, float scale, int causal, const int32_t* key_lens, void* workspace, size_t workspace_bytes,
                fa_stream_t stream) {
    bool empty = false;
    int st = validate(q, k, v, o, lse, B, H, N_q, N_k, d, scale, key_lens, &empty);
    if (st != FA_OK || empty) return st;
    const HostLayout L = host_layout(B, H, N_q, N_k, d, key_lens != nullptr);
    if (workspace == nullptr || workspace_bytes < L.total) return FA_ERR_INVALID_ARG;
    if (!aligned(workspace, 256)) return FA_ERR_MISALIGNED;
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail("cudaGetDevice", e);
    if (dev < 0 || dev >= kMaxDevices) return FA_ERR_UNSUPPORTED;
    HostPipe* hp = host_pipe(dev);
    if (hp->status != cudaSuccess) return cuda_fail("copy streams for fa_fwd_host", hp->status);
    std::lock_guard<std::mutex> lock(hp->mu);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    char* ws = static_cast<char*>(workspace);
    const size_t q_head = (size_t)N_q * d * 2, kv_head = (size_t)N_k * d * 2;
    // Chunks of about 1/kHostChunksTarget of the (b, h) pairs: runs of heads inside
    // one batch entry, or of whole batch entries when a batch entry is smaller than
    // that.  The copies of chunk c+1 and the read-back of chunk c-1 overlap the
    // forward of chunk c (H2D and D2H on their own streams and copy engines), so the
    // call costs about the longer of the two transfers instead of their sum.
    const long long total = (long long)B * H;
    const long long want = (total + kHostChunksTarget - 1) / kHostChunksTarget;   // pairs per chunk
    const bool by_heads = want <= H;
    const int per = by_heads ? (int)std::max(1LL, want) : H;                      // heads per chunk
    const int bc = by_heads ? 1 : (int)((want + H - 1) / H);                      // batch entries per chunk
    // Chunks as (first batch entry, batch entries, first head, heads).  What is left
    // after the last host-to-device copy -- the last chunk's forward and read-back --
    // is not overlapped, so with chunks of heads the last chunk is cut into halves
    // (per/2, per/4, .., 1, 1 heads): the tail is about one head's work.
    struct Chunk { int b, nb, h0, hc; };
    Chunk chunks[kHostChunksMax];
    int n_chunks = 0;
    if (by_heads) {
        for (int b = 0; b < B; ++b)
            for (int h0 = 0; h0 < H; h0 += per) {
                const int hc = std::min(per, H - h0);
                if (b == B - 1 && h0 + hc == H) {
                    int left = hc, at = h0;
                    while (left > 1 && n_chunks < kHostChunksMax) {
                        const int half = left / 2;
                        chunks[n_chunks++] = {b, 1, at, left - half};
                        at += left - half;
                        left = half;
                    }
                    if (left > 0) {
                        if (n_chunks >= kHostChunksMax) return FA_ERR_UNSUPPORTED;
                        chunks[n_chunks++] = {b, 1, at, left};
                    }
                } else {
                    if (n_chunks >= kHostChunksMax) return FA_ERR_UNSUPPORTED;
                    chunks[n_chunks++] = {b, 1, h0, hc};
                }
            }
    } else {
        for (int b = 0; b < B; b += bc) {
            if (n_chunks >= kHostChunksMax) return FA_ERR_UNSUPPORTED;
            chunks[n_chunks++] = {b, std::min(bc, B - b), 0, H};
        }
    }
    // the workspace may still be in use by earlier work on `stream`
    e = cudaEventRecord(hp->start, s);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(hp->h2d, hp->start, 0);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(hp->d2h, hp->start, 0);
    const int32_t* kl_dev = nullptr;
    if (e == cudaSuccess && key_lens != nullptr) {
        e = cudaMemcpyAsync(ws + L.kl, key_lens, (size_t)B * 4, cudaMemcpyHostToDevice, hp->h2d);
        kl_dev = reinterpret_cast<const int32_t*>(ws + L.kl);
    }
    if (e != cudaSuccess) return cuda_fail("fa_fwd_host setup", e);
    for (int c = 0; c < n_chunks; ++c) {
        const int b = chunks[c].b, nb = chunks[c].nb;           // batch entries of the chunk
        const int h0 = chunks[c].h0, hc = chunks[c].hc;         // heads per batch entry
        const size_t row0 = (size_t)b * H + h0;                 // first (b, h) pair of the chunk
        const size_t rows = (size_t)nb * hc;                    // (b, h) pairs of the chunk
        e = cudaMemcpyAsync(ws + L.q + row0 * q_head, static_cast<const char*>(q) + row0 * q_head, rows * q_head,
                            cudaMemcpyHostToDevice, hp->h2d);
        if (e == cudaSuccess && kv_head > 0)
            e = cudaMemcpyAsync(ws + L.k + row0 * kv_head, static_cast<const char*>(k) + row0 * kv_head,
                                rows * kv_head, cudaMemcpyHostToDevice, hp->h2d);
        if (e == cudaSuccess && kv_head > 0)
            e = cudaMemcpyAsync(ws + L.v + row0 * kv_head, static_cast<const char*>(v) + row0 * kv_head,
                                rows * kv_head, cudaMemcpyHostToDevice, hp->h2d);
        if (e == cudaSuccess) e = cudaEventRecord(hp->in_done[c], hp->h2d);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(s, hp->in_done[c], 0);
        if (e != cudaSuccess) return cuda_fail("cudaMemcpyAsync (host to device)", e);
        // the chunk as a problem of its own: nb batch entries of hc heads
        st = fa_fwd(ws + L.q + row0 * q_head, N_k > 0 ? ws + L.k + row0 * kv_head : nullptr,
                    N_k > 0 ? ws + L.v + row0 * kv_head : nullptr, ws + L.o + row0 * q_head,
                    reinterpret_cast<float*>(ws + L.lse) + row0 * N_q, nb, hc, N_q, N_k, d, scale, causal,
                    kl_dev != nullptr ? kl_dev + b : nullptr, stream);
        if (st != FA_OK) return st;
        e = cudaEventRecord(hp->fwd_done[c], s);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(hp->d2h, hp->fwd_done[c], 0);
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(static_cast<char*>(o) + row0 * q_head, ws + L.o + row0 * q_head, rows * q_head,
                                cudaMemcpyDeviceToHost, hp->d2h);
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(lse + row0 * N_q, ws + L.lse + row0 * N_q * 4, rows * N_q * 4,
                                cudaMemcpyDeviceToHost, hp->d2h);
        if (e != cudaSuccess) return cuda_fail("cudaMemcpyAsync (device to host)", e);
    }
    // `stream` is complete only after the last read-back
    e = cudaEventRecord(hp->last_out, hp->d2h);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s, hp->last_out, 0);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    return e == cudaSuccess ? FA_OK : cuda_fail("cudaStreamSynchronize", e);
}

const char* fa_status_string(int status) {
    switch (status) {
        case FA_OK: return "FA_OK";
        case FA_ERR_INVALID_ARG: return "FA_ERR_INVALID_ARG: invalid argument";
        case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED: unsupported configuration or device";
        case FA_ERR_MISALIGNED: return "FA_ERR_MISALIGNED: pointer misaligned";
        case FA_ERR_CUDA: return "FA_ERR_CUDA: CUDA call failed";
        case FA_ERR_NO_DEVICE: return "FA_ERR_NO_DEVICE: no CUDA device";
        case FA_ERR_DEVICE_TIMEOUT: return "FA_ERR_DEVICE_TIMEOUT: kernel pipeline wait timed out";
        default: return "unknown status";
    }
}

int fa_get_device_status(fa_stream_t stream) {
    int ndev = 0;
    if (cudaGetDeviceCount(&ndev) != cudaSuccess || ndev == 0) {
        cudaGetLastError();
        return FA_ERR_NO_DEVICE;
    }
    cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail("cudaStreamSynchronize", e);
    int v = 0;
    e = cudaMemcpyFromSymbol(&v, fa::g_fa_status, sizeof(int));
    if (e != cudaSuccess) return cuda_fail("cudaMemcpyFromSymbol(status)", e);
    const int zero = 0;
    e = cudaMemcpyToSymbol(fa::g_fa_status, &zero, sizeof(int));
    if (e != cudaSuccess) return cuda_fail("cudaMemcpyToSymbol(status)", e);
    return v == 0 ? FA_OK : v;
}

int fa_selftest_wait_timeout(unsigned long long limit_cycles, fa_stream_t stream) {
    int ndev = 0;
    if (cudaGetDeviceCount(&ndev) != cudaSuccess || ndev == 0) {
        cudaGetLastError();
        return FA_ERR_NO_DEVICE;
    }
    if (limit_cycles > (1ull << 32)) return FA_ERR_INVALID_ARG;
    selftest_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(limit_cycles);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail("self-test kernel launch", e);
    return fa_get_device_status(stream);
}

int fa_selftest_fwd_timeout(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N_q,
                            int N_k, int d, float scale, int causal, unsigned long long limit_cycles,
                            fa_stream_t stream) {
    bool empty = false;
    int st = validate(q, k, v, o, lse, B, H, N_q, N_k, d, scale, nullptr, &empty);
    if (st != FA_OK) return st;
    if (limit_cycles < 1 || limit_cycles > (1ull << 32)) return FA_ERR_INVALID_ARG;
    if (empty || N_k == 0) return FA_ERR_INVALID_ARG;   // nothing would wait
    int ndev = 0, dev = -1;
    if (cudaGetDeviceCount(&ndev) != cudaSuccess || ndev == 0) {
        cudaGetLastError();
        return FA_ERR_NO_DEVICE;
    }
    const cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail("cudaGetDevice", e);
    st = prepare_device(dev);
    if (st != FA_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const SplitParts none{0, nullptr, nullptr, nullptr};
    const BiasArgs nob{fa::kBiasNone, nullptr, 0};
    st = (d == 64) ? launch<64>(q, k, v, o, lse, B, H, N_q, N_k, scale, causal, nullptr, s, none, -1, nob, 1.f,
                                limit_cycles)
                   : launch<128>(q, k, v, o, lse, B, H, N_q, N_k, scale, causal, nullptr, s, none, -1, nob, 1.f,
                                 limit_cycles);
    if (st != FA_OK) return st;
    return fa_get_device_status(stream);
}

int fa_selftest_bwd_timeout(const void* q, const void* k, const void* v, const void* o, const float* lse,
                            const void* dout, void* dq, void* dk, void* dv, int B, int H, int N_q, int N_k, int d,
                            float scale, int causal, void* workspace, size_t workspace_bytes,
                            unsigned long long limit_cycles, fa_stream_t stream) {
    if (limit_cycles < 1 || limit_cycles > (1ull << 32)) return FA_ERR_INVALID_ARG;
    if (B <= 0 || H <= 0 || N_q <= 0 || N_k <= 0) return FA_ERR_INVALID_ARG;   // nothing would wait
    const int st = bwd_entry(q, k, v, o, lse, dout, dq, dk, dv, B, H, N_q, N_k, d, scale, causal, nullptr,
                             workspace, workspace_bytes, stream, limit_cycles);
    if (st != FA_OK) return st;
    return fa_get_device_status(stream);
}

const char* fa_last_error(void) { return t_last_error; }

int fa_version(void) { return kVersion; }

}  // extern "C"
