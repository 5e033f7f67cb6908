/*
 * fa.h -- C ABI of libfa_b200.so: exact attention forward on NVIDIA B200 (sm_100a).
 *
 * Operation (all entry points compute the same thing):
 *
 *     S   = scale * Q K^T                       (per batch b, head h)
 *     S_ij = -inf where key j is masked for query i
 *     O   = softmax_rowwise(S) V
 *     LSE_i = ln sum_j exp(S_ij)                (natural log, scale included)
 *
 * This is the computation described in "FlashAttention 与边缘设备上的注意力
 * 内存瓶颈" (section 2: standard attention forms S and P; sections 3.1-3.2:
 * the tiled, online-softmax method is exact) and "FlashAttention：把注意力从
 * 公式写成数据流" (opening paragraph: S = QK^T, softmax, times V; section
 * "分块与在线 softmax": per Q tile, stream K/V tiles keeping the running max,
 * exp-sum and output accumulator, never storing S).  The library computes it
 * that way on the GPU: S and P never reach global memory.
 *
 * Masking (section "精度、掩码和边界情况" of the second page: masked positions
 * must stay out of the normaliser; tail blocks must be handled).  The pages
 * leave the details open; this library fixes them as:
 *   - key_lens: if non-NULL, key_lens[b] is clamped to [0, N_k] and keys
 *     j >= key_lens[b] are masked for every query of sequence b;
 *   - causal: bottom-right aligned, key j is visible to query i iff
 *     j <= i + (N_k - N_q) (the usual j <= i when N_q == N_k);
 *   - both masks combine (AND);
 *   - a query row with no visible key gets O = +0.0 and LSE = -inf.
 *
 * Layout: Q is [B, H, N_q, d], K and V are [B, H, N_k, d], O is
 * [B, H, N_q, d], all bf16, dense, row-major (d fastest).  LSE is fp32
 * [B, H, N_q].  key_lens is int32 [B].  Supported head dims: d = 64, 128.
 *
 * Status codes: every entry point returns an int, FA_OK (0) or one of the
 * negative FA_ERR_* values below.  Argument errors are detected on the host
 * before any CUDA call is made.
 */
#ifndef FA_B200_H
#define FA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define FA_API __attribute__((visibility("default")))
#else
#define FA_API
#endif

/* Same type as cudaStream_t; NULL means the legacy default stream. */
struct CUstream_st;
typedef struct CUstream_st *fa_stream_t;

enum {
    FA_OK = 0,
    FA_ERR_INVALID_ARG = -1,     /* bad size, NULL pointer, scale not finite and > 0 */
    FA_ERR_UNSUPPORTED = -2,     /* head dim not 64/128, sizes beyond the launch limits, or not an sm_100 device */
    FA_ERR_MISALIGNED = -3,      /* q/k/v/o not 16-byte aligned, lse/key_lens not 4-byte aligned */
    FA_ERR_CUDA = -4,            /* a CUDA runtime/driver call failed (launch, copy, tensor-map encode) */
    FA_ERR_NO_DEVICE = -5,       /* no CUDA device is visible */
    FA_ERR_DEVICE_TIMEOUT = -6   /* a kernel gave up on a pipeline wait (see fa_get_device_status) */
};

/*
 * fa_fwd -- attention forward on device buffers, asynchronous on `stream`.
 *
 *   q, k, v   device pointers, bf16, layout above, 16-byte aligned.  k and v
 *             may be NULL when N_k == 0.
 *   o         device pointer, bf16 [B,H,N_q,d], 16-byte aligned, written in full.
 *             Must not overlap q, k, v or lse.
 *   lse       device pointer, fp32 [B,H,N_q], 4-byte aligned, written in full.
 *   B, H      batch and heads, >= 0; B <= 65535, H <= 65535.
 *   N_q, N_k  query and key lengths, >= 0 (any value, no multiple required).
 *   d         head dim, 64 or 128.
 *   scale     finite and > 0 (usually 1/sqrt(d)), applied to QK^T before the
 *             softmax; scale*log2(e) must not underflow to 0 in fp32.
 *   causal    0 or non-zero (bottom-right aligned, see above).
 *   key_lens  NULL, or device int32 [B] (values outside [0,N_k] are clamped).
 *   stream    CUDA stream to launch on.
 *
 * Ownership: the caller owns every buffer; the library allocates nothing and
 * keeps no per-call state (only a per-device cache of kernel attributes and
 * the driver's tensor-map encoder).  Thread-safe.
 * Returns FA_OK once the kernel is enqueued (B*H*N_q == 0 is a no-op that
 * returns FA_OK without touching any pointer).  Errors in device execution
 * surface at the caller's next synchronisation, or via fa_get_device_status.
 * NaN/Inf in unmasked inputs propagate to the outputs.
 */
FA_API int fa_fwd(const void *q, const void *k, const void *v, void *o, float *lse,
           int B, int H, int N_q, int N_k, int d, float scale, int causal,
           const int32_t *key_lens, fa_stream_t stream);

/*
 * fa_fwd_host_workspace_size -- bytes of device workspace fa_fwd_host needs
 * for this problem (room for Q, K, V, O, LSE and key_lens on the device,
 * each 256-byte aligned).  Returns 0 for invalid sizes.
 */
FA_API size_t fa_fwd_host_workspace_size(int B, int H, int N_q, int N_k, int d,
                                  int has_key_lens);

/*
 * fa_fwd_host -- the same forward for HOST-resident inputs and outputs.
 *
 *   q, k, v, o, lse, key_lens   host pointers, same layouts as fa_fwd (pinned
 *                               memory gives asynchronous, full-speed copies).
 *   workspace                   device buffer of at least
 *                               fa_fwd_host_workspace_size(...) bytes, 256-byte
 *                               aligned, owned by the caller.
 *
 * Copies the inputs to the workspace, runs fa_fwd on `stream`, copies O and
 * LSE back, and synchronises `stream` before returning, so on FA_OK the host
 * outputs are complete.  Returns FA_ERR_INVALID_ARG if the workspace is too
 * small, FA_ERR_CUDA if a copy fails, plus every fa_fwd error.
 */
FA_API int fa_fwd_host(const void *q, const void *k, const void *v, void *o, float *lse,
                int B, int H, int N_q, int N_k, int d, float scale, int causal,
                const int32_t *key_lens, void *workspace, size_t workspace_bytes,
                fa_stream_t stream);

/* Human-readable name of a status code (static string, never NULL). */
FA_API const char *fa_status_string(int status);

/*
 * fa_get_device_status -- synchronise `stream`, then report and clear the
 * current device's error word.  Every pipeline wait inside the kernels is
 * bounded; a wait that runs out records FA_ERR_DEVICE_TIMEOUT there and the
 * kernel returns early instead of hanging.  Returns FA_OK,
 * FA_ERR_DEVICE_TIMEOUT, or FA_ERR_CUDA if the synchronisation itself failed.
 */
FA_API int fa_get_device_status(fa_stream_t stream);

/*
 * fa_selftest_wait_timeout -- failure-detection self test.  Launches a tiny
 * kernel that waits on an mbarrier nothing ever arrives on, with the same
 * bounded-wait routine the attention kernel uses and a limit of
 * `limit_cycles` SM clock cycles (at most 2^32), then returns what
 * fa_get_device_status reports: FA_ERR_DEVICE_TIMEOUT when the bound works.
 * The CUDA context stays usable afterwards.
 */
FA_API int fa_selftest_wait_timeout(unsigned long long limit_cycles, fa_stream_t stream);

/*
 * fa_last_error -- the CUDA call and error text behind the most recent
 * FA_ERR_CUDA returned on the calling thread ("" if none).  The string
 * belongs to the library and stays valid until the thread's next failing call.
 */
FA_API const char *fa_last_error(void);

/* Library version, major*10000 + minor*100 + patch. */
FA_API int fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_B200_H */
