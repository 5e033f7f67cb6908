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
 * fa_fwd_window -- fa_fwd with a sliding (local) window on top of the causal
 * and key_lens masks: key j is also masked for query i when
 * j < i + (N_k - N_q) - window_left, so a row sees at most the window_left
 * keys before its diagonal position plus that position (with causal), and
 * never keys before the window (without causal, the window bounds keys from
 * below only).  This is the local-attention mask among the mask variants that
 * "FlashAttention：把注意力从公式写成数据流" (section "精度、掩码和边界情况")
 * groups with causal and padding masks.  Tiles wholly before a query block's
 * window are never loaded; partially covered tiles are masked per element.
 *
 *   window_left   >= 0 (window_left >= N_k gives the same result as fa_fwd).
 *   other arguments, ownership and errors as fa_fwd; FA_ERR_INVALID_ARG for a
 *   negative window_left.
 */
FA_API int fa_fwd_window(const void *q, const void *k, const void *v, void *o, float *lse,
                  int B, int H, int N_q, int N_k, int d, float scale, int causal,
                  const int32_t *key_lens, int window_left, fa_stream_t stream);

/*
 * fa_fwd_bias -- fa_fwd with an additive positional bias (and, optionally, the
 * sliding window of fa_fwd_window): before the softmax every visible score
 * gets -slopes[h] * |i + (N_k - N_q) - j|, a linear penalty on the distance
 * from the row's diagonal position (the "additive positional bias" mask
 * variant of "FlashAttention：把注意力从公式写成数据流", section
 * "精度、掩码和边界情况"; with the usual per-head slopes this is the ALiBi
 * bias).  The LSE includes the bias.
 *
 *   slopes        device fp32 [H], 4-byte aligned, non-NULL (finite; >= 0 for
 *                 the usual decaying bias, any sign is computed as given).
 *   window_left   < 0: no window; >= 0: as fa_fwd_window.
 *   other arguments, ownership and errors as fa_fwd; FA_ERR_INVALID_ARG for
 *   NULL slopes, FA_ERR_MISALIGNED for unaligned slopes.
 */
FA_API int fa_fwd_bias(const void *q, const void *k, const void *v, void *o, float *lse,
                int B, int H, int N_q, int N_k, int d, float scale, int causal,
                const int32_t *key_lens, const float *slopes, int window_left,
                fa_stream_t stream);

/*
 * fa_fwd_bias_table -- fa_fwd with a custom positional bias: any per-head
 * function of the key's position relative to the query, given as a table.
 * Key j of query i gets, added to its scaled score,
 *     table[h * (2R+1) + clamp(j - (i + N_k - N_q), -R, R) + R]
 * (R = radius; relative positions beyond +-R use the table's end values), so
 *   S_ij = scale * q_i . k_j + bias,  O and LSE as fa_fwd (the LSE includes
 * the bias).  This is the general "custom positional bias" among the mask
 * variants of "FlashAttention：把注意力从公式写成数据流", section
 * "精度、掩码和边界情况"; a learned relative-position bias, or any distance
 * penalty, is one table.
 *
 *   table         device fp32 [H, 2*radius+1], 4-byte aligned, non-NULL,
 *                 natural-log units (the same units as scale * q . k); finite
 *                 values (NaN/Inf propagate like NaN/Inf inputs).  Read only.
 *   radius        R, 0 .. 2^30.
 *   window_left   < 0: no window; >= 0: as fa_fwd_window.
 *   other arguments, ownership and errors as fa_fwd; FA_ERR_INVALID_ARG for a
 *   NULL table or a radius out of range, FA_ERR_MISALIGNED for an unaligned
 *   table.
 */
FA_API int fa_fwd_bias_table(const void *q, const void *k, const void *v, void *o, float *lse,
                             int B, int H, int N_q, int N_k, int d, float scale, int causal,
                             const int32_t *key_lens, const float *table, int radius,
                             int window_left, fa_stream_t stream);

/*
 * fa_fwd_fp8 -- fa_fwd on 8-bit E4M3 inputs with per-tensor scales: computes
 * the attention of the dequantised tensors Q = q_descale * Q8,
 * K = k_descale * K8, V = v_descale * V8, i.e.
 *   O = softmax(scale * Q K^T + mask) V,  LSE as fa_fwd,
 * with E4M3 tensor-core products (the low-precision arithmetic the Hopper
 * kernel brings in, "FlashAttention：把注意力从公式写成数据流", section
 * "FA2 与 FA3"; FP8 saves HBM bytes but needs scaling and an error report
 * against a 16-bit baseline, same page, section "用实验验证而不是背诵结论").
 * The probabilities are rounded to E4M3 before the PV product and O is
 * normalised by the sum of those rounded values, so O's error is set by P's
 * 3-bit mantissa; the LSE uses the unrounded sum.
 *
 *   q8, k8, v8  device uint8 E4M3 codes (OCP 8-bit float, no infinities,
 *               0x7F/0xFF NaN), [B,H,N_q|N_k|N_k,d] contiguous, 16-byte aligned.
 *   o           device bf16 [B,H,N_q,d], 16-byte aligned.
 *   lse         device fp32 [B,H,N_q], 4-byte aligned.
 *   d           64 or 128 (FA_ERR_UNSUPPORTED otherwise).
 *   q_descale, k_descale, v_descale   finite, > 0 (FA_ERR_INVALID_ARG
 *               otherwise).  The kernel applies the product
 *               scale * q_descale * k_descale as one fp32 number (two fp32
 *               roundings, a relative change of at most 2^-23 in every score);
 *               it must stay finite and > 0.
 *   other arguments, ownership, empty cases and errors as fa_fwd.
 */
FA_API int fa_fwd_fp8(const void *q8, const void *k8, const void *v8, void *o, float *lse,
               int B, int H, int N_q, int N_k, int d, float scale, float q_descale,
               float k_descale, float v_descale, int causal, const int32_t *key_lens,
               fa_stream_t stream);

/*
 * fa_bwd -- backward pass of fa_fwd: given the upstream gradient dO of O, the
 * gradients of O = softmax(scale * Q K^T + mask) V with respect to Q, K and V.
 * The attention matrix is recomputed tile by tile from Q, K and the forward's
 * LSE and never stored (the backward and its recomputation are named by
 * "FlashAttention：把注意力从公式写成数据流", section "用实验验证而不是背诵结论",
 * and "[2205.14135] FlashAttention: Fast and Memory-Efficient Exact Attention with
 * IO-Awareness", section "三、FLOPs（計算能力）並非 Speedup 的主因素"):
 *   P = exp(scale * Q K^T - LSE) on visible pairs, 0 elsewhere;
 *   dV = P^T dO;  dS = P * (dO V^T - D), D_i = dO_i . O_i;
 *   dQ = scale * dS K;  dK = scale * dS^T Q.
 *
 *   q, k, v       device bf16 [B,H,N_q|N_k|N_k,d], as given to fa_fwd.
 *   o, lse        device: the outputs fa_fwd returned for these inputs (bf16
 *                 [B,H,N_q,d], fp32 [B,H,N_q]).
 *   dout          device bf16 [B,H,N_q,d], 16-byte aligned: dL/dO.
 *   dq            device bf16 [B,H,N_q,d]; dk, dv device bf16 [B,H,N_k,d];
 *                 16-byte aligned, written in full (rows of keys no query sees,
 *                 and rows of queries that see no key, get 0).
 *   B,H,N_q,N_k,d,scale,causal,key_lens   as for fa_fwd (same mask).
 *   workspace     device, 256-byte aligned, at least fa_bwd_workspace_size(B,H,N_q,d)
 *                 bytes, owned by the caller; overwritten (D and an fp32 dQ
 *                 accumulator). Calls sharing a workspace must be ordered.
 *   stream        as for fa_fwd; three kernels are enqueued (D and zeroing, the
 *                 main kernel, dQ to bf16; with N_q = 0 two memsets instead).
 *
 * Returns FA_OK once enqueued.  Errors as fa_fwd, plus FA_ERR_INVALID_ARG for a
 * NULL or short workspace or NULL gradient buffers, FA_ERR_MISALIGNED for
 * unaligned dout/dq/dk/dv/workspace.  B = 0 or H = 0: no-op.  N_q = 0: dk = dv = 0.
 * N_k = 0: dq = 0.  The dQ sums across key blocks are tensor reduce-adds (atomic
 * at L2, in arrival order), so dq may differ in the last bits between runs; dk
 * and dv are deterministic.
 */
FA_API size_t fa_bwd_workspace_size(int B, int H, int N_q, int d);
FA_API int fa_bwd(const void *q, const void *k, const void *v, const void *o, const float *lse,
           const void *dout, void *dq, void *dk, void *dv, int B, int H, int N_q, int N_k,
           int d, float scale, int causal, const int32_t *key_lens, void *workspace,
           size_t workspace_bytes, fa_stream_t stream);

/*
 * fa_fwd_varlen -- attention over a batch of sequences of different lengths
 * packed back to back without padding (the packed variable-length batches of
 * the mask variants, "FlashAttention：把注意力从公式写成数据流", section
 * "精度、掩码和边界情况": ragged tails and no work on padding).  Sequence b
 * is an independent problem: its queries are tokens cu_seqlens_q[b] ..
 * cu_seqlens_q[b+1]-1, its keys tokens cu_seqlens_k[b] .. cu_seqlens_k[b+1]-1,
 * with the causal alignment of fa_fwd applied to its own lengths.
 *
 *   q           device bf16 [total_q, H, d] (token-major), 16-byte aligned.
 *   k, v        device bf16 [total_k, H, d], 16-byte aligned (may be NULL when
 *               total_k == 0).
 *   o           device bf16 [total_q, H, d], 16-byte aligned; rows of every
 *               sequence written, nothing else.
 *   lse         device fp32 [total_q, H], 4-byte aligned.
 *   cu_seqlens_q, cu_seqlens_k   device int32 [B+1], 4-byte aligned,
 *               non-decreasing, starting at 0 and ending at total_q / total_k.
 *               A sequence whose offsets fall outside [0, total] is treated as
 *               empty (nothing written for it).
 *   max_seqlen_q  at least every query length (sizes the grid; longer
 *               sequences are cut at it).
 *   scale, causal, d, stream   as for fa_fwd (no key_lens: lengths come from
 *               cu_seqlens_k).
 *
 * Returns FA_OK once enqueued, FA_ERR_INVALID_ARG / FA_ERR_MISALIGNED /
 * FA_ERR_UNSUPPORTED for bad arguments (checked before any CUDA call),
 * FA_ERR_NO_DEVICE or FA_ERR_CUDA otherwise.  B, H, total_q or max_seqlen_q
 * equal to 0 is a no-op.
 */
FA_API int fa_fwd_varlen(const void *q, const void *k, const void *v, void *o, float *lse,
                  const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k, int B, int H,
                  int total_q, int total_k, int max_seqlen_q, int d, float scale, int causal,
                  fa_stream_t stream);

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
 * outputs are complete.  The work is cut into chunks of about 1/8 of the
 * (batch, head) pairs (runs of heads of one batch entry, or whole batch
 * entries; with runs of heads the last chunk is cut further into halves, so
 * little work is left after the last input copy), each its own fa_fwd
 * launch; the library's own copy streams move
 * chunk c+1 in and chunk c-1 out while chunk c runs (it waits for earlier work
 * on `stream` before touching the workspace).  The result is the same, bit for
 * bit, as fa_fwd on the whole problem.  Calls on one device are serialised.  Returns FA_ERR_INVALID_ARG if the workspace is too
 * small, FA_ERR_CUDA if a copy fails, plus every fa_fwd error.
 */
FA_API int fa_fwd_host(const void *q, const void *k, const void *v, void *o, float *lse,
                int B, int H, int N_q, int N_k, int d, float scale, int causal,
                const int32_t *key_lens, void *workspace, size_t workspace_bytes,
                fa_stream_t stream);

/*
 * Split-KV forward (decode-shaped problems: few query rows, long keys).
 *
 * Same operation, masks, layouts and outputs as fa_fwd.  The K/V tiles each
 * 128-row query block must visit are cut into num_splits contiguous ranges;
 * one CTA per (range, query block, head, batch) computes that range's
 * normalised partial output O_s and log-sum-exp LSE_s into the workspace and
 * counts its arrival for its query block; the last of the block's CTAs to
 * arrive merges the ranges of the block's rows: with M = max_s LSE_s and
 * w_s = exp(LSE_s - M), O = sum_s w_s O_s / sum_s w_s and LSE = M + ln sum_s w_s
 * (a row with no visible key in any range: O = 0, LSE = -inf).  One kernel
 * launch per call: the arrival words carry a ticket drawn for each call, so
 * they need no reset between calls.  This is the
 * decode / FlashDecoding case "FlashAttention：把注意力从公式写成数据流"
 * (section "端侧与专用加速器") and "[2205.14135] FlashAttention: Fast and
 * Memory-Efficient Exact Attention with IO-Awareness" point to, merged with the
 * same running-max rule as the online softmax ("分块与在线 softmax").  It
 * spreads a small query batch over all SMs.
 */

/*
 * fa_splitkv_num_splits -- a range count for this problem: 1 when the plain
 * grid (one CTA per 128 query rows and head) already covers 4/5 of the current
 * device's SMs, else as many ranges as keep the grid within one wave (one CTA
 * per SM), with at least two K/V tiles (256 keys) per range and at most 256
 * ranges.  The SM count is the current device's multiProcessorCount (148 on a
 * B200); with no device visible it is taken as 148.  Returns 1 for empty or
 * invalid sizes.  Host arithmetic plus that one device query.
 */
FA_API int fa_splitkv_num_splits(int B, int H, int N_q, int N_k);

/*
 * fa_fwd_splitkv_workspace_size -- bytes of device workspace fa_fwd_splitkv
 * needs: num_splits*B*H*N_q*d fp32 partial outputs, num_splits*B*H*N_q fp32
 * partial LSEs and ceil(N_q/128)*B*H 64-bit arrival words, each part 256-byte
 * aligned.  Returns 0 for invalid sizes or num_splits outside [1, 256].
 */
FA_API size_t fa_fwd_splitkv_workspace_size(int B, int H, int N_q, int d, int num_splits);

/*
 * fa_fwd_splitkv -- split-KV forward on device buffers, asynchronous on `stream`.
 *
 *   q .. key_lens, stream   as for fa_fwd.
 *   num_splits              1 .. 256 (more ranges than K/V tiles leaves some
 *                           ranges empty, which is allowed).
 *   workspace               device buffer of at least
 *                           fa_fwd_splitkv_workspace_size(B,H,N_q,d,num_splits)
 *                           bytes, 256-byte aligned, owned by the caller; it
 *                           needs no initial contents.  Calls that share a
 *                           workspace must be ordered (same stream or events).
 *
 * Returns what fa_fwd returns, plus FA_ERR_INVALID_ARG for num_splits out of
 * range or a NULL / too small workspace and FA_ERR_MISALIGNED for a workspace
 * that is not 256-byte aligned (all checked before any CUDA call).
 */
FA_API int fa_fwd_splitkv(const void *q, const void *k, const void *v, void *o, float *lse,
                   int B, int H, int N_q, int N_k, int d, float scale, int causal,
                   const int32_t *key_lens, int num_splits, void *workspace,
                   size_t workspace_bytes, fa_stream_t stream);

/*
 * fa_fwd_splitkv_noalloc -- fa_fwd_splitkv for callers that cannot allocate
 * device memory: the same kernels, with the workspace taken from a scratch
 * array the library holds in a file-scope device variable of 16 MiB
 * (16777216 bytes) per device, sized when the library's module loads.  The
 * paper has no counterpart: this is a library convenience, not part of the
 * method.
 *
 *   q .. key_lens, num_splits, stream   as for fa_fwd_splitkv.
 *
 * Returns what fa_fwd_splitkv returns, except that a problem whose workspace
 * (fa_fwd_splitkv_workspace_size) exceeds 16 MiB is rejected with
 * FA_ERR_UNSUPPORTED before any CUDA call.  Nothing in the scratch needs to
 * start at zero.  All calls on one device share the one scratch array: calls
 * must not overlap in time (issue them on one stream, or order them with
 * events); two calls running concurrently on different streams corrupt each
 * other's partial results.  The first call on each device looks up the
 * scratch address and sets kernel attributes (host-side setup, no stream
 * work): make that first call outside any stream capture.
 */
FA_API int fa_fwd_splitkv_noalloc(const void *q, const void *k, const void *v, void *o, float *lse,
                           int B, int H, int N_q, int N_k, int d, float scale, int causal,
                           const int32_t *key_lens, int num_splits, fa_stream_t stream);

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
 * fa_selftest_fwd_timeout -- failure-detection self test of the forward
 * kernel's own wind-down.  Runs the fa_fwd kernel (arguments as fa_fwd, no
 * key_lens) with every pipeline wait bounded by `limit_cycles` SM clock cycles
 * (1 .. 2^32) instead of the default of about a second, synchronises `stream`
 * and returns what fa_get_device_status reports.  With a limit of a few
 * cycles some wait runs out: that CTA and every role in it stop, each role
 * first waiting (with the default limit) for the copies and MMAs it has
 * already issued, so no asynchronous work lands in released shared memory or
 * TMEM; the call returns FA_ERR_DEVICE_TIMEOUT and the CUDA context stays
 * usable.  o and lse then hold unspecified values.  N_k must be > 0 and
 * B*H*N_q > 0 (otherwise nothing would wait: FA_ERR_INVALID_ARG).
 */
FA_API int fa_selftest_fwd_timeout(const void *q, const void *k, const void *v, void *o,
                                   float *lse, int B, int H, int N_q, int N_k, int d,
                                   float scale, int causal, unsigned long long limit_cycles,
                                   fa_stream_t stream);

/*
 * fa_selftest_bwd_timeout -- failure-detection self test of the backward
 * kernel's wind-down.  Runs fa_bwd (arguments as fa_bwd, no key_lens) with
 * every pipeline wait of the main kernel bounded by `limit_cycles` SM clock
 * cycles (1 .. 2^32) instead of about a second, synchronises `stream` and
 * returns what fa_get_device_status reports.  With a limit of a few cycles
 * some wait runs out: every role of that CTA stops after waiting (with the
 * default limit, ignoring the abort) for the copies, MMAs and tensor
 * reduce-adds it has already issued, so nothing lands in released shared
 * memory or TMEM; the call returns FA_ERR_DEVICE_TIMEOUT and the CUDA context
 * stays usable.  dq, dk and dv then hold unspecified values.  B, H, N_q and N_k
 * must be > 0 (otherwise nothing would wait: FA_ERR_INVALID_ARG).
 */
FA_API int fa_selftest_bwd_timeout(const void *q, const void *k, const void *v, const void *o,
                                   const float *lse, const void *dout, void *dq, void *dk,
                                   void *dv, int B, int H, int N_q, int N_k, int d, float scale,
                                   int causal, void *workspace, size_t workspace_bytes,
                                   unsigned long long limit_cycles, fa_stream_t stream);

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
