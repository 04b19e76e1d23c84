/*
 * fa.h -- C ABI of the B200 (sm_100a) exact attention forward library
 * (libfa.so).
 *
 * The operation: exact attention O = softmax(scale * Q K^T) V together with
 * the per-row logsumexp, computed tile by tile with the online-softmax running
 * maximum and running sum so that the score and probability matrices never
 * reach device memory.  Pages: "Flash Attention" (14cs17.netlify.app),
 * sections "Tiling Strategy", "Online Softmax" (Theorem 2) and "Flash
 * Attention Algorithm"; the problem statement there is Q, K, V in R^{N x d}
 * and softmax(QK^T)V.  "Flash Attention 2 Improvements" on the same page adds
 * the variable sequence lengths and grouped-query attention supported here.
 *
 * All entry points are plain C: pointers, sizes, and an opaque stream handle.
 */
#ifndef FA_B200_H
#define FA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes.  Every entry point returns FA_OK (0) or a negative code. */
typedef enum {
    FA_OK = 0,
    FA_ERR_NULL = -1,            /* a required pointer is NULL                        */
    FA_ERR_SHAPE = -2,           /* a size is negative or out of the supported range  */
    FA_ERR_HEADDIM = -3,         /* d is not 64 or 128                                */
    FA_ERR_GQA = -4,             /* Hkv < 1 or Hq is not a multiple of Hkv            */
    FA_ERR_ALIGN = -5,           /* q, k, v or o not 16-byte aligned, lse not 4-byte  */
    FA_ERR_ARCH = -6,            /* current device is not compute capability 10.0     */
    FA_ERR_LAUNCH = -7,          /* the CUDA runtime refused the launch (or no device)*/
    FA_ERR_DEVICE_TIMEOUT = -8,  /* device watchdog: a pipeline wait ran out          */
    FA_ERR_SEQLENS = -9          /* cu_seqlens inconsistent (found on the device)     */
} fa_status;

/*
 * fa_fwd -- attention forward, asynchronous on `stream`.
 *
 *   q, k, v     bf16 inputs (device memory, read only).
 *   o           bf16 output (device memory), same layout as q.
 *   lse         fp32 output (device memory): natural-log logsumexp of each
 *               row of scale * Q K^T over its allowed keys; -inf for a row
 *               with no allowed key (its O row is then 0).
 *   B           dense: batch size.  Packed: number of sequences.
 *   Hq, Hkv     query heads and key/value heads; Hq % Hkv == 0.  Query head h
 *               reads key/value head h / (Hq / Hkv).
 *   N           dense: sequence length.  Packed: total tokens (must equal
 *               cu_seqlens[B]).
 *   d           head dimension, 64 or 128.
 *   scale       multiplies Q K^T before the softmax (1/sqrt(d) is usual).
 *   causal      nonzero: key j is allowed for query i iff j <= i, positions
 *               counted inside the row's own sequence.
 *   cu_seqlens  NULL for a dense batch.  Otherwise device memory holding B+1
 *               int32 offsets, cu_seqlens[0] = 0, non-decreasing; sequence s
 *               owns tokens [cu_seqlens[s], cu_seqlens[s+1]).
 *   stream      a cudaStream_t (NULL = legacy default stream).
 *
 * Layouts (all contiguous, row-major):
 *   dense   q, o [B, Hq, N, d]   k, v [B, Hkv, N, d]   lse [B, Hq, N]
 *   packed  q, o [N, Hq, d]      k, v [N, Hkv, d]      lse [Hq, N]
 *
 * Limits: packed batches hold at most 1024 sequences, each at most 262144
 * tokens long (FA_ERR_SHAPE / device FA_ERR_SEQLENS otherwise).  B == 0 or
 * N == 0 is an empty problem: FA_OK, nothing is launched and the pointers
 * may be NULL.
 *
 * Ownership: the caller owns every buffer.  The library allocates only a
 * small per-device status word and a ring of 64 work counters (8 bytes each),
 * once, on the first call on that device.  A launch with at least 4 work
 * items (pairs of 128-row query tiles) per SM hands the items to its CTAs
 * through one of those counters; consecutive calls take consecutive counters,
 * each tagged with the call's number, so calls in flight together on
 * different streams do not share one; a launch that completes leaves its
 * counter at zero, so a captured call (a CUDA graph) can be replayed.  (A
 * replay of a launch that reported FA_ERR_DEVICE_TIMEOUT may find its counter
 * not at zero; make a new call instead.)
 *
 * Errors: argument errors are found on the host before any launch and return
 * the codes above.  Errors found on the device (a pipeline wait that ran past
 * its time limit, inconsistent cu_seqlens) do not abort the context: the
 * kernel records a code in the device status word and returns; read it with
 * fa_get_device_status().
 */
int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
           int B, int Hq, int Hkv, int N, int d, float scale, int causal,
           const int32_t* cu_seqlens, void* stream);

/*
 * fa_fwd_kvcache -- forward for a chunk of Nq queries against Nk keys (dense
 * batches), asynchronous on `stream`.  This is the shape of chunked prefill
 * ("FlashAttention and Chunked Prefill Mechanics", section 1: a long prompt is
 * split into chunks, each attending to the keys and values of all earlier
 * tokens) and of attending to a KV cache ("Flash Attention", KV Cache named as
 * composable with the method).
 *
 *   q, o   [B, Hq, Nq, d] bf16      k, v  [B, Hkv, Nk, d] bf16
 *   lse    [B, Hq, Nq] fp32         Nq >= 1, Nk >= 1
 *
 * The chunk's rows are the LAST Nq positions of the Nk-long sequence: query
 * row i sits at position Nk - Nq + i.  causal != 0 allows key j for row i iff
 * j <= Nk - Nq + i (so Nk >= Nq is required); causal == 0 allows every key.
 * With Nq == Nk this is exactly fa_fwd.  Running a sequence through
 * consecutive chunks [a, b) against keys [0, b) reproduces the rows of the
 * whole causal forward.  Other arguments, ownership and errors as fa_fwd
 * (FA_ERR_SHAPE also for Nk == 0, or causal with Nk < Nq).
 */
int fa_fwd_kvcache(const void* q, const void* k, const void* v, void* o, float* lse,
                   int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                   void* stream);

/*
 * fa_fwd_fp8 -- the forward with FP8 inputs (dense batches, d = 64 or 128),
 * asynchronous on `stream`.  "FlashAttention and Chunked Prefill Mechanics"
 * (section 1) names FlashAttention-3's FP8 support; the same tiled algorithm
 * runs on E4M3 operands with fp32 accumulation:
 *
 *   q, k, v        FP8 E4M3 codes (1 byte each, OCP E4M3: 4 exponent bits with
 *                  bias 7, 3 mantissa bits), dense layouts of fa_fwd.  The
 *                  values are code * q_scale, code * k_scale, code * v_scale
 *                  (per-tensor scales, finite and > 0).
 *   o, lse         bf16 output and fp32 logsumexp, as fa_fwd.
 *
 * S = Q K^T is computed exactly from the codes (E4M3 products are exact in
 * fp32) and scaled by scale * q_scale * k_scale; the exponentials are rounded
 * to E4M3 for the P V product (relative error <= 2^-4 for P >= 2^-6), O is
 * divided by the fp32 row sum and multiplied by v_scale.  At d = 64 each
 * 64-byte row is read into a 128-byte shared-memory row whose other half the
 * copy fills with zeros, so the score MMAs run over 128 columns (half of
 * them zero; the FP8 forward is bound by its exponentials, not its MMAs).
 * Errors: as fa_fwd; FA_ERR_HEADDIM for d other than 64 or 128, FA_ERR_SHAPE
 * for a scale that is not finite and positive.
 */
int fa_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse,
               int B, int Hq, int Hkv, int N, int d, float scale, int causal,
               float q_scale, float k_scale, float v_scale, void* stream);

/*
 * fa_fwd_fp8_varlen -- fa_fwd_fp8 on a packed batch of variable-length
 * sequences ("Flash Attention" page, "Flash Attention 2 Improvements":
 * variable sequence lengths; "FlashAttention and Chunked Prefill Mechanics",
 * section 1: FP8).  Layouts, masks and errors are those of fa_fwd with
 * cu_seqlens != NULL (q, o [N_total, Hq, d]; k, v [N_total, Hkv, d], d = 64 or 128;
 * lse [Hq, N_total]; cu_seqlens int32 [B + 1] on the device with
 * cu_seqlens[B] == N, checked on the device: FA_ERR_SEQLENS through
 * fa_get_device_status), with E4M3 q, k, v codes and per-tensor scales as
 * fa_fwd_fp8.  cu_seqlens must not be NULL (FA_ERR_NULL) unless B or N is 0.
 */
int fa_fwd_fp8_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                      int B, int Hq, int Hkv, int N, int d, float scale, int causal,
                      float q_scale, float k_scale, float v_scale, const int32_t* cu_seqlens,
                      void* stream);

/*
 * fa_fwd_kvcache_varlen -- fa_fwd_kvcache on a packed batch: B sequences, each
 * with its own query chunk against its own keys ("FlashAttention and Chunked
 * Prefill Mechanics", section 1: a prefill split into chunks, the chunks of
 * several requests run together; "Flash Attention" page, "Flash Attention 2
 * Improvements": variable sequence lengths).  Sequence s has query rows
 * [cu_seqlens_q[s], cu_seqlens_q[s+1]) and keys [cu_seqlens_k[s],
 * cu_seqlens_k[s+1]) (both int32 [B + 1] on the device); its Lq rows are the
 * last Lq of its Lk positions, so with causal row i may attend keys
 * 0 .. Lk - Lq + i (bottom-right alignment; Lk >= Lq is required).
 *   q, o   [Nq, Hq, d] bf16 (Nq = cu_seqlens_q[B] query tokens in total)
 *   k, v   [Nk, Hkv, d] bf16 (Nk = cu_seqlens_k[B] key tokens in total)
 *   lse    [Hq, Nq] fp32
 * The offsets are checked on the device (starts at 0, totals Nq and Nk, no
 * negative lengths, Lk >= Lq when causal, Lk > 0 for a non-empty chunk when
 * not causal): a failure writes nothing and reports FA_ERR_SEQLENS through
 * fa_get_device_status.  Host errors: as fa_fwd; FA_ERR_NULL also for a NULL
 * offset array, FA_ERR_SHAPE for B > 1024.  A sequence may have Lq = 0.
 */
int fa_fwd_kvcache_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                          int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                          const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, void* stream);

/*
 * fa_fwd_partial -- one key range's share of the forward, for merging later
 * (ring attention, any split of the keys).  Same arguments, layouts and
 * masks as fa_fwd_kvcache (query row i at key position Nk - Nq + i), but the
 * results go, in fp32, to
 *   o_part    [B, Hq, Nq, d]: O / l over this call's keys (0 for a row with
 *             no allowed key),
 *   lse_part  [B, Hq, Nq]: the logsumexp over this call's keys (-inf for a
 *             row with no allowed key).
 * fa_merge_partials combines such shares of the same rows (the online-softmax
 * rescale of "Flash Attention", Online Softmax, Theorem 2, applied to whole
 * key ranges).  Errors as fa_fwd_kvcache.
 */
int fa_fwd_partial(const void* q, const void* k, const void* v, float* o_part, float* lse_part,
                   int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                   void* stream);

/*
 * fa_merge_partials -- merges nparts shares of the same `rows` query rows:
 * o_parts [nparts][rows][d] and lse_parts [nparts][rows] (fp32, device) as
 * fa_fwd_partial writes them, into bf16 o [rows][d] and fp32 lse [rows]:
 *   lse = ln sum_s exp(lse_s),  O = sum_s exp(lse_s - lse) O_s.
 * A share with lse_s = -inf carries weight 0; a row without any allowed key
 * gets O = 0, lse = -inf.  d is 64 or 128; 1 <= nparts <= 4096;
 * rows * nparts <= 2^40 and rows <= 8 * (2^31 - 1) (one block per 8 rows),
 * else FA_ERR_SHAPE.  Asynchronous on `stream`.  Errors: FA_ERR_SHAPE,
 * FA_ERR_HEADDIM, FA_ERR_NULL,
 * FA_ERR_ALIGN (o 16-byte aligned), FA_ERR_LAUNCH.
 */
int fa_merge_partials(const float* o_parts, const float* lse_parts, int nparts, long long rows, int d,
                      void* o, float* lse, void* stream);

/*
 * fa_fwd_splitkv -- fa_fwd_kvcache for decode-shaped problems (a few query
 * rows against a long KV cache), asynchronous on `stream`.  Same arguments,
 * layouts, masks and result as fa_fwd_kvcache, plus:
 *
 *   num_splits       1 .. 256: the key blocks of every query tile are cut
 *                    into this many contiguous ranges ("splits") that run as
 *                    separate work items on different SMs.
 *   workspace        device memory, 16-byte aligned, of at least
 *                    fa_splitkv_workspace_bytes(B, Hq, Nq, d, num_splits)
 *                    bytes (0 when num_splits == 1; it may then be NULL).
 *                    Each split writes its normalised output and logsumexp
 *                    there in fp32; a second kernel on the same stream merges
 *                    them with the rescaling of "Online Softmax" (Theorem 2):
 *                    lse = ln sum_s exp(lse_s), O = sum_s exp(lse_s - lse) O_s.
 *                    The workspace must not be used by anything else until
 *                    that kernel is done; nothing in it needs initialising.
 *
 * When Hq > Hkv and Nq < 128, the query rows of the Hq / Hkv heads that
 * share a key/value head are processed in one 128-row tile, so each K/V
 * block is read once for all of them.  The page gives no decode algorithm;
 * splitting the keys is the same block-wise combination the method applies
 * within one sequence (the split results are combined exactly, up to fp32
 * rounding).  Errors as fa_fwd_kvcache; FA_ERR_SHAPE also for num_splits out
 * of range or a workspace smaller than required, FA_ERR_NULL for a missing
 * workspace, FA_ERR_ALIGN for a misaligned one.
 */
int fa_fwd_splitkv(const void* q, const void* k, const void* v, void* o, float* lse,
                   int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                   int num_splits, void* workspace, size_t workspace_bytes, void* stream);

/*
 * fa_splitkv_num_splits -- the split count fa_fwd_splitkv runs best with on
 * the current device for this shape (from the number of work items and the
 * device's SM count), >= 1; or a negative fa_status for invalid sizes or no
 * usable device.
 */
int fa_splitkv_num_splits(int B, int Hq, int Hkv, int Nq, int Nk, int d);

/*
 * fa_splitkv_workspace_bytes -- workspace fa_fwd_splitkv needs:
 * num_splits * B * Hq * Nq * (d + 1) * 4 bytes, 0 when num_splits == 1 and 0
 * for invalid arguments.  Needs no device.
 */
size_t fa_splitkv_workspace_bytes(int B, int Hq, int Nq, int d, int num_splits);

/*
 * fa_bwd -- gradients of fa_fwd, asynchronous on `stream`.  The backward
 * pass recomputes the scores block by block from Q and K and the logsumexp
 * that fa_fwd saved, instead of storing them ("Flash Attention",
 * 14cs17.netlify.app, "Common Pitfalls", Pitfall 3; fromzero2ai.dev, "Core
 * Mechanisms of FlashAttention", item 3).  The gradients are those of the
 * forward's definition: with P = softmax(scale Q K^T) (masked) and the
 * upstream gradient dO,
 *     dV = P^T dO,  dS = P * (dO V^T - D),  D_i = sum_c dO_ic O_ic,
 *     dQ = scale dS K,  dK = scale dS^T Q,
 * the query heads of a group adding into their key/value head's dK and dV.
 *
 *   q, k, v, o, lse   the forward's inputs and outputs (o bf16, lse fp32 as
 *                     fa_fwd wrote them), device memory, read only.
 *   dout              bf16 upstream gradient, same layout as o.
 *   dq                bf16 output, layout of q.
 *   dk, dv            bf16 outputs, layout of k (written, not accumulated).
 *   B, Hq, Hkv, N, d, scale, causal, cu_seqlens
 *                     as fa_fwd: dense (cu_seqlens NULL) q, o, dout, dq
 *                     [B, Hq, N, d], k, v, dk, dv [B, Hkv, N, d], lse
 *                     [B, Hq, N]; packed (cu_seqlens: B+1 device offsets,
 *                     at most 1024 sequences) q, o, dout, dq [N, Hq, d],
 *                     k, v, dk, dv [N, Hkv, d], lse [Hq, N].
 *   workspace         device memory, 16-byte aligned, at least
 *                     fa_bwd_workspace_bytes(B, Hq, N, d, packed) bytes: an
 *                     fp32 dQ accumulator and two per-row fp32 vectors on rows
 *                     padded to 128 per sequence (packed: and the schedule
 *                     tables).  Nothing in it needs initialising; it must not
 *                     be used by anything else until the call's kernels have
 *                     finished on `stream`.
 *
 * Kernels on `stream`: (packed) a table pass that checks cu_seqlens and
 * orders the sequences longest first, a pass computing D and clearing the
 * accumulator, the main kernel (one 128-key block of one (sequence, kv head)
 * per work item, dK and dV kept in tensor memory, each block's dQ share added
 * into the accumulator with fp32 reductions), and the dQ conversion.  The
 * order of the fp32 reductions varies from run to run, so dQ may differ in
 * its last bits between runs; dK and dV do not.
 *
 * Errors as fa_fwd (FA_ERR_NULL also for a missing workspace, FA_ERR_ALIGN for
 * a misaligned one, FA_ERR_SHAPE for one that is too small or more than 1024
 * sequences; inconsistent cu_seqlens are reported on the device as
 * FA_ERR_SEQLENS and leave the outputs unwritten).  B == 0 or N == 0 is an
 * empty problem (FA_OK, nothing launched).
 */
int fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
           const void* dout, void* dq, void* dk, void* dv,
           int B, int Hq, int Hkv, int N, int d, float scale, int causal,
           const int32_t* cu_seqlens, void* workspace, size_t workspace_bytes, void* stream);

/*
 * fa_bwd_workspace_bytes -- workspace fa_bwd needs.  Dense (packed == 0):
 * B * Hq * Npad * (d + 2) * 4 bytes with Npad = N rounded up to 128.
 * Packed: Hq * Npad * (d + 2) * 4 + (3 B + 4) * 4 bytes with Npad = N + 128 B
 * rounded up to 128.  0 for invalid arguments.  Needs no device.
 */
size_t fa_bwd_workspace_bytes(int B, int Hq, int N, int d, int packed);

/*
 * fa_get_device_status -- reads and clears the status word of the current
 * device.  Synchronises `stream` (a cudaStream_t) first, so it reports every
 * fa_fwd launched on that stream before the call.  Returns FA_OK, a negative
 * device-side code (FA_ERR_DEVICE_TIMEOUT, FA_ERR_SEQLENS), or FA_ERR_LAUNCH
 * if the runtime reports an error.
 */
int fa_get_device_status(void* stream);

/*
 * fa_selftest_watchdog -- checks the device-side watchdog without any fault.
 * Launches on `stream` one thread that waits, through the same bounded wait
 * the forward kernel uses, on a barrier nothing ever completes; after
 * timeout_ms (1 .. 2000) the wait gives up, records FA_ERR_DEVICE_TIMEOUT in
 * the status word (read it with fa_get_device_status) and the kernel returns.
 * The context stays usable.  Returns FA_OK once launched, FA_ERR_SHAPE for a
 * timeout out of range, or the device set-up error.
 */
int fa_selftest_watchdog(int timeout_ms, void* stream);

/* fa_status_string -- static, human-readable text for a status code. */
const char* fa_status_string(int status);

/*
 * fa_fwd_noalloc -- fa_fwd for callers that must not allocate device memory.
 * (An addition of this library; the pages have no counterpart.)
 *
 * fa_fwd allocates one small device buffer, its status word, with cudaMalloc
 * the first time it runs on a device.  Some callers cannot allow that: a
 * process whose device memory is reserved up front by another allocator
 * (a serving runtime that claims nearly all of HBM at start-up), so that a
 * stray cudaMalloc fails or fragments its pool; a latency-critical loop where
 * cudaMalloc's implicit device-wide synchronisation is not acceptable; or a
 * code base whose policy forbids new allocations after initialisation.
 *
 * This entry point takes the same arguments, has the same layouts, limits and
 * host-side error codes as fa_fwd, and computes the same result with the same
 * kernel.  It calls no cudaMalloc, cudaFree or other allocating routine: its
 * only scratch, the status words (16 bytes) and a ring of 16 work counters
 * (128 bytes) whatever the problem size, lives in a fixed 256-byte array
 * compiled into the library, which every GPU that loads the library holds
 * until the process exits.  Since the need does not grow with B, N, Hq or d,
 * no problem is too large for the array.
 *
 * The first call on each device sets that device up (device properties, the
 * kernels' shared-memory limits and the array's device address); make that
 * first call before any stream capture.
 *
 * All calls share the array, which keeps the last call's contents; each call
 * clears the status words on its stream before its kernel starts.  Calls that
 * overlap on the GPU (different streams, or several host threads) race on the
 * status words (the work counters they take are distinct unless 16 or more
 * calls are in flight at once).  Device-side errors of this entry point (FA_ERR_DEVICE_TIMEOUT,
 * FA_ERR_SEQLENS) are written to that array only: read them with
 * fa_get_noalloc_status, not fa_get_device_status (which reports fa_fwd's
 * word).
 */
int fa_fwd_noalloc(const void* q, const void* k, const void* v, void* o, float* lse,
                   int B, int Hq, int Hkv, int N, int d, float scale, int causal,
                   const int32_t* cu_seqlens, void* stream);

/*
 * fa_get_noalloc_status -- reads and clears the device-side status word of
 * fa_fwd_noalloc on the current device.  (Part of the no-allocation addition;
 * the pages have no counterpart.)
 *
 * Copies the status words out of the library's fixed array with
 * cudaMemcpyAsync on `stream` into a host variable, zeroes them with
 * cudaMemsetAsync on the same stream, and waits for `stream`; so it reports
 * the last fa_fwd_noalloc call ordered before it on `stream`.  Allocates no
 * device memory (on a device where fa_fwd_noalloc has not run yet it does that
 * device's set-up first, which allocates nothing either).
 *
 * Returns FA_OK, the first device-side error recorded since the words were
 * last cleared (FA_ERR_DEVICE_TIMEOUT, FA_ERR_SEQLENS), or a host-side error
 * (FA_ERR_ARCH, FA_ERR_LAUNCH).  Shares the array's race: a fa_fwd_noalloc
 * call running concurrently on another stream may be reported or cleared.
 */
int fa_get_noalloc_status(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* FA_B200_H */
