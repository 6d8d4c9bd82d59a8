/*
 * fa.h -- C ABI of the B200 (sm_100a) exact-attention forward library
 *         (libfa_b200.so, built from exact_attention_122_b200/csrc/).
 *
 * The operation (page "Flash attention optimization", section "Attention is
 * not slow because of arithmetic"): for every batch b and head h, with Q, K,
 * V in R^{N x d},
 *
 *     S = scale * Q K^T,   P = softmax(S) row-wise,   O = P V,
 *
 * computed tile by tile with the online-softmax recurrence (same page, "The
 * fix: tile the computation, never materialize the full matrix"; page
 * "FlashAttention: The GPU Memory Hack That Changed Everything", "The Tiling
 * Strategy"), so no N x N matrix ever reaches device memory.  With causal
 * masking (that page's is_causal=True, "Integration: It's Everywhere") key j
 * is allowed for query i iff j <= i.  The result is exact up to rounding
 * order; O is rounded to bf16 once at the end.
 *
 * Conventions shared by every entry point:
 *  - Pointers named q, k, v, o, lse are DEVICE pointers owned by the caller
 *    (fa_fwd_host alone takes HOST pointers there).  The library never
 *    allocates, frees or retains them.
 *  - Work is enqueued on `stream` (a cudaStream_t passed as void*; NULL is
 *    the legacy default stream) and the call returns without synchronising
 *    (fa_fwd_host on pageable host memory excepted: CUDA copies pageable
 *    memory synchronously).  Results are valid once the caller has
 *    synchronised that stream.
 *  - Arguments are validated before anything is enqueued; an invalid call
 *    returns an error status and has no side effect.
 *  - Calls are thread-safe.  Calls on different streams compute
 *    independently (each uses only its own arguments and workspace), with
 *    one exception: the watchdog status word read by fa_get_device_status
 *    is one per device, shared by all streams (see there).
 *  - Inputs holding NaN or Inf are not detected; they propagate.
 */
#ifndef FA_B200_H
#define FA_B200_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FA_OK = 0,
    FA_ERR_INVALID_ARG = 1,   /* NULL pointer, size < 1, bad flag, scale not finite or <= 0 */
    FA_ERR_UNSUPPORTED = 2,   /* head dim not 64/128, sizes beyond the limits, device not sm_100 */
    FA_ERR_MISALIGNED = 3,    /* q/k/v/o not 16-byte aligned, lse not 4-byte aligned */
    FA_ERR_LAUNCH = 4,        /* the CUDA runtime refused the launch (see fa_last_cuda_error) */
    FA_ERR_TIMEOUT = 5,       /* a kernel-side wait gave up (reported by fa_get_device_status) */
    FA_ERR_NO_DEVICE = 6      /* no usable CUDA device is current */
} fa_status;

/*
 * fa_fwd -- exact attention forward, O and the per-row log-sum-exp.
 *
 *  q, k, v : const bf16 [B][H][N][d], contiguous, d innermost (the
 *            (batch, heads, seq_len, head_dim) layout of the "Try It
 *            Yourself" script of the FlashAttention explainer page).
 *  o       : bf16 [B][H][N][d], contiguous; O = softmax(S) V rounded to bf16
 *            (round-to-nearest-even).
 *  lse     : float [B][H][N]; lse[b][h][i] = ln sum_j exp(S_ij) over the
 *            allowed keys, natural-log units, scale included.  It is the
 *            O(N) per-row statistic ("m and l") that the page keeps for a
 *            backward pass that recomputes P ("Sizing a tile, and why the
 *            backward pass recomputes instead of storing").
 *  B, H, N : batch, heads, sequence length; each >= 1.  N need not be a
 *            multiple of the tile size.  B*H <= 2^31-1, N <= 2^30, and
 *            B*H*ceil(N/256) <= 2^30.
 *  d       : head dimension, 64 or 128 (else FA_ERR_UNSUPPORTED).
 *  causal  : 0 = no mask, 1 = key j allowed for query i iff j <= i.
 *  scale   : multiplier of Q K^T, finite and > 0 (usually 1/sqrt(d)).
 *  stream  : cudaStream_t as void*.
 *
 * Errors: FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_MISALIGNED are
 * returned before any device work; FA_ERR_NO_DEVICE if no device is
 * current; FA_ERR_LAUNCH if the launch fails.  The buffers q/k/v/o/lse must
 * not overlap o or lse.  Uses no device memory besides its arguments.
 */
fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                 int B, int H, int N, int d, int causal, float scale, void* stream);

/*
 * fa_fwd_strided -- fa_fwd for strided operands, e.g. [B][N][H][d] tensors
 * viewed as (B, H, N, d) (the layout transformer projections produce).
 *
 *  strides : 12 int64 values, element strides (batch, head, sequence) of q,
 *            k, v and o in that order.  The head dimension d is always
 *            contiguous.  Each stride must be >= d and a multiple of 8
 *            elements (16 bytes, a TMA requirement), except that the stride
 *            of a dimension of size 1 is ignored.  Rows of o must not
 *            overlap and o must not overlap q, k, v or lse.
 *  lse     : contiguous float [B][H][N] as in fa_fwd.
 * Other arguments as fa_fwd.  Errors: FA_ERR_INVALID_ARG for a NULL
 * `strides` or a stride < d, FA_ERR_MISALIGNED for a stride that is not a
 * multiple of 8 elements, FA_ERR_UNSUPPORTED for a stride of 2^39 elements or
 * more; otherwise as fa_fwd.
 */
fa_status fa_fwd_strided(const void* q, const void* k, const void* v, void* o, float* lse,
                         int B, int H, int N, int d, const long long* strides, int causal,
                         float scale, void* stream);

/* Bytes of device workspace fa_fwd_dynamic needs (one work counter, padded). */
#define FA_DYNAMIC_WORKSPACE_BYTES 256

/*
 * fa_fwd_dynamic -- fa_fwd / fa_fwd_strided with dynamic work distribution.
 *
 * The persistent CTAs claim 256-row units of work from a counter in
 * `workspace` (longest causal rows first, heads grouped for L2 reuse)
 * instead of following a fixed assignment.  This balances long causal
 * problems better (measured on B200: 2-5 % faster from about 1000 units),
 * while on small ones (under about 4 units per SM) the counter's reset and
 * claims cost a few microseconds, so fa_fwd is faster there.  The result is
 * identical to fa_fwd.  The
 * parallel split over the sequence is the one of the page "FlashAttention:
 * The GPU Memory Hack That Changed Everything", "FlashAttention-2: Even
 * Faster".
 *
 *  strides         : NULL (contiguous [B][H][N][d]) or 12 strides as in
 *                    fa_fwd_strided.
 *  workspace       : device memory owned by the caller, 16-byte aligned,
 *                    at least FA_DYNAMIC_WORKSPACE_BYTES bytes.  The call
 *                    clears it on `stream` before the kernel runs, so its
 *                    contents on entry do not matter; it must not be used
 *                    by another call that may run at the same time.
 *  workspace_bytes : its size.
 * Other arguments as fa_fwd.  Errors: FA_ERR_INVALID_ARG for a NULL or too
 * small workspace, FA_ERR_MISALIGNED for a misaligned one; otherwise as
 * fa_fwd / fa_fwd_strided.
 */
fa_status fa_fwd_dynamic(const void* q, const void* k, const void* v, void* o, float* lse,
                         int B, int H, int N, int d, const long long* strides, int causal,
                         float scale, void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of the library's static device scratch used by fa_fwd_dynamic_noalloc. */
#define FA_NOALLOC_SCRATCH_BYTES 256
/* Largest B*H*ceil(N/256) fa_fwd_dynamic_noalloc accepts (its counter's range). */
#define FA_NOALLOC_MAX_UNITS (1LL << 30)

/*
 * fa_fwd_dynamic_noalloc -- fa_fwd_dynamic without a workspace argument, for
 * callers that cannot allocate device memory (a plugin inside an
 * application that owns every device allocation, or a latency-critical
 * loop that must not call cudaMalloc, which can synchronise the device).
 * The pages have no counterpart: this is a deployment variant, not part of
 * the method.
 *
 * The dynamic schedule's work counter lives in a static device array of
 * FA_NOALLOC_SCRATCH_BYTES bytes inside the library; every device that
 * loads the library holds it until the process exits.  The call allocates
 * nothing (no cudaMalloc, cudaFree or allocating library routine); the
 * caller still passes q, k, v, o and lse.
 *
 *  - The first call on a device resolves the array's device address
 *    (cudaGetSymbolAddress) with that device current; make that first call
 *    before any stream capture.
 *  - Every call shares the array and leaves its last contents there; the
 *    call clears the counter on `stream` before its kernel runs.  Calls that
 *    may overlap on the GPU (different streams not ordered by events) race
 *    on the counter and give wrong results: serialise them.
 *  - Problems with more than FA_NOALLOC_MAX_UNITS units (B*H*ceil(N/256))
 *    exceed the counter's range and return FA_ERR_UNSUPPORTED.
 *
 * Arguments (strides NULL or 12 strides as in fa_fwd_strided), results and
 * other errors as fa_fwd_dynamic; FA_ERR_LAUNCH if the set-up fails.
 */
fa_status fa_fwd_dynamic_noalloc(const void* q, const void* k, const void* v, void* o, float* lse,
                                 int B, int H, int N, int d, const long long* strides, int causal,
                                 float scale, void* stream);

/*
 * fa_fwd_host_workspace_bytes -- device workspace fa_fwd_host needs: two
 * slots, each holding Q, K, V, O and LSE of one chunk of heads plus a work
 * counter.  Returns 0 for sizes fa_fwd_host would reject.
 */
size_t fa_fwd_host_workspace_bytes(int B, int H, int N, int d);

/*
 * fa_fwd_host -- fa_fwd on tensors that live in HOST memory, with the
 * transfers overlapped with the attention.  A deployment variant (the pages
 * have no counterpart): the operation and the result are those of fa_fwd.
 *
 * The B*H heads are cut into up to 16 chunks of whole heads.  Chunk c is
 * copied into slot c % 2 of `workspace`, computed there by the persistent
 * forward kernel (dynamic schedule), and its O and LSE are copied back, on
 * three streams internal to the library, so the copy in of one chunk, the
 * attention of the previous one and the copy out of the one before run at
 * the same time.  With page-locked host memory the call is bound by the
 * host <-> device link; pageable memory gives the same result, serialised.
 *
 *  q, k, v  : HOST pointers, bf16 [B][H][N][d], contiguous (any alignment).
 *  o        : HOST pointer, bf16 [B][H][N][d];  lse : HOST pointer, float
 *             [B][H][N], natural log.  All five are owned by the caller and
 *             must stay valid, and o/lse unread, until `stream` is
 *             synchronised.
 *  workspace: DEVICE memory of the current device, owned by the caller,
 *             256-byte aligned, at least fa_fwd_host_workspace_bytes(...)
 *             bytes; calls that share it must be ordered (the same stream,
 *             or events).
 *  stream   : the call starts after the work queued on it and the stream
 *             waits for the last copy back, so synchronising it (or an event
 *             recorded on it after the call) covers the whole call.
 * Other arguments as fa_fwd.  Errors: as fa_fwd (no alignment rule on the
 * host buffers), plus FA_ERR_INVALID_ARG for a NULL or too small workspace
 * and FA_ERR_MISALIGNED for a workspace that is not 256-byte aligned.  Every
 * check runs before anything is enqueued.  FA_ERR_LAUNCH if a copy or a
 * launch is refused part-way; `stream` then still waits for the chunks
 * already queued, and o / lse hold only part of the result.
 */
fa_status fa_fwd_host(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                      int H, int N, int d, int causal, float scale, void* workspace,
                      size_t workspace_bytes, void* stream);

/* Largest number of query rows per (batch, head) fa_fwd_decode accepts (2^30). */
#define FA_DECODE_MAX_QUERIES 1073741824
/* Largest explicit split count of fa_fwd_decode. */
#define FA_DECODE_MAX_SPLITS 256

/*
 * fa_fwd_decode_workspace_bytes -- device workspace fa_fwd_decode needs for
 * these sizes (num_splits 0 = the automatic choice).  Returns 0 for sizes
 * fa_fwd_decode would reject as invalid.
 */
size_t fa_fwd_decode_workspace_bytes(int B, int H, int Nq, int Nk, int d, int num_splits);

/*
 * fa_fwd_decode -- exact attention for N_q queries against N_k keys with
 * N_q != N_k: decoding (few queries) and prefill against a cache.
 *
 * Same operation as fa_fwd with separate lengths: q, o bf16 [B][H][Nq][d]
 * and k, v bf16 [B][H][Nk][d], contiguous; lse float [B][H][Nq].  With
 * causal = 1 the queries are the last Nq positions of the key sequence:
 * query i may see key j iff j <= i + Nk - Nq (needs Nq <= Nk).
 *  - Nq <= 32: the keys are cut into `num_splits` ranges (0 = automatic)
 *    processed in parallel, each keeping the online-softmax running state of
 *    the page "Flash attention optimization" ("The fix: tile the computation
 *    ..."); a second kernel merges the ranges with that page's
 *    rescale-and-merge rule.  The queries go in blocks of 16 rows (one CTA
 *    each, the last block padded) to warp-level bf16 tensor-core MMAs.  This
 *    shape is bound by reading K and V once from device memory.
 *  - Nq > 32: the persistent tiled kernel of fa_fwd_dynamic (128-row tcgen05
 *    tiles), with the causal alignment above; num_splits is ignored and the
 *    workspace holds only its work counter.
 * In both, P is rounded to bf16 before the P V product, as in fa_fwd.
 *
 *  Nq          : 1 .. FA_DECODE_MAX_QUERIES.
 *  Nk          : >= 1 (>= Nq when causal), <= 2^30;  B*H <= 65535.
 *  num_splits  : 0 (automatic) .. FA_DECODE_MAX_SPLITS.
 *  workspace   : device memory owned by the caller, 256-byte aligned, at
 *                least fa_fwd_decode_workspace_bytes(...) bytes; it holds
 *                the per-split partial results (or the work counter) and
 *                must not be shared by calls that may run at the same time.
 * Errors: FA_ERR_INVALID_ARG (NULL pointers or workspace, sizes < 1,
 * causal with Nq > Nk, bad scale or split count, workspace too small),
 * FA_ERR_UNSUPPORTED (d not 64/128, Nq > FA_DECODE_MAX_QUERIES, sizes beyond
 * the limits, device not sm_100), FA_ERR_MISALIGNED, FA_ERR_NO_DEVICE,
 * FA_ERR_LAUNCH.
 */
fa_status fa_fwd_decode(const void* q, const void* k, const void* v, void* o, float* lse,
                        int B, int H, int Nq, int Nk, int d, int causal, float scale,
                        int num_splits, void* workspace, size_t workspace_bytes, void* stream);

/*
 * fa_fwd_fp8_workspace_bytes -- device workspace fa_fwd_fp8 needs: 256 bytes
 * of work counter and the transposed V (B*H*d*Npad bytes, Npad = N rounded
 * up to a multiple of 128).  Returns 0 for sizes fa_fwd_fp8 would reject.
 */
size_t fa_fwd_fp8_workspace_bytes(int B, int H, int N, int d);

/*
 * fa_fwd_fp8 -- exact attention forward over FP8 E4M3 inputs on the FP8 tensor
 * cores (page "FlashAttention: The GPU Memory Hack That Changed Everything",
 * "FlashAttention-3: Hopper Architecture": attention run in FP8 precision).
 *
 *  q8, k8, v8 : E4M3 codes [B][H][N][d], contiguous, d in {64, 128}; the values are
 *               code * descale_q (resp. _k, _v), one scale per tensor.
 *  o          : bf16 [B][H][N][d];  lse : fp32 [B][H][N], natural-log units
 *               of scale * (descale_q q8) . (descale_k k8).
 *  workspace  : device memory owned by the caller, 256-byte aligned, at least
 *               fa_fwd_fp8_workspace_bytes(...) bytes; not shared by calls
 *               that may run at the same time.
 * S = Q K^T is formed exactly from the codes in fp32; P is rounded to E4M3
 * (relative error up to 2^-4, values below 2^-6 on the E4M3 subnormal grid)
 * before the P V product, while the row sum uses the unrounded fp32 P.  The
 * work schedule is the one of fa_fwd_dynamic; a first pass writes V^T into
 * the workspace so both tensor-core operands are K-major.
 * Errors: FA_ERR_INVALID_ARG (NULL pointers, sizes < 1, bad causal flag, scale
 * or descale not finite and > 0, workspace too small), FA_ERR_UNSUPPORTED
 * (d not 64 or 128, B*H > 65535, sizes beyond the limits of fa_fwd, device not
 * sm_100), FA_ERR_MISALIGNED (inputs or o not 16-byte aligned, lse not
 * 4-byte aligned, workspace not 256-byte aligned), FA_ERR_NO_DEVICE,
 * FA_ERR_LAUNCH.
 */
fa_status fa_fwd_fp8(const void* q8, const void* k8, const void* v8, void* o, float* lse, int B,
                     int H, int N, int d, int causal, float scale, float descale_q,
                     float descale_k, float descale_v, void* workspace, size_t workspace_bytes,
                     void* stream);

/*
 * fa_bwd_workspace_bytes -- device workspace fa_bwd needs for these sizes:
 * an fp32 dQ accumulator [B][H][Npad][d] and two fp32 per-row vectors
 * [B][H][Npad], Npad = N rounded up to a multiple of 128.  Returns 0 for
 * sizes fa_bwd would reject.
 */
size_t fa_bwd_workspace_bytes(int B, int H, int N, int d);

/*
 * fa_bwd -- gradients of exact attention by recomputation.
 *
 * For O = softmax(scale * Q K^T [+ causal mask]) V with upstream gradient
 * dO = dL/dO, computes dQ, dK, dV without storing P: each P block is rebuilt
 * on chip from Q, K and the forward's LSE, as the page "Flash attention
 * optimization" describes in "Sizing a tile, and why the backward pass
 * recomputes instead of storing" (only the O(N) row statistics are kept).
 * With D_i = sum_t dO_it O_it and P = exp(scale Q K^T - LSE):
 *   dV = P^T dO,  dS = P * (dO V^T - D),  dQ = scale dS K,  dK = scale dS^T Q.
 *
 *  q, k, v, o, dout : bf16 [B][H][N][d] contiguous (o and lse as returned by
 *                     fa_fwd for the same q, k, v, causal and scale).
 *  lse              : fp32 [B][H][N], natural-log units.
 *  dq, dk, dv       : bf16 [B][H][N][d] contiguous, written.
 *  workspace        : device memory owned by the caller, 256-byte aligned,
 *                     >= fa_bwd_workspace_bytes(B, H, N, d) bytes; overwritten
 *                     and must not be shared by calls that may run at the same
 *                     time.  Nothing is allocated per call.
 *  B, H, N, d, causal, scale : as fa_fwd.
 * Products P and dS are rounded to bf16 before their tensor-core products;
 * accumulation is fp32.  dQ is accumulated with floating-point atomic adds,
 * so its low bits may differ from run to run; dK and dV are deterministic.
 * Errors: FA_ERR_INVALID_ARG (NULL pointers, sizes < 1, bad causal or scale,
 * workspace too small), FA_ERR_UNSUPPORTED (d not 64/128, sizes beyond the
 * limits of fa_fwd, device not sm_100), FA_ERR_MISALIGNED (tensors not
 * 16-byte aligned, lse not 4-byte aligned, workspace not 256-byte aligned),
 * FA_ERR_NO_DEVICE, FA_ERR_LAUNCH.  A watchdog timeout inside the kernel is
 * reported by fa_get_device_status.
 */
fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
                 const float* lse, void* dq, void* dk, void* dv, int B, int H, int N, int d,
                 int causal, float scale, void* workspace, size_t workspace_bytes, void* stream);

/*
 * fa_bwd_strided -- fa_bwd for strided operands, e.g. [B][N][H][d] tensors
 * viewed as (B, H, N, d).
 *
 *  strides : 24 int64 values, element strides (batch, head, sequence) of q,
 *            k, v, o, dout, dq, dk and dv in that order, with the rules of
 *            fa_fwd_strided (>= d, a multiple of 8 elements, below 2^39, the
 *            stride of a dimension of size 1 ignored).  The head dimension d
 *            is always contiguous.  Rows of dq, dk and dv must not overlap
 *            each other or any input.
 *  lse     : contiguous float [B][H][N] as in fa_bwd.
 * Other arguments, results and errors as fa_bwd; FA_ERR_INVALID_ARG also for
 * a NULL `strides`, and the stride errors of fa_fwd_strided.
 */
fa_status fa_bwd_strided(const void* q, const void* k, const void* v, const void* o,
                         const void* dout, const float* lse, void* dq, void* dk, void* dv, int B,
                         int H, int N, int d, const long long* strides, int causal, float scale,
                         void* workspace, size_t workspace_bytes, void* stream);

/*
 * fa_bwd_debug -- fa_bwd with the kernel watchdog exposed, for tests.
 *
 *  watchdog_ms : every wait inside the backward kernel gives up after this
 *                many milliseconds (0 = the default of 4000 ms), with the
 *                same recovery as fa_fwd_debug (status word, bounded drain of
 *                the CTA's own copies and MMAs, TMEM freed, context usable).
 *  inject      : 0 = normal run.  1 = the producer of the first CTA never
 *                issues its first Q / dO block, so the waits on it can only
 *                end by the watchdog (host-chosen; no fault is involved).
 * Other arguments and errors as fa_bwd.  dQ, dK, dV are undefined when the
 * watchdog fires.
 */
fa_status fa_bwd_debug(const void* q, const void* k, const void* v, const void* o,
                       const void* dout, const float* lse, void* dq, void* dk, void* dv, int B,
                       int H, int N, int d, int causal, float scale, void* workspace,
                       size_t workspace_bytes, void* stream, unsigned watchdog_ms, int inject);

/*
 * fa_fwd_debug -- fa_fwd with the kernel watchdog exposed, for tests.
 *
 *  watchdog_ms : every wait inside the kernel gives up after this many
 *                milliseconds (0 = the default of 4000 ms); the CTA then
 *                records FA_ERR_TIMEOUT in the device status word, stops
 *                issuing work, waits (bounded) for its own copies and
 *                tensor-core operations in flight, frees its tensor memory
 *                and exits.  The context stays usable.
 *  inject      : 0 = normal run.  1 = the producer of the first CTA never
 *                issues its first K-tile copy, so the consumer's wait can
 *                only end by the watchdog (host-chosen fault injection; no
 *                fault, trap or bad address is involved).
 * Other arguments and errors as fa_fwd.  O and LSE are undefined when the
 * watchdog fires.
 */
fa_status fa_fwd_debug(const void* q, const void* k, const void* v, void* o, float* lse,
                       int B, int H, int N, int d, int causal, float scale, void* stream,
                       unsigned watchdog_ms, int inject);

/*
 * fa_get_device_status -- read and clear the device status word of the
 * current device.  Synchronises `stream` first.  Returns FA_OK, or the
 * status a kernel recorded since the last read: FA_ERR_TIMEOUT (a watchdog
 * fired), or FA_ERR_LAUNCH (the d = 128 backward kernel found its dynamic
 * shared memory placed so that its 226 KiB layout did not fit, and returned
 * without writing dK or dV).  *detail, if not NULL, receives the raw word:
 * status << 24 | role << 20 | unit (or CTA) of the first event.
 * Returns FA_ERR_NO_DEVICE / FA_ERR_LAUNCH if the CUDA calls fail.
 *
 * The word is one per device (one for the forward kernels, one for the
 * backward kernels, reported together), not one per stream or call: a
 * timeout in a call on any stream is reported to, and cleared by, the next
 * reader on that device, whichever stream it synchronises.  Only the first
 * timeout since the last read is kept.  Callers that run several streams
 * and need to know which call timed out should synchronise all of them
 * before reading.
 */
fa_status fa_get_device_status(void* stream, unsigned* detail);

/* Human-readable name of a status code (static string, never NULL). */
const char* fa_status_string(int status);

/* cudaError_t value behind the last FA_ERR_LAUNCH / FA_ERR_NO_DEVICE in this thread. */
int fa_last_cuda_error(void);

/* Library version: major*10000 + minor*100 + patch. */
int fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_B200_H */
