/*
 * attn.h - C ABI of the B200 (sm_100a) exact softmax attention library
 * (libattn_b200.so): forward pass (device or host buffers), grouped-query and
 * block-local forms, backward pass, decode against rolling key/value caches.
 *
 * The operation (all entry points that compute):
 *
 *   O = softmax(scale * Q K^T) V,   row-wise softmax over the allowed keys,
 *   LSE_i = ln sum_{j allowed for i} exp(scale * q_i . k_j)
 *
 * Scaled dot-product attention is defined on "week17 efficiency attention"
 * (recall at the top of the page: softmax(Q K^T / sqrt(d_k)) V) and on
 * "Quadratic cost and efficient attention" (section "Where the n^2 hides").
 * It is computed tile by tile with an online softmax (running row maximum and
 * normaliser), as described under FlashAttention on "week17 efficiency
 * attention" and in "The online softmax trick" on "Efficient Transformers:
 * Sparse Attention, Linear Attention and FlashAttention"; the n x n score
 * matrix is never written to device memory (same page, "Family 3").
 *
 * Masks (key j allowed for query i):
 *   causal = 0, window < 0  : every j in [0, n)               (no mask)
 *   causal = 1, window < 0  : j <= i                          (causal; the triu
 *                              mask of naive_attention, "Family 3")
 *   causal = 1, window >= 0 : max(0, i - window) <= j <= i    (causal sliding
 *                              window; the window-mask snippet on "week17
 *                              efficiency attention", local attention section;
 *                              min(i, window) + 1 keys including i itself)
 *   causal = 0, window >= 0 : max(0, i - window) <= j <= min(n - 1, i + window)
 *                              (symmetric local window: each token attends to
 *                              its window nearest neighbours on either side;
 *                              local attention section of the same page)
 * A window of n - 1 or more allows the same keys as no window. The
 * block-local mask has entry points of its own (attn_fwd_blocklocal,
 * attn_bwd_blocklocal). A key the mask excludes gets a weight of exactly 0:
 * its values never reach O, whatever they are (finite).
 *
 * Layout: Q, K, V and O are bf16, contiguous [B, H, n, d] (token-major inside
 * each head, d fastest). LSE is fp32, contiguous [B, H, n], natural-log units.
 * Arithmetic: bf16 inputs, fp32 accumulation (QK^T and PV on the tensor
 * cores), fp32 softmax, P rounded to bf16 before PV, O rounded to bf16 (round
 * to nearest even).
 *
 * Ownership: the caller owns every buffer passed in and keeps it alive until
 * the work enqueued on `stream` has finished. The library owns only: one
 * lazily allocated device status word per device; for attn_fwd_host, a
 * per-device set of device staging buffers (grown on demand, released by
 * attn_host_staging_release) and two side streams with their events (created
 * once per device); for attn_fwd_host_noalloc, one static device array per
 * device. No entry point prints, exits, aborts or traps.
 *
 * Streams: `stream` is a cudaStream_t passed as void* (NULL = legacy default
 * stream). Work is enqueued on it on the calling thread's current device; the
 * device pointers must belong to that device. attn_fwd_host also runs copies
 * on its side streams, ordered with `stream` by events (see there).
 */
#ifndef ATTN_B200_H
#define ATTN_B200_H

#include <stddef.h>
#include <stdint.h>

/* Exported symbols of the shared library (everything else is hidden). */
#if defined(__GNUC__)
#define ATTN_API __attribute__((visibility("default")))
#else
#define ATTN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes returned by every entry point. */
typedef enum {
    ATTN_OK = 0,              /* success (for async calls: enqueued)            */
    ATTN_ERR_INVALID = 1,     /* a bad argument; nothing was enqueued           */
    ATTN_ERR_UNSUPPORTED = 2, /* valid but not provided (d not 64/128, ...)     */
    ATTN_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed              */
    ATTN_ERR_TIMEOUT = 4,     /* a kernel's bounded wait expired (device side)  */
    ATTN_ERR_TOO_LARGE = 5    /* exceeds the fixed scratch of attn_fwd_host_noalloc */
} attn_status;

/*
 * attn_fwd - enqueue the attention forward pass on device buffers.
 *
 *   q, k, v : device, bf16 [B, H, n, d], 16-byte aligned, read only
 *   o       : device, bf16 [B, H, n, d], 16-byte aligned, written
 *   lse     : device, fp32 [B, H, n], 4-byte aligned, written
 *   B, H, n : >= 1; B*H*n*d must fit in int64 and B*H < 2^31
 *   d       : head size; 64 or 128 (else ATTN_ERR_UNSUPPORTED)
 *   scale   : finite and > 0 (the pages' choice is 1/sqrt(d))
 *   causal, window : the mask, see the table above
 *   stream  : cudaStream_t as void*
 *
 * Returns ATTN_OK once the kernel is enqueued; ATTN_ERR_INVALID /
 * ATTN_ERR_UNSUPPORTED before touching the device; ATTN_ERR_CUDA if
 * encoding the TMA descriptors or the launch fails. A device-side timeout
 * is reported later by attn_sync_status. o and lse must not overlap q, k, v.
 */
ATTN_API int attn_fwd(const void *q, const void *k, const void *v, void *o, float *lse,
             int B, int H, int n, int d, float scale, int causal, int window,
             void *stream);

/*
 * attn_fwd_schedule - how the forward kernels (attn_fwd, attn_fwd_gqa,
 * attn_fwd_blocklocal and the host-buffer forms) spread their work over the
 * SMs; a process-wide setting for tuning and testing, read at each launch.
 *
 *   ATTN_SCHEDULE_AUTO       : by the mask and n (the default): the
 *                              persistent form when a query tile walks few
 *                              key tiles on average, else one CTA per item
 *   ATTN_SCHEDULE_PER_ITEM   : one CTA per work item (two 128-row query
 *                              tiles of one head)
 *   ATTN_SCHEDULE_PERSISTENT : one CTA per SM walking the work items
 *
 * Both forms compute the same result bit for bit (the same arithmetic per
 * tile in the same order). Returns the previous mode, or -1 (and changes
 * nothing) for an unknown mode. Not synchronised with launches in flight on
 * other threads: set it before enqueueing work.
 */
#define ATTN_SCHEDULE_AUTO 0
#define ATTN_SCHEDULE_PER_ITEM 1
#define ATTN_SCHEDULE_PERSISTENT 2
ATTN_API int attn_fwd_schedule(int mode);

/*
 * attn_fwd_schedule_for - the form the forward kernels would take for a
 * problem of n tokens with this mask under the current setting:
 * ATTN_SCHEDULE_PER_ITEM or ATTN_SCHEDULE_PERSISTENT (never AUTO); -1 for
 * n < 1. causal, window and block as for attn_fwd / attn_fwd_blocklocal
 * (block <= 0: no block mask). Reports only; launches nothing.
 */
ATTN_API int attn_fwd_schedule_for(int n, int causal, int window, int block);

/*
 * attn_fwd_gqa - grouped-query (and multi-query) attention on device buffers.
 *
 * Grouped-query attention ("week17 efficiency attention", MQA / GQA section):
 * G = Hkv groups of query heads share one key/value head; Hkv = 1 is
 * multi-query attention, Hkv = H is attn_fwd.
 *
 *   q, o    : device, bf16 [B, H, n, d]
 *   k, v    : device, bf16 [B, Hkv, n, d]
 *   lse     : device, fp32 [B, H, n]
 *   Hkv     : >= 1 and divides H (else ATTN_ERR_INVALID); query head h reads
 *             key/value head h / (H / Hkv)
 * Everything else (alignment, d, scale, masks, stream, errors) as attn_fwd.
 */
ATTN_API int attn_fwd_gqa(const void *q, const void *k, const void *v, void *o, float *lse,
                          int B, int H, int Hkv, int n, int d, float scale, int causal,
                          int window, void *stream);

/*
 * attn_fwd_blocklocal - the forward pass with the block-local mask: with
 * blocks of `block` consecutive tokens, query i attends to the keys of its
 * own block and of the previous one, floor(j/block) in {floor(i/block) - 1,
 * floor(i/block)}, and only to j <= i when causal = 1 (the block-sparse
 * pattern of "Sparse & sub-quadratic attention", section "Escape 1": a
 * token sees the keys of its own block and of the block before). A block of
 * n tokens or more is one block: the same keys as attn_fwd without a window.
 *
 *   block  : >= 1 (else ATTN_ERR_INVALID)
 *   Hkv    : key/value heads, as attn_fwd_gqa (Hkv = H for multi-head)
 * Everything else as attn_fwd_gqa.
 */
ATTN_API int attn_fwd_blocklocal(const void *q, const void *k, const void *v, void *o,
                                 float *lse, int B, int H, int Hkv, int n, int d, float scale,
                                 int causal, int block, void *stream);

/*
 * attn_fwd_host - the same operation on HOST buffers, copies included.
 *
 *   q, k, v : host, bf16 [B, H, n, d] (pinned memory makes the copies async)
 *   o, lse  : host, written (bf16 [B, H, n, d] and fp32 [B, H, n])
 *
 * Enqueues host-to-device copies of q, k, v into library-owned staging
 * buffers, attn_fwd, and device-to-host copies of o and lse. Problems of
 * 16 MB of inputs or more are cut into up to 8 chunks of heads and
 * pipelined: the copies run on two library-owned side streams (one per
 * direction) and the kernels on `stream`, so one chunk is copied in while
 * another is computed and a third is copied out. The side streams start
 * after the work already on `stream`, and `stream` waits for the last copy,
 * so the call is ordered on `stream` as a whole. The caller synchronizes
 * `stream` (or calls attn_sync_status) before reading o and lse. Staging
 * buffers and side streams are per device and shared by all calls: calls
 * on different streams of one device must not overlap. Returns as attn_fwd,
 * or ATTN_ERR_CUDA if growing the staging buffers or creating the side
 * streams fails.
 */
ATTN_API int attn_fwd_host(const void *q, const void *k, const void *v, void *o, float *lse,
                  int B, int H, int n, int d, float scale, int causal, int window,
                  void *stream);

/* Frees this device's attn_fwd_host staging buffers (synchronizes the device). */
ATTN_API int attn_host_staging_release(void);

/* Size of the fixed device scratch of attn_fwd_host_noalloc, per device. */
#define ATTN_NOALLOC_SCRATCH_BYTES (64u << 20)

/*
 * attn_fwd_host_noalloc - attn_fwd_host for callers that must not allocate
 * device memory. The pages have no counterpart to it: it exists for programs
 * that run under a fixed device-memory budget owned by someone else, or that
 * cannot afford the device-wide synchronisation cudaMalloc/cudaFree may
 * cause, and therefore cannot let a library allocate on their behalf.
 *
 * Same arguments and result as attn_fwd_host (host buffers in, host buffers
 * out), but every device-side scratch byte it uses (the staging copies of q,
 * k, v, o, lse and the kernel's status word) lives in one statically sized
 * device array of ATTN_NOALLOC_SCRATCH_BYTES that the library holds on every
 * device that loads it, until the process exits. It never calls cudaMalloc,
 * cudaFree or any allocating routine.
 *
 *   Limit: 4 * B*H*n*d*2 + B*H*n*4 bytes (each part rounded up to 256) plus
 *          256 must fit in ATTN_NOALLOC_SCRATCH_BYTES; larger problems return
 *          ATTN_ERR_TOO_LARGE before any device work.
 *   Synchronous: the call waits for its own copies and kernel to finish
 *          (it synchronizes `stream`) and returns once o and lse hold the
 *          result. ATTN_ERR_TIMEOUT if the kernel gave up a bounded wait,
 *          ATTN_ERR_CUDA if a kernel refused to run (the status word read
 *          as attn_sync_status reads it).
 *   Set-up: the first call on a device looks up the array's device address
 *          (cudaGetSymbolAddress) with that device current; make that first
 *          call before any stream capture.
 *   Sharing: all calls on a device use the same array, which keeps the last
 *          call's contents; calls whose work overlaps on the GPU (other
 *          streams or threads) race and must be serialised by the caller.
 */
ATTN_API int attn_fwd_host_noalloc(const void *q, const void *k, const void *v, void *o,
                                   float *lse, int B, int H, int n, int d, float scale,
                                   int causal, int window, void *stream);

/*
 * attn_bwd - enqueue the attention backward pass on device buffers.
 *
 * Gradients of a loss L with respect to Q, K and V given dO = dL/dO, for the
 * forward pass of attn_fwd with the same mask and scale. The attention
 * weights are recomputed from Q, K and the forward pass's LSE rather than
 * stored (the recompute in the backward pass named in "Efficient
 * Transformers: Sparse Attention, Linear Attention and FlashAttention",
 * section "Family 3"). With P_ij = exp(scale * q_i . k_j - LSE_i) on the
 * allowed pairs (0 elsewhere):
 *
 *   dV_j = sum_i P_ij dO_i
 *   dS_ij = P_ij (dO_i . v_j - dO_i . O_i)
 *   dQ_i = scale * sum_j dS_ij k_j,   dK_j = scale * sum_i dS_ij q_i
 *
 * (dO_i . O_i equals sum_j P_ij dO_i . v_j, the row term of the softmax
 * Jacobian.)
 *
 *   q, k, v, o, dout : device, bf16 [B, H, n, d], 16-byte aligned, read only;
 *                      o and lse are attn_fwd's outputs for q, k, v
 *   lse              : device, fp32 [B, H, n], 4-byte aligned, read only
 *   dq, dk, dv       : device, bf16 [B, H, n, d], 16-byte aligned, written
 *   workspace        : device scratch owned by the caller, 16-byte aligned,
 *                      at least attn_bwd_workspace_bytes(B, H, n, d) bytes
 *                      (two fp32 per-row arrays and, for d = 64, an fp32 dQ
 *                      accumulator of 4 * B*H*n*d bytes);
 *                      its contents on entry do not matter, and it must not
 *                      be used by other work until this call's work is done
 *   B, H, n, d, scale, causal, window, stream : as attn_fwd (K and V have H
 *                      heads; attn_bwd_gqa below is the grouped-query form)
 *
 * Arithmetic: bf16 tensor-core products with fp32 accumulation; P and dS
 * are rounded to bf16 before their products; all sums are fp32 and each
 * gradient is rounded to bf16 once. d = 128: three kernels (per-row terms;
 * dK and dV, one CTA per key tile; dQ, one CTA per query tile), results
 * identical from run to run. d = 64: three kernels (per-row terms and a
 * zeroed accumulator; one CTA per key tile computing dK, dV and adding its
 * dQ contributions into the fp32 accumulator by bulk reduce-adds, whose
 * order varies, so dQ's last bits may differ between runs; dQ conversion).
 * Returns as attn_fwd; ATTN_ERR_INVALID also for a short or misaligned
 * workspace. Outputs must not overlap inputs or the workspace.
 */
ATTN_API int attn_bwd(const void *q, const void *k, const void *v, const void *o,
                      const float *lse, const void *dout, void *dq, void *dk, void *dv,
                      void *workspace, size_t workspace_bytes, int B, int H, int n, int d,
                      float scale, int causal, int window, void *stream);

/*
 * attn_bwd_gqa - the backward pass of attn_fwd_gqa (grouped-query and
 * multi-query attention): K, V, dK and dV have Hkv heads, Hkv divides H,
 * query head h reads key/value head h / (H / Hkv), and the gradient of a
 * key/value head sums the contributions of every query head that reads it.
 *
 *   q, o, dout, dq : device, bf16 [B, H, n, d]
 *   k, v, dk, dv   : device, bf16 [B, Hkv, n, d]
 *   lse            : device, fp32 [B, H, n]
 *   workspace      : at least attn_bwd_workspace_bytes(B, H, n, d) bytes
 * Everything else as attn_bwd; Hkv < 1 or not dividing H gives
 * ATTN_ERR_INVALID.
 */
ATTN_API int attn_bwd_gqa(const void *q, const void *k, const void *v, const void *o,
                          const float *lse, const void *dout, void *dq, void *dk, void *dv,
                          void *workspace, size_t workspace_bytes, int B, int H, int Hkv, int n,
                          int d, float scale, int causal, int window, void *stream);

/*
 * attn_bwd_blocklocal - the backward pass of attn_fwd_blocklocal: arguments
 * as attn_bwd_gqa with the block-local mask of attn_fwd_blocklocal in place
 * of the window (block >= 1, else ATTN_ERR_INVALID).
 */
ATTN_API int attn_bwd_blocklocal(const void *q, const void *k, const void *v, const void *o,
                                 const float *lse, const void *dout, void *dq, void *dk,
                                 void *dv, void *workspace, size_t workspace_bytes, int B,
                                 int H, int Hkv, int n, int d, float scale, int causal,
                                 int block, void *stream);

/* Device workspace bytes attn_bwd (and attn_bwd_gqa, with the query head
 * count H) needs for this shape, or -1 if the shape is invalid or
 * unsupported. */
ATTN_API int64_t attn_bwd_workspace_bytes(int B, int H, int n, int d);

/*
 * attn_decode - one decode step against rolling key/value caches.
 *
 * Every sequence b has one new query token at position pos[b] (>= 0). Its
 * keys and values live in a rolling cache of W slots per key/value head:
 * position p is stored in slot p mod W, so after the current token's own
 * key and value have been written the cache holds positions
 * max(0, pos[b] - W + 1) .. pos[b] (the rolling buffer of the worked example
 * on "Beyond attention", section "For engineers -- Show the maths": a
 * 4,096-position cache serving n = 32,768). The query attends to exactly those positions:
 *
 *   O[b,h]   = softmax(scale * q[b,h] . k) v   over the cached positions,
 *   LSE[b,h] = ln sum exp(scale * q[b,h] . k)  (natural-log units),
 *
 * with key/value head h / (H / Hkv) (grouped-query attention; Hkv = H for
 * multi-head attention). This equals row pos[b] of attn_fwd with causal = 1
 * and window = W - 1 over the sequence that filled the cache.
 *
 *   q                : device, bf16 [B, H, d], 16-byte aligned
 *   k_cache, v_cache : device, bf16 [B, Hkv, W, d], 16-byte aligned, read only
 *   pos              : device, int32 [B], read by the kernel (so a step can be
 *                      enqueued without the host knowing the positions)
 *   o, lse           : device, bf16 [B, H, d] and fp32 [B, H], written
 *   workspace        : device scratch owned by the caller, 16-byte aligned,
 *                      at least attn_decode_workspace_bytes(...) bytes
 *                      (per-split partial results)
 *   H / Hkv          : 1 .. 16 (else ATTN_ERR_UNSUPPORTED); d: 64 or 128
 *   B * Hkv          : at most 65535
 *   scale, stream    : as attn_fwd
 *
 * A negative pos[b] is read as 0. Slots no cached position occupies yet
 * (slot >= pos[b] + 1 while pos[b] < W - 1) may hold any bits, NaN included:
 * they never reach the result. Arithmetic: tensor cores (bf16 products,
 * fp32 scores and accumulation, softmax weights rounded to bf16 for the
 * value product, as in attn_fwd); O is rounded to bf16. Two kernels are
 * enqueued: per (split of the slots, sequence, kv head) partial results,
 * then their log-sum-exp merge. Returns as attn_fwd.
 */
ATTN_API int attn_decode(const void *q, const void *k_cache, const void *v_cache, const int *pos,
                         void *o, float *lse, void *workspace, size_t workspace_bytes, int B,
                         int H, int Hkv, int W, int d, float scale, void *stream);

/* Device workspace bytes attn_decode needs, or -1 if the shape is invalid
 * or unsupported. */
ATTN_API int64_t attn_decode_workspace_bytes(int B, int H, int Hkv, int W, int d);

/*
 * attn_decode_multi - a decode step with a few new query tokens per sequence
 * (speculative decoding, chunked steps) against rolling key/value caches.
 *
 * Every sequence b has T new tokens at positions t_u = pos[b] - T + 1 + u,
 * u = 0 .. T-1 (pos[b], >= T - 1, is the last of them), and their keys and
 * values have already been written to the rolling cache of W slots
 * (position p in slot p mod W; the rolling buffer of "Beyond attention",
 * section "For engineers -- Show the maths"). Token u attends causally: to
 * the positions max(0, t_u - window) .. t_u of its sliding window (the
 * causal window-w mask of "week17 efficiency attention", local attention
 * section), so the T outputs are rows t_0 .. t_{T-1} of attn_fwd with
 * causal = 1 and window = `window` over the sequence that filled the cache:
 *
 *   O[b,h,u]   = softmax(scale * q[b,h,u] . k) v   over that window,
 *   LSE[b,h,u] = ln sum exp(scale * q[b,h,u] . k)  (natural-log units),
 *
 * with key/value head h / (H / Hkv). A W-slot cache still holds every
 * position of every token's window when window + T <= W; other windows give
 * ATTN_ERR_INVALID. attn_decode is the case T = 1, window = W - 1.
 *
 *   q                : device, bf16 [B, H, T, d], 16-byte aligned
 *   k_cache, v_cache : device, bf16 [B, Hkv, W, d], 16-byte aligned, read only
 *   pos              : device, int32 [B] (a value below T - 1 is read as T - 1)
 *   o, lse           : device, bf16 [B, H, T, d] and fp32 [B, H, T], written
 *   workspace        : device scratch owned by the caller, 16-byte aligned, at
 *                      least attn_decode_multi_workspace_bytes(...) bytes
 *   (H / Hkv) * T    : at most 16 (the query rows of one key/value head fill
 *                      one 16-wide MMA), else ATTN_ERR_UNSUPPORTED
 *   B, Hkv, d, scale, stream : as attn_decode
 *
 * The step reads every cached slot (W slots once the cache is full), also
 * those that only lie outside every token's window when window + T < W;
 * size the cache W = window + T to read no slot in vain. Slots no position
 * has reached yet may hold any bits, NaN included. Arithmetic, kernels and
 * return values as attn_decode.
 */
ATTN_API int attn_decode_multi(const void *q, const void *k_cache, const void *v_cache,
                               const int *pos, void *o, float *lse, void *workspace,
                               size_t workspace_bytes, int B, int H, int Hkv, int T, int W,
                               int window, int d, float scale, void *stream);

/* Device workspace bytes attn_decode_multi needs, or -1 if the arguments are
 * invalid or unsupported. */
ATTN_API int64_t attn_decode_multi_workspace_bytes(int B, int H, int Hkv, int T, int W, int window,
                                                   int d);

/*
 * attn_sync_status - synchronize `stream`, then read and clear this device's
 * status word. Returns ATTN_ERR_TIMEOUT if any kernel since the last call gave
 * up on a bounded wait (its outputs are then undefined), ATTN_ERR_CUDA if the
 * synchronization reported a CUDA error or a kernel found its shared memory
 * unusable and did no work, else ATTN_OK.
 */
ATTN_API int attn_sync_status(void *stream);

/* Static English text for a status code; never NULL. */
ATTN_API const char *attn_strerror(int status);

/* Number of attended (query, key) pairs in one head for the given mask;
 * 4*d FLOPs per pair is the unmasked FLOP count. Returns -1 on bad input. */
ATTN_API int64_t attn_attended_pairs(int64_t n, int causal, int64_t window);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_B200_H */
