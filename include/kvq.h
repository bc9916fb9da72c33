/*
 * kvq.h -- C ABI of the routed mixed-precision KV cache for NVIDIA B200 (sm_100a).
 *
 * The operations come from "TriRoute: Unified Learned Routing for Joint Adaptive
 * Attention, Experts, and KV-Cache Allocation" (paper review page, section 3):
 *   - Eq. 4 (KV-cache bit-width, asymmetric per-token group quantization): each
 *     token's K and V are written at a width b in {2, 4, 8, 16}; for b < 16,
 *     s = (max - min) / (2^b - 1), z = min, code = round((x - z) / s); b = 16 keeps
 *     native fp16. The group is one (token, head) vector of head_dim values, and one b
 *     covers a token's K and V (the equation quantizes the pair (k_t, v_t) together).
 *   - Eq. 2 (attention resolution): each (token, head) query has a mode
 *     skip -> 0, local-w -> attention over keys [t - w, t], full -> keys [0, t].
 *   - Inference paragraph after Algorithm 1: the router takes the hard argmax of its
 *     logits (Eq. 5's attention and bit heads: kvq_route_argmax), skipped attention is
 *     never materialised, and each token's KV is stored at its chosen width.
 *   - Experimental setup, model table: KV heads shared by groups of query heads
 *     (kvq_cache_create_gqa).
 *
 * Conventions shared by every entry point:
 *   - All tensor arguments are DEVICE pointers owned by the caller, except where marked
 *     host. Element types: fp16 = IEEE binary16 (2 bytes), fp32 output.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy default
 *     stream) and never synchronize, except kvq_check().
 *   - Return value: KVQ_OK, or a kvq_status code for errors detectable on the host
 *     (null pointer, bad size, bad w, unsupported head_dim, CUDA launch failure); in that
 *     case nothing was launched and kvq_last_error() describes the problem.
 *   - Values that only the device sees (a bits entry outside {2,4,8,16}, a mode outside
 *     {0,1,2}, a write that would exceed a sequence's capacity, cu_seqlens that are not
 *     non-decreasing) never fault: the kernel skips the offending work, records the
 *     error in the cache's device status word, and kvq_check() reports it.
 *   - Calls that touch one cache must be ordered (same stream, or events); the cache
 *     holds per-call scratch, so two calls on one cache that overlap on the GPU race.
 */
#ifndef KVQ_H
#define KVQ_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t, declared without the CUDA headers. */
typedef struct CUstream_st *kvq_stream_t;

/* Opaque cache handle; owned by the library (kvq_cache_create / kvq_cache_destroy). */
typedef struct kvq_cache kvq_cache;

typedef enum kvq_status {
    KVQ_OK = 0,
    KVQ_ERR_ARG = 1,          /* bad pointer, size, w or head_dim (host check) */
    KVQ_ERR_BITS = 2,         /* a bits entry outside {2, 4, 8, 16} (device check) */
    KVQ_ERR_MODE = 3,         /* a mode entry outside {0, 1, 2} (device check) */
    KVQ_ERR_CAPACITY = 4,     /* a write past a sequence's capacity (device check) */
    KVQ_ERR_CUDA = 5,         /* a CUDA runtime call or launch failed */
    KVQ_ERR_DEVICE_CHECK = 6, /* any other device-side consistency check */
    KVQ_ERR_NOMEM = 7         /* device allocation failed (create only) */
} kvq_status;

/* Query modes of Eq. 2. */
enum { KVQ_MODE_SKIP = 0, KVQ_MODE_LOCAL = 1, KVQ_MODE_FULL = 2 };

/*
 * Create an empty cache for `batch` sequences of `heads` KV heads, head_dim in {64, 128}.
 * capacity_tokens: HOST array [batch], the most tokens each sequence may ever hold
 * (1 <= capacity <= 8388607). Device memory is allocated once here, at the worst case
 * of b = 16 for every token (4 * head_dim bytes of records + 16 bytes of fp32 side
 * entry + 4 bytes of record offset per (token, head)), plus the decode scheduler's work
 * list and split-K partials. All lengths start at 0. `stream` orders the initialisation.
 * On success *out receives the handle; on failure *out is NULL.
 */
int kvq_cache_create(kvq_cache **out, int batch, int heads, int head_dim,
                     const int64_t *capacity_tokens, kvq_stream_t stream);

/*
 * Grouped-query attention variant of kvq_cache_create (the pages' models share each KV
 * head among a group of query heads; model table, H_kv = H/4). `heads` is the number of KV
 * heads, which is what kvq_write stores (k, v, bits are [n_tok][heads]...). The attention
 * calls on this cache take heads * query_group query heads: q, modes and out are
 * [..][heads * query_group][..], and query head hq reads KV head hq / query_group with its
 * own mode. query_group = 1 is kvq_cache_create. 1 <= query_group <= 64.
 */
int kvq_cache_create_gqa(kvq_cache **out, int batch, int heads, int query_group, int head_dim,
                         const int64_t *capacity_tokens, kvq_stream_t stream);

/*
 * Paged variant of kvq_cache_create_gqa (the pages' inference procedure says the routed
 * cache works with KV paging; their limitations section notes that variable-width records
 * complicate it). The record bytes live in a pool of pool_pages pages of page_bytes bytes
 * each (a power of two in [4 KiB, 2 MiB]) instead of a worst-case stream per (sequence,
 * head): pool memory can be sized for the expected average width. Each (sequence, KV head)
 * stream is a list of logical pages; a write takes physical pages from the pool when its
 * records first reach a logical page (in a scrambled pool order, so pages of different
 * streams interleave), and a stream keeps its pages until kvq_cache_reset returns all of
 * them. Records are packed back to back in the logical stream as in a contiguous cache
 * and may straddle two pages; every call reads and writes through the page table.
 * Offsets, side entries and capacities are as in kvq_cache_create_gqa (capacity_tokens
 * bounds each sequence's tokens; the record offsets and side table stay per token).
 * A write that would need more pages than the pool has left is refused for that head with
 * KVQ_ERR_CAPACITY (device check), like a capacity overflow. page_bytes = 0 creates a
 * contiguous cache (pool_pages ignored).
 */
int kvq_cache_create_paged(kvq_cache **out, int batch, int heads, int query_group, int head_dim,
                           const int64_t *capacity_tokens, int64_t page_bytes, int64_t pool_pages,
                           kvq_stream_t stream);

/* Free every device buffer of the cache (synchronizes the device first). NULL is a no-op. */
int kvq_cache_destroy(kvq_cache *cache);

/* Set every sequence's length to 0 and clear the device status word; a paged cache's
   pages all go back to its pool. */
int kvq_cache_reset(kvq_cache *cache, kvq_stream_t stream);

/*
 * Roll sequences back: lengths is a DEVICE int32 array [batch]; sequence s keeps its
 * first min(lengths[s], current length) tokens (a negative entry keeps the sequence
 * unchanged). The dropped tokens' records are overwritten by later writes.
 */
int kvq_cache_truncate(kvq_cache *cache, const int32_t *lengths, kvq_stream_t stream);

/* Copy the current lengths into a DEVICE int32 array [batch]. */
int kvq_cache_lengths(const kvq_cache *cache, int32_t *lengths, kvq_stream_t stream);

/*
 * Quantize-on-write (Eq. 4): append n_tok tokens to the cache.
 *   k, v:        fp16 [n_tok][heads][head_dim], tokens of sequence s are rows
 *                cu_seqlens[s] .. cu_seqlens[s+1]-1 (ragged, packed).
 *   bits:        uint8 [n_tok][heads], each in {2, 4, 8, 16}; one width covers the
 *                token's K and V for that head.
 *   cu_seqlens:  int32 [batch + 1], cu_seqlens[0] = 0, non-decreasing,
 *                cu_seqlens[batch] = n_tok. Sequence s gets cu_seqlens[s+1]-cu_seqlens[s]
 *                new tokens (possibly 0) appended after its current length.
 *   n_tok:       host int, rows of k / v / bits (0 is a no-op).
 * Per (token, head) and for each of K and V: mn/mx are the fp32 min/max of the
 * head_dim values, s = fp32(mx - mn) / fp32(2^b - 1) (IEEE round-to-nearest-even),
 * z = mn, code_i = rint(fp32(x_i - z) / s) clamped to [0, 2^b - 1], code 0 when s == 0.
 * The codes are stored packed (code of channel c at bits [b*c, b*c + b) of the record
 * part), (s, z) go to the fp32 side table; b = 16 stores the fp16 bits and side (1, 0).
 * A sequence whose write would exceed its capacity is left unchanged (status
 * KVQ_ERR_CAPACITY); an invalid bits entry rejects its sequence's whole write, for
 * every head (status KVQ_ERR_BITS).
 */
int kvq_write(const void *k, const void *v, const uint8_t *bits, const int32_t *cu_seqlens,
              int64_t n_tok, kvq_cache *cache, kvq_stream_t stream);

/*
 * Routed causal prefill attention (Eq. 2) for tokens already written by kvq_write.
 *   q:           fp16 [n_tok][heads][head_dim]; query i of sequence s (row
 *                cu_seqlens[s] + i) sits at position t = len_s - n_s + i, where len_s is the
 *                sequence's current length and n_s = cu_seqlens[s+1] - cu_seqlens[s]
 *                (so: call kvq_write for the same tokens first).
 *   modes:       uint8 [n_tok][heads], 0 skip, 1 local-w, 2 full.
 *   w:           local window, >= 0; local reads keys max(0, t - w) .. t inclusive.
 *   cu_seqlens:  int32 [batch + 1], as for kvq_write; n_tok host int.
 *   out:         fp32 [n_tok][heads][head_dim]; skip rows are written as zeros.
 * Logits are q . deq(k_j) / sqrt(head_dim); softmax over the mode's key set; the output
 * is sum_j p_j deq(v_j), with deq = code * s + z (b = 16: the fp16 value).
 */
int routed_attn_prefill(const void *q, const kvq_cache *cache, const uint8_t *modes, int w,
                        const int32_t *cu_seqlens, int64_t n_tok, float *out,
                        kvq_stream_t stream);

/*
 * Routed decode attention (Eq. 2), one query per (sequence, head) at t = len_s - 1.
 *   q:      fp16 [batch][heads][head_dim];  modes: uint8 [batch][heads];  w >= 0.
 *   out:    fp32 [batch][heads][head_dim]; skip heads and empty sequences are zeros.
 * Work is split over key chunks (split-K) by an on-device scheduler that drops skip
 * heads and clamps local heads to their w + 1 keys, then merged by log-sum-exp.
 */
int routed_attn_decode(const void *q, const kvq_cache *cache, const uint8_t *modes, int w,
                       float *out, kvq_stream_t stream);

/*
 * One decode step in three launches: the step's tokens are written (Eq. 4) and then every
 * query attends over the cache that holds them (Eq. 2), the per-layer order of the
 * inference procedure after Algorithm 1 (attention in the routed mode, KV stored at the
 * routed width). Same results as kvq_cache_truncate (when positions is given), kvq_write
 * and routed_attn_decode called in turn.
 *   q, modes, w, out:           as routed_attn_decode.
 *   k, v, bits, cu_seqlens, n_tok: as kvq_write (one token per sequence in a decode step;
 *                               any n_tok is accepted, appended by one CTA per sequence).
 *   positions:                  DEVICE int32 [batch] or NULL. When given, sequence s first
 *                               keeps only its first min(len, positions[s]) tokens (a
 *                               negative entry keeps it whole), then its tokens are appended:
 *                               re-decoding a position, as after a rejected speculation.
 */
int kvq_decode_step(const void *q, const void *k, const void *v, const uint8_t *bits,
                    const int32_t *cu_seqlens, int64_t n_tok, const int32_t *positions,
                    const uint8_t *modes, int w, kvq_cache *cache, float *out, kvq_stream_t stream);

/*
 * Allocation-free variant of routed_attn_decode (no counterpart in the paper).
 * Same arguments, same arithmetic and the same kernels, but the per-call scratch (the
 * scheduler's work list and the split-K partials) lives in a 16 MiB array in the library's
 * static device memory instead of the cache's workspace, and the call allocates nothing:
 * no cudaMalloc or cudaFree. It is meant for callers that cannot allocate device memory at
 * the point of the call: code whose allocations are owned by a host framework's own pool,
 * code that must not trigger the implicit synchronization of an allocation, or code
 * running where allocation is not permitted.
 *   - Every GPU that loads the library holds the 16 MiB array until the process exits.
 *   - The first call on a device looks up the array's device address (cudaGetSymbolAddress)
 *     with that device current; make that first call before any stream capture.
 *   - All calls share the one array and it keeps the last call's contents (nothing in it
 *     needs clearing: each call rewrites its work list). Calls that overlap on the GPU, from
 *     any stream or thread, race on it: order them.
 *   - A cache whose worst case (every head full at capacity) needs more scratch than the
 *     array holds is rejected with KVQ_ERR_ARG before anything is launched; use
 *     routed_attn_decode for it.
 */
int routed_attn_decode_noalloc(const void *q, const kvq_cache *cache, const uint8_t *modes, int w,
                               float *out, kvq_stream_t stream);

/*
 * Read back stored records of one (sequence, head) for tokens first .. first+count-1
 * (all below the current length; checked on the device).
 *   k_codes, v_codes: uint16 [count][head_dim]: codes (b < 16) or raw fp16 bits (b = 16).
 *   side:             fp32 [count][4] = (s_K, z_K, s_V, z_V).
 *   bits:             uint8 [count].
 * Any of the four may be NULL. Used to verify the stored bytes; not on the hot path.
 */
int kvq_cache_export(const kvq_cache *cache, int seq, int head, int64_t first, int64_t count,
                     uint16_t *k_codes, uint16_t *v_codes, float *side, uint8_t *bits,
                     kvq_stream_t stream);

/*
 * Synchronize `stream`, read the cache's device status word and clear it.
 * Returns KVQ_OK or the first device-side error recorded since the last check.
 */
int kvq_check(kvq_cache *cache, kvq_stream_t stream);

/*
 * Profiling hook for benchmarks. With non-NULL `before` / `after` (each a cudaEvent_t
 * created by the caller), every following kvq_write, routed_attn_decode and
 * routed_attn_prefill call records `before` on its stream immediately before its main
 * kernel and `after` immediately after it (kvq_write: the quantize kernel; decode: the
 * split-K kernel; prefill: the attention kernel), so the pair times that kernel alone.
 * NULL, NULL turns recording off. Process-wide and not thread-safe.
 */
int kvq_set_profile_events(void *before, void *after);

/*
 * Router hard argmax at inference (section 3 item 5, Eq. 5: the controller's attention head
 * z^a and bit head z^b; the inference paragraph: the router takes the hard argmax and each
 * token's KV is stored at its chosen width). For n rows, one per (token, head):
 *   z_attn: fp32 [n][3] logits over (skip, local, full) -> modes: uint8 [n] in {0, 1, 2};
 *   z_bits: fp32 [n][4] logits over the widths (2, 4, 8, 16) -> bits: uint8 [n] in
 *           {2, 4, 8, 16}.
 * The first index wins a tie; NaN entries are passed over, and an all-NaN row gives
 * index 0. Either pair (z_attn, modes) or (z_bits, bits) may be NULL, not both. All four
 * are DEVICE pointers: z_attn and z_bits 16-byte aligned, modes and bits 4-byte aligned.
 * The outputs are the `bits` of kvq_write and the `modes` of routed_attn_prefill /
 * routed_attn_decode (laid out [n_tok][heads] or [batch][heads]).
 */
int kvq_route_argmax(const float *z_attn, const float *z_bits, int64_t n, uint8_t *modes,
                     uint8_t *bits, kvq_stream_t stream);

/*
 * Testing hooks for the failure paths (no counterpart in the paper). Neither faults,
 * traps or hangs the GPU; both exist so that tests can drive an error path on demand.
 *
 * kvq_test_fail_alloc: the nth device allocation (1-based) made by the next
 * kvq_cache_create / kvq_cache_create_gqa call is reported as failed, as if cudaMalloc had
 * returned an error. That create then frees what it had allocated, leaves *out NULL and
 * returns KVQ_ERR_NOMEM. nth = 0 turns a pending injection off. Process-wide; consumed
 * by the next create call whether or not it reaches the nth allocation.
 */
int kvq_test_fail_alloc(int nth);

/*
 * kvq_test_bounded_wait: launch on `stream` a one-thread kernel that waits, with the same
 * bounded mbarrier wait the kernels of this library use, on a barrier that no thread ever
 * completes. After limit_ns nanoseconds (1e3 <= limit_ns <= 1e8) the wait gives up,
 * records KVQ_ERR_DEVICE_CHECK in the cache's device status word and the kernel returns;
 * kvq_check() then reports it. The CUDA context stays usable.
 */
int kvq_test_bounded_wait(kvq_cache *cache, int64_t limit_ns, kvq_stream_t stream);

/* Text of the last host-side error on this thread ("" if none). */
const char *kvq_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_H */
