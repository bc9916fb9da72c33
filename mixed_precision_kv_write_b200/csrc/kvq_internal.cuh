// Internal definitions of the routed mixed-precision KV cache (B200, sm_100a).
//
// Cache layout in HBM (per sequence s, head h, token j; "slot" = one (s, h, j)):
//   records  one byte stream per (s, h), tokens in order; token j's record is
//            [K part | V part], each part b*D/8 bytes: for b < 16 the codes are packed
//            LSB-first (channel c occupies bits [b*c, b*c + b) of the part), for b = 16
//            the part is the fp16 vector. Record size b*D/4 bytes, a multiple of 16.
//            Stream (s, h) starts at byte slot(s, h, 0) * 4 * D, room for the worst case.
//   meta     uint32 per slot: byte offset of the record inside its stream (a multiple of
//            16) OR'ed with the width code (0, 1, 2, 3 for b = 2, 4, 8, 16).
//   side     float4 per slot: (s_K, z_K, s_V, z_V) of Eq. 4; (1, 0, 1, 0) for b = 16.
//   len/end  per (s, h): tokens held and the stream's end offset in bytes.
// Slots: slot(s, h, j) = slot_base[s] + h * cap_pad[s] + j, cap_pad a multiple of 4 that
// leaves at least one spare slot, so 16-byte bulk copies of meta may round to 4 slots.
// Record bytes, contiguous cache: stream (s, h) starts at byte slot(s, h, 0) * 4 * D of
// `rec`, with room for the worst case. Paged cache: `rec` is a pool of fixed-size pages
// (2^page_shift bytes); stream (s, h) is a sequence of logical pages, logical page lp at
// physical page ptab[(s * H + h) * max_lpages + lp]. Pages are taken from the pool when a
// write first reaches them (pool_list[pool_next ..], in the order the pool hands them
// out) and stay with (s, h) until kvq_cache_reset. Offsets inside a stream are the same in
// both layouts; a record may straddle two pages (every 16-byte chunk lies in one page).
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "kvq.h"

namespace kvq {

struct CacheView {
    int B, H, D;
    int G;                    // query heads per KV head (grouped-query attention); 1 = MHA
    const int32_t *cap;       // [B] capacity in tokens
    const int32_t *cap_pad;   // [B] slots per (s, h)
    const int64_t *slot_base; // [B] first slot of sequence s
    uint8_t *rec;             // record bytes
    uint32_t *meta;           // [slots]
    float4 *side;             // [slots]
    int32_t *len;             // [B*H]
    uint32_t *end;            // [B*H]
    int32_t *wstart;          // [B*H] start position of the current write, -1 = rejected
    uint32_t *wend;           // [B*H] stream end after the current write
    uint32_t *bad;            // [B] id of the last write call that saw a bad width
    int32_t *status;          // [1] first device-side error (kvq_status), 0 = none
    // paged record storage (ptab == nullptr: contiguous streams)
    uint32_t *ptab;           // [B*H][max_lpages] physical page of each logical page
    int32_t *npages;          // [B*H] logical pages mapped
    int32_t *pool_next;       // [1] pages handed out since the last reset
    const uint32_t *pool_list;// [pool_pages] the order in which the pool hands out pages
    int32_t max_lpages, pool_pages;
    uint32_t page_shift;      // log2 of the page size (31 for contiguous caches)
};

__device__ __forceinline__ int64_t slot_of(const CacheView &c, int s, int h, int64_t j)
{
    return c.slot_base[s] + (int64_t)h * c.cap_pad[s] + j;
}

__device__ __forceinline__ uint8_t *stream_of(const CacheView &c, int s, int h)
{
    return c.rec + slot_of(c, s, h, 0) * (int64_t)(4 * c.D);
}

// Locator of record bytes of one stream: at(rel) is the address of logical byte off + rel.
// A chunk of up to 16 bytes at a 16-byte aligned logical offset never straddles a page.
struct RecLoc {
    uint8_t *base;            // contiguous: stream + off; paged: the pool
    const uint32_t *pt;       // paged: the stream's page table row; contiguous: nullptr
    uint32_t off, shift;
    __device__ __forceinline__ uint8_t *at(uint32_t rel) const
    {
        if (!pt) return base + rel;
        const uint32_t o = off + rel;
        return base + ((size_t)pt[o >> shift] << shift) + (o & ((1u << shift) - 1u));
    }
};

__device__ __forceinline__ RecLoc rec_loc(const CacheView &c, int s, int h, uint32_t off)
{
    RecLoc r;
    if (c.ptab) {
        r.base = c.rec;
        r.pt = c.ptab + (size_t)(s * c.H + h) * c.max_lpages;
        r.off = off;
        r.shift = c.page_shift;
    } else {
        r.base = stream_of(c, s, h) + off;
        r.pt = nullptr;
        r.off = 0;
        r.shift = 0;
    }
    return r;
}

// Paged caches: give (s, h) physical pages for every logical page that a stream end of
// end_bytes reaches (one thread per (s, h)). Returns false, mapping nothing, when the
// pool has too few pages left. Contiguous caches: always true.
__device__ __forceinline__ bool map_pages(const CacheView &c, int s, int h, uint32_t end_bytes)
{
    if (!c.ptab) return true;
    const int sh = s * c.H + h;
    const int need = (int)(((uint64_t)end_bytes + (1u << c.page_shift) - 1u) >> c.page_shift);
    const int have = c.npages[sh];
    if (need <= have) return true;
    if (need > c.max_lpages) return false;
    const int k = need - have;
    int old = *reinterpret_cast<volatile int32_t *>(c.pool_next);
    while (true) {
        if (old + k > c.pool_pages) return false;
        const int prev = atomicCAS(c.pool_next, old, old + k);
        if (prev == old) break;
        old = prev;
    }
    uint32_t *pt = c.ptab + (size_t)sh * c.max_lpages;
    for (int i = 0; i < k; ++i) pt[have + i] = c.pool_list[old + i];
    c.npages[sh] = need;
    return true;
}

constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ int width_code(int bits)
{
    return bits == 2 ? 0 : bits == 4 ? 1 : bits == 8 ? 2 : bits == 16 ? 3 : -1;
}

__device__ __forceinline__ void set_status(int32_t *status, int code)
{
    atomicCAS(status, 0, code);
}

// ---- scheduler work list (decode) ----------------------------------------------------
#ifndef KVQ_DECODE_ITEM_KEYS
#define KVQ_DECODE_ITEM_KEYS 1152
#endif
constexpr int kDecodeItemKeys = KVQ_DECODE_ITEM_KEYS;   // keys per split-K work item, at most (w + 1 = 513 fits one)
constexpr int kDecodeWindowKeys = 128; // keys per window of record offsets inside an item
constexpr int kDecodeMaxQ = 4;         // query heads served by one item (a subgroup of a GQA group)
constexpr int kDecodeCountWords = 7;   // decode count words: front pair, item cursor, back pair, middle pair

struct __align__(16) DecodeItem {
    int32_t sh, j0, j1;  // (sequence, KV head) = s * H + hk, and key range [j0, j1)
    uint32_t end_off;    // byte offset of key j1 in the stream (the stream end if j1 = len)
    int64_t sbase;       // slot of key 0 of (sequence, KV head)
    int32_t qinfo;       // first query g0 of the subgroup | active-query mask << 8 (bit i: g0 + i)
    int32_t role;        // front items: pair role (kSolo, kPairHead, kPairTail); 0 otherwise
};

struct DecodeWork {
    DecodeItem *items;   // [max_items]
    // The list has three regions. [0, mid_base) holds the front items, filled from the
    // start, and the back items (the local window's keys), filled from the end (back item x
    // sits at mid_base - 1 - x); [mid_base, max_items) holds the middle items (the last
    // piece of each range outside the window). The split-K CTAs claim front, middle, then
    // back items, so the long items come first and the short ones last.
    // Item counts, a pair of words per region, used by calls of alternating generation
    // parity: a call of generation g reserves its items with atomicAdd on `count`,
    // `count_back` and `count_mid` (g << 32 | items; a word still tagged 0 has never been
    // used) and prepares the `_next` words, those of call g + 1, as (g + 1) << 32. A word
    // with any other tag is stale: the call lists nothing and reports KVQ_ERR_DEVICE_CHECK.
    unsigned long long *count;
    unsigned long long *count_next;
    unsigned long long *count_back;
    unsigned long long *count_back_next;
    unsigned long long *count_mid;
    unsigned long long *count_mid_next;
    uint32_t *cursor;    // items claimed so far by the split-K CTAs (reset by the planning kernel)
    uint32_t gen;        // the call's generation
    // [3 * B*H]: entry r * B*H + s * H + hk, the first item of (sequence, KV head) in region
    // r (0 front, 1 back, 2 middle) and their number (all subgroups): the run
    // [first, first + cnt) of item indices
    int32_t *head_first;
    int32_t *head_cnt;
    float *partials;     // [max_items][qslots][D + 4]: (m, l, -, -, o[D])
    int64_t max_items;
    int64_t mid_base;    // first index of the middle region
    int qslots;          // min(G, kDecodeMaxQ)
};

// Upper bound of the front and back items a decode call lists for a cache: per (sequence,
// KV head) and subgroup of at most kDecodeMaxQ query heads, ceil(cap / kDecodeItemKeys) + 1
// (the key range may be cut once where the local window starts).
inline int64_t decode_max_items(int64_t cap, int G)
{
    return (int64_t)((G + kDecodeMaxQ - 1) / kDecodeMaxQ) * ((cap + kDecodeItemKeys - 1) / kDecodeItemKeys + 1);
}

// Middle items per (sequence, KV head): at most one per subgroup.
inline int64_t decode_mid_items(int G) { return (G + kDecodeMaxQ - 1) / kDecodeMaxQ; }

// ---- PTX helpers -----------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ uint64_t global_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Wait until the barrier's phase `parity` has completed. Each try_wait lets the hardware
// hold the thread for a short, implementation-defined time; a suspend-time hint
// (KVQ_WAIT_HINT_NS > 0) would let it sleep longer but measured slower wake-ups on B200
// (prefill and decode), so the default passes none. Bounded: gives up after `limit_ns`
// (about two seconds by default), records KVQ_ERR_DEVICE_CHECK and returns false, so a
// logic error ends the kernel with a status instead of hanging the GPU.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

#ifndef KVQ_WAIT_HINT_NS
#define KVQ_WAIT_HINT_NS 0
#endif
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, int32_t *status,
                                          uint64_t limit_ns = kWaitLimitNs)
{
    const uint32_t addr = smem_u32(bar);
    uint32_t done = 0;
    uint64_t t0 = 0;
    for (uint32_t it = 0;; ++it) {
#if KVQ_WAIT_HINT_NS > 0
        asm volatile("{\n\t.reg .pred p;\n\t"
                     "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
                     "selp.u32 %0, 1, 0, p;\n\t}"
                     : "=r"(done)
                     : "r"(addr), "r"(parity), "r"((uint32_t)KVQ_WAIT_HINT_NS)
                     : "memory");
#else
        asm volatile("{\n\t.reg .pred p;\n\t"
                     "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                     "selp.u32 %0, 1, 0, p;\n\t}"
                     : "=r"(done)
                     : "r"(addr), "r"(parity)
                     : "memory");
#endif
        if (done) return true;
        if ((it & 15u) == 0) {
            const uint64_t t = global_ns();
            if (t0 == 0) t0 = t;
            else if (t - t0 > limit_ns) {
                set_status(status, KVQ_ERR_DEVICE_CHECK);
                return false;
            }
        }
    }
}

// Non-blocking test of a barrier phase (no suspension).
__device__ __forceinline__ bool mbar_test(uint64_t *bar, uint32_t parity)
{
    uint32_t done;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(done)
                 : "r"(smem_u32(bar)), "r"(parity)
                 : "memory");
    return done != 0;
}

// 1-D bulk copy global -> shared (TMA engine), completion counted on `bar` in bytes.
// dst, src 16-byte aligned, bytes a multiple of 16. No multicast.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void named_bar_sync(int id, int threads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Named barrier that also ORs a predicate over the participating threads.
__device__ __forceinline__ bool named_bar_or(int id, int threads, bool pred)
{
    uint32_t r;
    asm volatile("{\n\t.reg .pred p, q;\n\t"
                 "setp.ne.u32 p, %1, 0;\n\t"
                 "bar.red.or.pred q, %2, %3, p;\n\t"
                 "selp.u32 %0, 1, 0, q;\n\t}"
                 : "=r"(r)
                 : "r"((uint32_t)pred), "r"(id), "r"(threads)
                 : "memory");
    return r != 0;
}

// Programmatic dependent launch. A kernel launched with launch_pdl may start while the
// previous kernel of the stream is still running; pdl_wait() blocks until that kernel has
// completed and its memory is visible, so it comes before any access to data another
// kernel of the stream produces or consumes. pdl_trigger() lets the next kernel of the
// stream be scheduled early (its own pdl_wait() still waits for this kernel to finish).
// Both are no-ops for a kernel launched without the attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args &&...args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

} // namespace kvq

// ---- launchers (implemented per kernel file, called by the C ABI) --------------------
struct kvq_cache {
    int B, H, D;
    int device;
    int64_t total_slots;
    int32_t max_cap;
    kvq::CacheView view;
    kvq::DecodeWork work;
    uint32_t write_gen;       // id of the last kvq_write call
    uint32_t decode_gen;      // id of the last decode call on the cache's own work list
    bool work_stale;          // a decode launch failed: the count words are cleared before the next call
    uint64_t *scan_flags;     // [B*H*scan_chunks]: the long write scan's per-chunk look-back words
    int scan_chunks;          // chunks of 1024 tokens in the largest capacity
    void *pf_tiles;           // prefill tile lists (PfTile = 8 x int32): as listed, then ordered
    int32_t *pf_count;        // [1]
    int32_t *pf_qidx;         // [total_slots] per-(sequence, head) query lists
    int64_t pf_max_tiles;
    int64_t page_bytes;       // 0: contiguous streams
    void *allocs[32];
    int n_allocs;
};

namespace kvq {
cudaError_t launch_route_argmax(const float *za, const float *zb, int64_t n, uint8_t *modes,
                                uint8_t *bits, cudaStream_t st);
cudaError_t launch_write(kvq_cache *c, const __half *k, const __half *v, const uint8_t *bits,
                         const int32_t *cu, int64_t n_tok, cudaStream_t st);
cudaError_t launch_decode(const kvq_cache *c, const __half *q, const uint8_t *modes, int w,
                          float *out, cudaStream_t st);
// one decode step: append the step's tokens (optionally after rolling sequences back to
// `positions`), then decode, in three launches
cudaError_t launch_decode_step(kvq_cache *c, const __half *q, const __half *k, const __half *v,
                               const uint8_t *bits, const int32_t *cu, int64_t n_tok,
                               const int32_t *positions, const uint8_t *modes, int w, float *out,
                               cudaStream_t st);
cudaError_t launch_prefill_tc(const kvq_cache *c, const __half *q, const uint8_t *modes, int w,
                              const int32_t *cu, int64_t n_tok, float *out, cudaStream_t st);
// SM count of the current device (cached per device ordinal)
int num_sms();
// Raise `func`'s dynamic shared-memory limit to `bytes` on the current device; done once
// per (kernel, device), thread-safe.
cudaError_t ensure_smem_attr(const void *func, size_t bytes);
// records a host-side status for kvq_last_error() and returns `code`
int report_error(int code, const char *msg);
// profiling hook (kvq_set_profile_events): record the caller's events around a main kernel
void profile_before(cudaStream_t st);
void profile_after(cudaStream_t st);
} // namespace kvq
