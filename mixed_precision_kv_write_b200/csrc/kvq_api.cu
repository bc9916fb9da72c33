// C ABI of the routed mixed-precision KV cache: argument checks, cache allocation,
// small maintenance kernels (reset, truncate, lengths, export) and the status word.
// The hot-path kernels live in kvq_write.cu, kvq_decode.cu, kvq_prefill_tc.cu and
// kvq_route.cu. Every compute entry point is an NVTX range (named after the call) for
// timeline tools; without a tool attached a range costs a few nanoseconds.
#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <atomic>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "kvq_internal.cuh"

namespace {

struct ApiRange {                 // NVTX range around one API call
    explicit ApiRange(const char *name) { nvtxRangePushA(name); }
    ~ApiRange() { nvtxRangePop(); }
};

thread_local std::string g_err;

int fail(int code, const char *fmt, ...) __attribute__((format(printf, 2, 3)));
int fail(int code, const char *fmt, ...)
{
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_err = buf;
    return code;
}

int ok()
{
    g_err.clear();
    return KVQ_OK;
}

int cuda_fail(cudaError_t e, const char *what)
{
    return fail(KVQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

__global__ void truncate_kernel(kvq::CacheView c, const int32_t *__restrict__ lengths)
{
    kvq::pdl_wait();
    kvq::pdl_trigger();
    const int sh = blockIdx.x * blockDim.x + threadIdx.x;
    if (sh >= c.B * c.H) return;
    const int s = sh / c.H, h = sh % c.H;
    const int want = lengths[s];
    const int have = c.len[sh];
    if (want < 0 || want >= have) return;
    c.end[sh] = c.meta[kvq::slot_of(c, s, h, want)] & ~15u;
    c.len[sh] = want;
}

__global__ void lengths_kernel(kvq::CacheView c, int32_t *__restrict__ out)
{
    const int s = blockIdx.x * blockDim.x + threadIdx.x;
    if (s < c.B) out[s] = c.len[s * c.H];
}

// one warp per exported token
__global__ void export_kernel(kvq::CacheView c, int s, int h, int64_t first, int64_t count,
                              uint16_t *k_codes, uint16_t *v_codes, float *side, uint8_t *bits)
{
    const int lane = threadIdx.x & 31;
    const int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (i >= count) return;
    const int64_t j = first + i;
    if (j < 0 || j >= c.len[s * c.H + h]) {
        if (lane == 0) kvq::set_status(c.status, KVQ_ERR_DEVICE_CHECK);
        return;
    }
    const int D = c.D;
    const int64_t slot = kvq::slot_of(c, s, h, j);
    const uint32_t mt = c.meta[slot];
    const int b = 2 << (mt & 3u);
    for (int part = 0; part < 2; ++part) {
        uint16_t *dst = part == 0 ? k_codes : v_codes;
        if (!dst) continue;
        const kvq::RecLoc p = kvq::rec_loc(c, s, h, (mt & ~15u) + part * (b * D / 8));
        for (int ch = lane; ch < D; ch += 32) {
            uint16_t val;
            if (b == 16) {
                val = *reinterpret_cast<const uint16_t *>(p.at(2u * ch));
            } else {
                const int bit = b * ch;
                val = (uint16_t)((*reinterpret_cast<const uint32_t *>(p.at(4u * (bit >> 5))) >> (bit & 31)) &
                                 ((1u << b) - 1u));
            }
            dst[i * D + ch] = val;
        }
    }
    if (lane == 0) {
        if (side) reinterpret_cast<float4 *>(side)[i] = c.side[slot];
        if (bits) bits[i] = (uint8_t)b;
    }
}

__global__ void init_side_kernel(float4 *side, int64_t n)
{
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x)
        side[i] = make_float4(1.f, 0.f, 1.f, 0.f);
}

bool valid_cache(const kvq_cache *c) { return c && c->B > 0 && c->H > 0; }

} // namespace

namespace kvq {
namespace {
cudaEvent_t g_prof_before = nullptr, g_prof_after = nullptr;
}
void profile_before(cudaStream_t st)
{
    if (g_prof_before) cudaEventRecord(g_prof_before, st);
}
void profile_after(cudaStream_t st)
{
    if (g_prof_after) cudaEventRecord(g_prof_after, st);
}

int report_error(int code, const char *msg)
{
    if (code == KVQ_OK) return ok();
    return fail(code, "%s", msg);
}

namespace {
// Launch state that depends on the device: the SM count, and which kernels already had
// their dynamic shared-memory limit raised on which device. One process may drive several
// GPUs (a thread per device), so both are kept per device ordinal under a mutex.
constexpr int kMaxDevices = 256;
std::mutex g_dev_mu;
int g_sms[kMaxDevices] = {};
std::vector<std::pair<const void *, int>> g_attr_done;   // (kernel, device)

int current_device()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) dev = 0;
    return dev;
}
} // namespace

int num_sms()
{
    const int dev = current_device();
    std::lock_guard<std::mutex> lock(g_dev_mu);
    if (g_sms[dev] <= 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        g_sms[dev] = n;
    }
    return g_sms[dev];
}

cudaError_t ensure_smem_attr(const void *func, size_t bytes)
{
    const int dev = current_device();
    std::lock_guard<std::mutex> lock(g_dev_mu);
    for (const auto &e : g_attr_done)
        if (e.first == func && e.second == dev) return cudaSuccess;
    const cudaError_t err = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (err == cudaSuccess) g_attr_done.emplace_back(func, dev);
    return err;
}

// Testing hook state: the n-th device allocation of the next cache creation fails.
std::atomic<int> g_fail_alloc_nth{0};

// One thread waits, with the library's bounded wait, on a barrier that no thread ever
// completes; after `limit_ns` it records KVQ_ERR_DEVICE_CHECK and returns.
__global__ void bounded_wait_kernel(int32_t *status, uint64_t limit_ns)
{
    __shared__ uint64_t bar;
    if (threadIdx.x != 0) return;
    mbar_init(&bar, 1);
    fence_mbar_init();
    mbar_wait(&bar, 0, status, limit_ns);
}
} // namespace kvq

extern "C" {

int kvq_route_argmax(const float *z_attn, const float *z_bits, int64_t n, uint8_t *modes,
                     uint8_t *bits, kvq_stream_t stream)
{
    const ApiRange range("kvq_route_argmax");
    if (n < 0) return fail(KVQ_ERR_ARG, "kvq_route_argmax: n = %lld < 0", (long long)n);
    if ((!z_attn) != (!modes)) return fail(KVQ_ERR_ARG, "kvq_route_argmax: z_attn and modes go together");
    if ((!z_bits) != (!bits)) return fail(KVQ_ERR_ARG, "kvq_route_argmax: z_bits and bits go together");
    if (!z_attn && !z_bits) return fail(KVQ_ERR_ARG, "kvq_route_argmax: nothing to do");
    if (((reinterpret_cast<uintptr_t>(z_attn) | reinterpret_cast<uintptr_t>(z_bits)) & 15u) ||
        ((reinterpret_cast<uintptr_t>(modes) | reinterpret_cast<uintptr_t>(bits)) & 3u))
        return fail(KVQ_ERR_ARG, "kvq_route_argmax: logits must be 16-byte aligned, outputs 4-byte aligned");
    cudaError_t e = kvq::launch_route_argmax(z_attn, z_bits, n, modes, bits, reinterpret_cast<cudaStream_t>(stream));
    return e ? cuda_fail(e, "kvq_route_argmax") : ok();
}

const char *kvq_last_error(void) { return g_err.c_str(); }

int kvq_set_profile_events(void *before, void *after)
{
    if ((before == nullptr) != (after == nullptr))
        return fail(KVQ_ERR_ARG, "kvq_set_profile_events: pass two events or two NULLs");
    kvq::g_prof_before = static_cast<cudaEvent_t>(before);
    kvq::g_prof_after = static_cast<cudaEvent_t>(after);
    return ok();
}

int kvq_cache_create(kvq_cache **out, int batch, int heads, int head_dim,
                     const int64_t *capacity_tokens, kvq_stream_t stream)
{
    return kvq_cache_create_gqa(out, batch, heads, 1, head_dim, capacity_tokens, stream);
}

int kvq_cache_create_gqa(kvq_cache **out, int batch, int heads, int query_group, int head_dim,
                         const int64_t *capacity_tokens, kvq_stream_t stream)
{
    return kvq_cache_create_paged(out, batch, heads, query_group, head_dim, capacity_tokens, 0, 0, stream);
}

int kvq_cache_create_paged(kvq_cache **out, int batch, int heads, int query_group, int head_dim,
                           const int64_t *capacity_tokens, int64_t page_bytes, int64_t pool_pages,
                           kvq_stream_t stream)
{
    if (!out) return fail(KVQ_ERR_ARG, "kvq_cache_create: out is NULL");
    *out = nullptr;
    if (batch <= 0 || heads <= 0) return fail(KVQ_ERR_ARG, "kvq_cache_create: batch and heads must be > 0");
    if (query_group < 1 || query_group > 64)
        return fail(KVQ_ERR_ARG, "kvq_cache_create: query_group = %d outside [1, 64]", query_group);
    if ((int64_t)batch * heads * query_group > (1 << 24))
        return fail(KVQ_ERR_ARG, "kvq_cache_create: batch*heads*query_group too large");
    if ((int64_t)batch * heads > (1 << 24)) return fail(KVQ_ERR_ARG, "kvq_cache_create: batch*heads too large");
    if (head_dim != 64 && head_dim != 128)
        return fail(KVQ_ERR_ARG, "kvq_cache_create: head_dim must be 64 or 128 (got %d)", head_dim);
    if (!capacity_tokens) return fail(KVQ_ERR_ARG, "kvq_cache_create: capacity_tokens is NULL");
    const bool paged = page_bytes != 0;
    int page_shift = 31;
    if (paged) {
        if (page_bytes < 4096 || page_bytes > (1 << 21) || (page_bytes & (page_bytes - 1)))
            return fail(KVQ_ERR_ARG, "kvq_cache_create_paged: page_bytes = %lld is not a power of two in [4 KiB, 2 MiB]",
                        (long long)page_bytes);
        if (pool_pages < 1 || pool_pages > (int64_t)INT32_MAX / 2)
            return fail(KVQ_ERR_ARG, "kvq_cache_create_paged: pool_pages = %lld out of range", (long long)pool_pages);
        page_shift = 0;
        while ((int64_t(1) << page_shift) < page_bytes) ++page_shift;
    }
    std::vector<int32_t> cap(batch), cap_pad(batch);
    std::vector<int64_t> slot_base(batch);
    int64_t slots = 0, max_items = 0, mid_items = 0;
    int32_t max_cap = 0;
    for (int s = 0; s < batch; ++s) {
        const int64_t cp = capacity_tokens[s];
        if (cp < 1 || cp > 8388607)
            return fail(KVQ_ERR_ARG, "kvq_cache_create: capacity_tokens[%d] = %lld outside [1, 8388607]", s,
                        (long long)cp);
        cap[s] = (int32_t)cp;
        cap_pad[s] = (int32_t)((cp + 4) & ~int64_t(3));    // >= cp + 1, multiple of 4
        slot_base[s] = slots;
        slots += (int64_t)heads * cap_pad[s];
        max_items += (int64_t)heads * (kvq::decode_max_items(cp, query_group) + kvq::decode_mid_items(query_group));
        mid_items += (int64_t)heads * kvq::decode_mid_items(query_group);
        max_cap = std::max(max_cap, cap[s]);
    }
    if (max_items > INT32_MAX / 2) return fail(KVQ_ERR_ARG, "kvq_cache_create: too many decode items");

    kvq_cache *c = new kvq_cache();
    std::memset(c, 0, sizeof(*c));
    c->B = batch;
    c->H = heads;
    c->D = head_dim;
    c->total_slots = slots;
    c->max_cap = max_cap;
    cudaGetDevice(&c->device);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);

    const int fail_nth = kvq::g_fail_alloc_nth.exchange(0);   // testing hook, normally 0
    int n_tried = 0;
    auto alloc = [&](size_t bytes) -> void * {
        void *p = nullptr;
        if (++n_tried == fail_nth) return nullptr;
        if (cudaMalloc(&p, std::max<size_t>(bytes, 16)) != cudaSuccess) return nullptr;
        c->allocs[c->n_allocs++] = p;
        return p;
    };
    const int BH = batch * heads;
    const int BHQ = BH * query_group;      // query heads
    kvq::CacheView &v = c->view;
    v.B = batch;
    v.H = heads;
    v.D = head_dim;
    v.G = query_group;
    bool okk = true;
    int32_t *cap_d = (int32_t *)alloc(sizeof(int32_t) * batch);
    int32_t *cap_pad_d = (int32_t *)alloc(sizeof(int32_t) * batch);
    int64_t *slot_base_d = (int64_t *)alloc(sizeof(int64_t) * batch);
    // paged: logical pages per stream, enough for the worst case (b = 16) at capacity
    const int64_t max_lpages = paged ? ((int64_t)max_cap * 4 * head_dim + page_bytes - 1) / page_bytes + 1 : 0;
    v.rec = (uint8_t *)alloc(paged ? (size_t)pool_pages * page_bytes : (size_t)slots * 4 * head_dim);
    if (paged) {
        v.ptab = (uint32_t *)alloc(sizeof(uint32_t) * (size_t)BH * max_lpages);
        v.npages = (int32_t *)alloc(sizeof(int32_t) * BH);
        v.pool_next = (int32_t *)alloc(sizeof(int32_t));
        v.pool_list = (const uint32_t *)alloc(sizeof(uint32_t) * (size_t)pool_pages);
    }
    v.max_lpages = (int32_t)max_lpages;
    v.pool_pages = (int32_t)pool_pages;
    v.page_shift = (uint32_t)page_shift;
    c->page_bytes = paged ? page_bytes : 0;
    v.meta = (uint32_t *)alloc(sizeof(uint32_t) * (size_t)slots);
    v.side = (float4 *)alloc(sizeof(float4) * (size_t)slots);
    v.len = (int32_t *)alloc(sizeof(int32_t) * BH);
    v.end = (uint32_t *)alloc(sizeof(uint32_t) * BH);
    v.wstart = (int32_t *)alloc(sizeof(int32_t) * BH);
    v.wend = (uint32_t *)alloc(sizeof(uint32_t) * BH);
    v.bad = (uint32_t *)alloc(sizeof(uint32_t) * batch);
    v.status = (int32_t *)alloc(sizeof(int32_t));
    kvq::DecodeWork &wk = c->work;
    wk.max_items = max_items;
    wk.mid_base = max_items - mid_items;
    wk.qslots = std::min(query_group, kvq::kDecodeMaxQ);
    wk.items = (kvq::DecodeItem *)alloc(sizeof(kvq::DecodeItem) * (size_t)max_items);
    // the front pair of count words, the cursor, the back pair, the middle pair
    wk.count = (unsigned long long *)alloc(kvq::kDecodeCountWords * sizeof(unsigned long long));
    wk.head_first = (int32_t *)alloc(sizeof(int32_t) * 3 * BH);
    wk.head_cnt = (int32_t *)alloc(sizeof(int32_t) * 3 * BH);
    wk.partials = (float *)alloc(sizeof(float) * (size_t)max_items * wk.qslots * (head_dim + 4));
    c->pf_max_tiles = slots * query_group / 128 + 2LL * BHQ;
    c->pf_tiles = alloc(sizeof(int32_t) * 16 * (size_t)c->pf_max_tiles);    // two lists of 32-byte tiles
    c->pf_count = (int32_t *)alloc(sizeof(int32_t));
    c->pf_qidx = (int32_t *)alloc(sizeof(int32_t) * (size_t)slots * query_group);
    c->scan_chunks = (max_cap + 1023) / 1024;
    c->scan_flags = (uint64_t *)alloc(sizeof(uint64_t) * (size_t)BH * std::max(1, c->scan_chunks));
    for (int i = 0; i < c->n_allocs; ++i) okk = okk && c->allocs[i];
    if (!okk || c->n_allocs != n_tried) {
        kvq_cache_destroy(c);
        return fail(KVQ_ERR_NOMEM, "kvq_cache_create: cudaMalloc failed (%lld slots, %.2f GB of records)",
                    (long long)slots,
                    (paged ? (double)pool_pages * page_bytes : (double)slots * 4 * head_dim) / 1e9);
    }
    // the pool hands out its pages in a scrambled order (xorshift-driven Fisher-Yates), so
    // neighbouring logical pages are not neighbours in memory; nothing depends on the order
    std::vector<uint32_t> plist(paged ? (size_t)pool_pages : 0);
    for (size_t i = 0; i < plist.size(); ++i) plist[i] = (uint32_t)i;
    uint64_t xs = 0x9E3779B97F4A7C15ull ^ (uint64_t)pool_pages;
    for (size_t i = plist.size(); i > 1; --i) {
        xs ^= xs << 13;
        xs ^= xs >> 7;
        xs ^= xs << 17;
        std::swap(plist[i - 1], plist[xs % i]);
    }
    v.cap = cap_d;
    v.cap_pad = cap_pad_d;
    v.slot_base = slot_base_d;
    cudaError_t e = cudaSuccess;
    e = e ? e : cudaMemcpyAsync(cap_d, cap.data(), sizeof(int32_t) * batch, cudaMemcpyHostToDevice, st);
    e = e ? e : cudaMemcpyAsync(cap_pad_d, cap_pad.data(), sizeof(int32_t) * batch, cudaMemcpyHostToDevice, st);
    e = e ? e : cudaMemcpyAsync(slot_base_d, slot_base.data(), sizeof(int64_t) * batch, cudaMemcpyHostToDevice, st);
    e = e ? e : cudaMemsetAsync(v.len, 0, sizeof(int32_t) * BH, st);
    e = e ? e : cudaMemsetAsync(v.end, 0, sizeof(uint32_t) * BH, st);
    e = e ? e : cudaMemsetAsync(v.wstart, 0, sizeof(int32_t) * BH, st);
    e = e ? e : cudaMemsetAsync(v.wend, 0, sizeof(uint32_t) * BH, st);
    e = e ? e : cudaMemsetAsync(v.bad, 0, sizeof(uint32_t) * batch, st);
    e = e ? e : cudaMemsetAsync(v.status, 0, sizeof(int32_t), st);
    e = e ? e : cudaMemsetAsync(v.meta, 0, sizeof(uint32_t) * (size_t)slots, st);
    e = e ? e : cudaMemsetAsync(wk.count, 0, kvq::kDecodeCountWords * sizeof(unsigned long long), st);
    e = e ? e : cudaMemsetAsync(c->scan_flags, 0, sizeof(uint64_t) * (size_t)BH * std::max(1, c->scan_chunks), st);
    if (paged) {
        e = e ? e : cudaMemsetAsync(v.npages, 0, sizeof(int32_t) * BH, st);
        e = e ? e : cudaMemsetAsync(v.pool_next, 0, sizeof(int32_t), st);
        e = e ? e : cudaMemcpyAsync(const_cast<uint32_t *>(v.pool_list), plist.data(), sizeof(uint32_t) * plist.size(),
                                    cudaMemcpyHostToDevice, st);
    }
    if (!e) {
        init_side_kernel<<<1024, 256, 0, st>>>(v.side, slots);
        e = cudaGetLastError();
    }
    // the host vectors above are pageable: finish the copies before they go out of scope
    if (!e) e = cudaStreamSynchronize(st);
    if (e) {
        kvq_cache_destroy(c);
        return cuda_fail(e, "kvq_cache_create");
    }
    *out = c;
    return ok();
}

int kvq_cache_destroy(kvq_cache *c)
{
    if (!c) return ok();
    cudaDeviceSynchronize();
    for (int i = 0; i < c->n_allocs; ++i)
        if (c->allocs[i]) cudaFree(c->allocs[i]);
    delete c;
    return ok();
}

int kvq_cache_reset(kvq_cache *c, kvq_stream_t stream)
{
    if (!valid_cache(c)) return fail(KVQ_ERR_ARG, "kvq_cache_reset: bad cache");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int BH = c->B * c->H;
    cudaError_t e = cudaMemsetAsync(c->view.len, 0, sizeof(int32_t) * BH, st);
    e = e ? e : cudaMemsetAsync(c->view.end, 0, sizeof(uint32_t) * BH, st);
    e = e ? e : cudaMemsetAsync(c->view.status, 0, sizeof(int32_t), st);
    if (c->view.ptab) {                          // every page goes back to the pool
        e = e ? e : cudaMemsetAsync(c->view.npages, 0, sizeof(int32_t) * BH, st);
        e = e ? e : cudaMemsetAsync(c->view.pool_next, 0, sizeof(int32_t), st);
    }
    return e ? cuda_fail(e, "kvq_cache_reset") : ok();
}

int kvq_cache_truncate(kvq_cache *c, const int32_t *lengths, kvq_stream_t stream)
{
    if (!valid_cache(c)) return fail(KVQ_ERR_ARG, "kvq_cache_truncate: bad cache");
    if (!lengths) return fail(KVQ_ERR_ARG, "kvq_cache_truncate: lengths is NULL");
    const int BH = c->B * c->H;
    kvq::launch_pdl(truncate_kernel, dim3((BH + 255) / 256), dim3(256), 0, reinterpret_cast<cudaStream_t>(stream),
                    c->view, lengths);
    cudaError_t e = cudaGetLastError();
    return e ? cuda_fail(e, "kvq_cache_truncate") : ok();
}

int kvq_cache_lengths(const kvq_cache *c, int32_t *lengths, kvq_stream_t stream)
{
    if (!valid_cache(c)) return fail(KVQ_ERR_ARG, "kvq_cache_lengths: bad cache");
    if (!lengths) return fail(KVQ_ERR_ARG, "kvq_cache_lengths: lengths is NULL");
    lengths_kernel<<<(c->B + 255) / 256, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(c->view, lengths);
    cudaError_t e = cudaGetLastError();
    return e ? cuda_fail(e, "kvq_cache_lengths") : ok();
}

int kvq_write(const void *k, const void *v, const uint8_t *bits, const int32_t *cu_seqlens,
              int64_t n_tok, kvq_cache *c, kvq_stream_t stream)
{
    const ApiRange range("kvq_write");
    if (!valid_cache(c)) return fail(KVQ_ERR_ARG, "kvq_write: bad cache");
    if (n_tok < 0 || n_tok > (int64_t)INT32_MAX / c->H)
        return fail(KVQ_ERR_ARG, "kvq_write: n_tok = %lld out of range", (long long)n_tok);
    if (!cu_seqlens) return fail(KVQ_ERR_ARG, "kvq_write: cu_seqlens is NULL");
    if (n_tok > 0 && (!k || !v || !bits)) return fail(KVQ_ERR_ARG, "kvq_write: k, v or bits is NULL");
    if ((reinterpret_cast<uintptr_t>(k) | reinterpret_cast<uintptr_t>(v)) & 15u)
        return fail(KVQ_ERR_ARG, "kvq_write: k and v must be 16-byte aligned");
    cudaError_t e = kvq::launch_write(c, static_cast<const __half *>(k), static_cast<const __half *>(v),
                                      bits, cu_seqlens, n_tok, reinterpret_cast<cudaStream_t>(stream));
    return e ? cuda_fail(e, "kvq_write") : ok();
}

int routed_attn_prefill(const void *q, const kvq_cache *c, const uint8_t *modes, int w,
                        const int32_t *cu_seqlens, int64_t n_tok, float *out, kvq_stream_t stream)
{
    const ApiRange range("routed_attn_prefill");
    if (!valid_cache(c)) return fail(KVQ_ERR_ARG, "routed_attn_prefill: bad cache");
    if (w < 0) return fail(KVQ_ERR_ARG, "routed_attn_prefill: w = %d < 0", w);
    if (n_tok < 0 || n_tok > (int64_t)INT32_MAX / ((int64_t)c->H * c->view.G))
        return fail(KVQ_ERR_ARG, "routed_attn_prefill: n_tok = %lld out of range", (long long)n_tok);
    if (!cu_seqlens) return fail(KVQ_ERR_ARG, "routed_attn_prefill: cu_seqlens is NULL");
    if (n_tok > 0 && (!q || !modes || !out))
        return fail(KVQ_ERR_ARG, "routed_attn_prefill: q, modes or out is NULL");
    if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(out)) & 15u)
        return fail(KVQ_ERR_ARG, "routed_attn_prefill: q and out must be 16-byte aligned");
    if (n_tok * c->H > c->total_slots)
        return fail(KVQ_ERR_ARG, "routed_attn_prefill: n_tok = %lld exceeds the cache's capacity", (long long)n_tok);
    cudaError_t e = kvq::launch_prefill_tc(c, static_cast<const __half *>(q), modes, w, cu_seqlens, n_tok, out,
                                           reinterpret_cast<cudaStream_t>(stream));
    return e ? cuda_fail(e, "routed_attn_prefill") : ok();
}

int routed_attn_decode(const void *q, const kvq_cache *c, const uint8_t *modes, int w, float *out,
                       kvq_stream_t stream)
{
    const ApiRange range("routed_attn_decode");
    if (!valid_cache(c)) return fail(KVQ_ERR_ARG, "routed_attn_decode: bad cache");
    if (w < 0) return fail(KVQ_ERR_ARG, "routed_attn_decode: w = %d < 0", w);
    if (!q || !modes || !out) return fail(KVQ_ERR_ARG, "routed_attn_decode: q, modes or out is NULL");
    if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(out)) & 15u)
        return fail(KVQ_ERR_ARG, "routed_attn_decode: q and out must be 16-byte aligned");
    cudaError_t e = kvq::launch_decode(c, static_cast<const __half *>(q), modes, w, out,
                                       reinterpret_cast<cudaStream_t>(stream));
    return e ? cuda_fail(e, "routed_attn_decode") : ok();
}

int kvq_decode_step(const void *q, const void *k, const void *v, const uint8_t *bits, const int32_t *cu_seqlens,
                    int64_t n_tok, const int32_t *positions, const uint8_t *modes, int w, kvq_cache *c,
                    float *out, kvq_stream_t stream)
{
    const ApiRange range("kvq_decode_step");
    if (!valid_cache(c)) return fail(KVQ_ERR_ARG, "kvq_decode_step: bad cache");
    if (w < 0) return fail(KVQ_ERR_ARG, "kvq_decode_step: w = %d < 0", w);
    if (n_tok < 0 || n_tok > (int64_t)INT32_MAX / c->H)
        return fail(KVQ_ERR_ARG, "kvq_decode_step: n_tok = %lld out of range", (long long)n_tok);
    if (!q || !modes || !out || !cu_seqlens) return fail(KVQ_ERR_ARG, "kvq_decode_step: q, modes, out or cu_seqlens is NULL");
    if (n_tok > 0 && (!k || !v || !bits)) return fail(KVQ_ERR_ARG, "kvq_decode_step: k, v or bits is NULL");
    if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(out) | reinterpret_cast<uintptr_t>(k) |
         reinterpret_cast<uintptr_t>(v)) & 15u)
        return fail(KVQ_ERR_ARG, "kvq_decode_step: q, k, v and out must be 16-byte aligned");
    cudaError_t e = kvq::launch_decode_step(c, static_cast<const __half *>(q), static_cast<const __half *>(k),
                                            static_cast<const __half *>(v), bits, cu_seqlens, n_tok, positions,
                                            modes, w, out, reinterpret_cast<cudaStream_t>(stream));
    return e ? cuda_fail(e, "kvq_decode_step") : ok();
}

int kvq_cache_export(const kvq_cache *c, int seq, int head, int64_t first, int64_t count,
                     uint16_t *k_codes, uint16_t *v_codes, float *side, uint8_t *bits, kvq_stream_t stream)
{
    if (!valid_cache(c)) return fail(KVQ_ERR_ARG, "kvq_cache_export: bad cache");
    if (seq < 0 || seq >= c->B || head < 0 || head >= c->H)
        return fail(KVQ_ERR_ARG, "kvq_cache_export: (seq, head) = (%d, %d) out of range", seq, head);
    if (first < 0 || count < 0 || first + count > c->max_cap)
        return fail(KVQ_ERR_ARG, "kvq_cache_export: token range out of capacity");
    if (count == 0) return ok();
    const int64_t threads = count * 32;
    export_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        c->view, seq, head, first, count, k_codes, v_codes, side, bits);
    cudaError_t e = cudaGetLastError();
    return e ? cuda_fail(e, "kvq_cache_export") : ok();
}

int kvq_test_fail_alloc(int nth)
{
    if (nth < 0) return fail(KVQ_ERR_ARG, "kvq_test_fail_alloc: nth = %d < 0", nth);
    kvq::g_fail_alloc_nth.store(nth);
    return ok();
}

int kvq_test_bounded_wait(kvq_cache *c, int64_t limit_ns, kvq_stream_t stream)
{
    if (!valid_cache(c)) return fail(KVQ_ERR_ARG, "kvq_test_bounded_wait: bad cache");
    if (limit_ns < 1000 || limit_ns > 100000000)
        return fail(KVQ_ERR_ARG, "kvq_test_bounded_wait: limit_ns = %lld outside [1e3, 1e8]", (long long)limit_ns);
    kvq::bounded_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(c->view.status,
                                                                               (uint64_t)limit_ns);
    cudaError_t e = cudaGetLastError();
    return e ? cuda_fail(e, "kvq_test_bounded_wait") : ok();
}

int kvq_check(kvq_cache *c, kvq_stream_t stream)
{
    if (!valid_cache(c)) return fail(KVQ_ERR_ARG, "kvq_check: bad cache");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    int32_t h = 0;
    cudaError_t e = cudaStreamSynchronize(st);
    e = e ? e : cudaMemcpy(&h, c->view.status, sizeof(int32_t), cudaMemcpyDeviceToHost);
    e = e ? e : cudaMemset(c->view.status, 0, sizeof(int32_t));
    if (e) return cuda_fail(e, "kvq_check");
    if (h) return fail(h, "device-side check failed with status %d", h);
    return ok();
}

} // extern "C"
