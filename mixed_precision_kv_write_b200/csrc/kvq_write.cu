// Quantize-on-write (TriRoute paper review page, section 3, Eq. 4).
//
// A call with at most 2 * batch tokens (decode steps) is one launch of
//   write_append_kernel a CTA per sequence doing both steps below for its tokens;
// longer calls take two launches:
//   write_scan_kernel   a warp (short appends) or a block (long ones) per (sequence, head):
//                       validates capacity and widths (a bad width rejects the sequence's
//                       write for every head) and assigns each new token's record offset
//                       (prefix sum of record sizes b*D/4 in token order).
//   write_quant_kernel  one CTA per tile of tokens x heads staged by bulk copies: for K
//                       and for V of every (token, head), min/max over the head_dim
//                       values, s = (max - min)/(2^b - 1), z = min, codes
//                       rint((x - z)/s) in IEEE fp32 round-to-nearest-even (s == 0 -> 0),
//                       packed LSB-first into the record; (s, z) into the side table;
//                       commits the new length and stream end of accepted sequences.
// HBM traffic per (token, head): reads 2*D*2 bytes, writes b*D/4 + 16 + 4 bytes.
#include <algorithm>

#include "kvq_quant.cuh"

namespace kvq {
namespace {

// TPS threads per (sequence, head): validates the call's widths of its head (a bad entry
// marks the sequence bad for this call, so no head of it is written), checks capacity,
// and assigns the new tokens' record offsets with a parallel prefix sum of the record
// sizes b*D/4. The new length/end are committed by the quantize kernel, which sees the
// per-sequence verdict of every head.
template <int TPS, int BS = (TPS < 256 ? 256 : TPS)>
__global__ void __launch_bounds__(BS)
write_scan_kernel(CacheView c, const uint8_t *__restrict__ bits, const int32_t *__restrict__ cu,
                  int64_t n_tok, uint32_t gen)
{
    constexpr int PER = 8;                       // tokens per thread per pass
    constexpr int WARPS = TPS / 32;
    __shared__ uint32_t wsum[BS / 32];
    pdl_wait();
    pdl_trigger();
    const int tid = threadIdx.x % TPS, lane = threadIdx.x & 31;
    const int grp = threadIdx.x / TPS, wig = tid >> 5;     // group in block, warp in group
    const int64_t gsh = (int64_t)blockIdx.x * (BS / TPS) + grp;
    const int H = c.H;
    if (gsh >= (int64_t)c.B * H) return;         // whole group exits together
    const int s = (int)(gsh / H), h = (int)(gsh % H), sh = s * H + h;

    const int64_t t0 = cu[s], t1 = cu[s + 1];
    if (t0 < 0 || t1 < t0 || t1 > n_tok || (s == 0 && t0 != 0)) {
        if (tid == 0) {
            set_status(c.status, KVQ_ERR_DEVICE_CHECK);
            c.wstart[sh] = -1;
        }
        return;
    }
    const int n = (int)(t1 - t0);
    const int L0 = c.len[sh];
    if ((int64_t)L0 + n > c.cap[s]) {
        if (tid == 0) {
            set_status(c.status, KVQ_ERR_CAPACITY);
            c.wstart[sh] = -1;
        }
        return;
    }
    const int64_t slot0 = slot_of(c, s, h, L0);
    uint32_t off = c.end[sh];
    bool bad = false;
    for (int base = 0; base < n; base += TPS * PER) {
        uint32_t sz[PER];
        uint32_t wcs[PER];
        uint32_t mine = 0;
#pragma unroll
        for (int e = 0; e < PER; ++e) {
            const int i = base + tid * PER + e;
            sz[e] = 0;
            wcs[e] = 0;
            if (i < n) {
                const int b = bits[(t0 + i) * H + h];
                const int wc = width_code(b);
                if (wc < 0) bad = true;
                else {
                    wcs[e] = (uint32_t)wc;
                    sz[e] = (uint32_t)(b * c.D / 4);
                }
            }
            mine += sz[e];
        }
        uint32_t incl = mine;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, incl, d);
            if (lane >= d) incl += y;
        }
        uint32_t before = incl - mine, total;
        if (WARPS > 1) {
            if (lane == 31) wsum[grp * WARPS + wig] = incl;
            __syncthreads();
            uint32_t wpre = 0, wtot = 0;
#pragma unroll
            for (int q = 0; q < WARPS; ++q) {
                const uint32_t t = wsum[grp * WARPS + q];
                if (q < wig) wpre += t;
                wtot += t;
            }
            __syncthreads();
            before += wpre;
            total = wtot;
        } else {
            total = __shfl_sync(0xffffffffu, incl, 31);
        }
        uint32_t o = off + before;
#pragma unroll
        for (int e = 0; e < PER; ++e) {
            const int i = base + tid * PER + e;
            if (i < n) c.meta[slot0 + i] = o | wcs[e];
            o += sz[e];
        }
        off += total;
    }
    if (bad) {
        c.bad[s] = gen;                          // same value from every writer
        set_status(c.status, KVQ_ERR_BITS);
    }
    if (tid == 0) {
        if (map_pages(c, s, h, off)) {           // paged caches: pages for the new bytes
            c.wstart[sh] = L0;
            c.wend[sh] = off;
        } else {
            set_status(c.status, KVQ_ERR_CAPACITY);
            c.wstart[sh] = -1;
        }
    }
}

// Long calls: the same results as write_scan_kernel, with each (sequence, head) split into
// chunks of 1024 tokens, one CTA of 256 threads per chunk, so that long sequences do not
// leave most SMs idle. A CTA scans its chunk's record sizes and sums those of the up to 16
// chunks before it straight from the widths (their loads go out with its own), so most
// CTAs wait on no other; a chunk further out adds the running prefix that the chunk 17
// places back published in a per-(sequence, head) array of 64-bit words (call generation
// << 34 | 2 << 32 | bytes through the chunk). That wait is on a CTA of lower index, which
// starts first, and is bounded. The last chunk of a (sequence, head) records the write
// start and the new stream end.
constexpr int kScanChunkThreads = 256, kScanChunkPer = 4, kScanChunk = kScanChunkThreads * kScanChunkPer;
constexpr int kScanDirect = 16;                  // chunks summed directly before the look-back

// The look-back words carry their whole message (no other data is published with them),
// so they are stored and polled with relaxed gpu-scope accesses: coherent in L2, no fence.
__device__ __forceinline__ void st_relaxed_u64(uint64_t *p, uint64_t v)
{
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

__device__ __forceinline__ uint64_t ld_relaxed_u64(const uint64_t *p)
{
    uint64_t v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

__global__ void __launch_bounds__(kScanChunkThreads)
write_scan_chunk_kernel(CacheView c, const uint8_t *__restrict__ bits, const int32_t *__restrict__ cu,
                        int64_t n_tok, uint32_t gen, uint64_t *__restrict__ flags, int n_chunks)
{
    __shared__ uint32_t wsum[kScanChunkThreads / 32], wpre_sh[kScanChunkThreads / 32];
    __shared__ uint32_t excl_sh;
    pdl_wait();
    pdl_trigger();
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int64_t gsh = blockIdx.x / n_chunks;
    const int ck = (int)(blockIdx.x % n_chunks);
    const int H = c.H;
    if (gsh >= (int64_t)c.B * H) return;
    const int s = (int)(gsh / H), h = (int)(gsh % H), sh = s * H + h;
    // every load that does not depend on the token range goes out with cu
    const int64_t t0 = cu[s], t1 = cu[s + 1];
    const int L0 = c.len[sh];
    const int cap = c.cap[s];
    const uint32_t off0 = c.end[sh];
    if (t0 < 0 || t1 < t0 || t1 > n_tok || (s == 0 && t0 != 0)) {
        if (ck == 0 && tid == 0) {
            set_status(c.status, KVQ_ERR_DEVICE_CHECK);
            c.wstart[sh] = -1;
        }
        return;
    }
    const int n = (int)(t1 - t0);
    if (ck > 0 && ck * kScanChunk >= n) return;  // past this sequence's tokens
    if ((int64_t)L0 + n > cap) {
        if (ck == 0 && tid == 0) {
            set_status(c.status, KVQ_ERR_CAPACITY);
            c.wstart[sh] = -1;
        }
        return;
    }
    const int nck = (n + kScanChunk - 1) / kScanChunk;
    // this chunk's tokens: kScanChunkPer consecutive ones per thread
    uint32_t sz[kScanChunkPer], wcs[kScanChunkPer], mine = 0;
    bool bad = false;
#pragma unroll
    for (int e = 0; e < kScanChunkPer; ++e) {
        const int i = ck * kScanChunk + tid * kScanChunkPer + e;
        sz[e] = 0;
        wcs[e] = 0;
        if (i < n) {
            const int b = bits[(t0 + i) * H + h];
            const int wc = width_code(b);
            if (wc < 0) bad = true;
            else {
                wcs[e] = (uint32_t)wc;
                sz[e] = (uint32_t)(b * c.D / 4);
            }
        }
        mine += sz[e];
    }
    // the bytes of the up to kScanDirect chunks before this one, summed from their widths
    // directly (a bad width counts 0 bytes, as in its own chunk)
    const int cd = max(0, ck - kScanDirect);
    uint32_t pre = 0;
    for (int cc = cd; cc < ck; ++cc) {
#pragma unroll
        for (int e = 0; e < kScanChunkPer; ++e) {
            const int b = bits[(t0 + cc * kScanChunk + tid * kScanChunkPer + e) * H + h];
            pre += width_code(b) >= 0 ? (uint32_t)(b * c.D / 4) : 0u;
        }
    }
    uint32_t incl = mine;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, d);
        if (lane >= d) incl += y;
    }
#pragma unroll
    for (int d = 16; d >= 1; d >>= 1) pre += __shfl_xor_sync(0xffffffffu, pre, d);
    if (lane == 31) wsum[wid] = incl;
    if (lane == 0) wpre_sh[wid] = pre;
    __syncthreads();
    uint32_t wpre = 0, agg = 0, pre_all = 0;
#pragma unroll
    for (int q = 0; q < kScanChunkThreads / 32; ++q) {
        const uint32_t t = wsum[q];
        if (q < wid) wpre += t;
        agg += t;
        pre_all += wpre_sh[q];
    }
    if (tid == 0) {
        // chunks more than kScanDirect back: the running prefix that chunk ck - kScanDirect - 1
        // publishes (gen << 34 | 2 << 32 | bytes through that chunk); every chunk publishes
        // its own
        uint64_t *fl = flags + gsh * n_chunks;
        const uint32_t g30 = gen & 0x3FFFFFFFu;
        const uint64_t tag = (uint64_t)g30 << 34;
        uint32_t excl = off0 + pre_all;
        if (ck > kScanDirect) {
            const int j = ck - kScanDirect - 1;
            uint64_t t_begin = 0;
            for (uint32_t it = 0;; ++it) {
                const uint64_t wv = ld_relaxed_u64(&fl[j]);
                if ((uint32_t)(wv >> 34) == g30 && ((uint32_t)(wv >> 32) & 3u) == 2u) {
                    excl = (uint32_t)wv + pre_all;
                    break;
                }
                if ((it & 63u) == 0) {            // bounded: about two seconds
                    const uint64_t tn = global_ns();
                    if (t_begin == 0) t_begin = tn;
                    else if (tn - t_begin > kWaitLimitNs) {
                        set_status(c.status, KVQ_ERR_DEVICE_CHECK);
                        break;
                    }
                }
            }
        }
        st_relaxed_u64(&fl[ck], tag | (2ull << 32) | (uint64_t)(excl + agg));
        excl_sh = excl;
    }
    __syncthreads();
    const int64_t slot0 = slot_of(c, s, h, L0);
    uint32_t o = excl_sh + wpre + incl - mine;
#pragma unroll
    for (int e = 0; e < kScanChunkPer; ++e) {
        const int i = ck * kScanChunk + tid * kScanChunkPer + e;
        if (i < n) c.meta[slot0 + i] = o | wcs[e];
        o += sz[e];
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) {
        c.bad[s] = gen;                          // same value from every writer
        set_status(c.status, KVQ_ERR_BITS);
    }
    if (tid == 0 && (nck == 0 || ck == nck - 1)) {   // the last chunk (or an empty write)
        const uint32_t end = excl_sh + agg;
        if (map_pages(c, s, h, end)) {           // paged caches: pages for the new bytes
            c.wstart[sh] = L0;
            c.wend[sh] = end;
        } else {
            set_status(c.status, KVQ_ERR_CAPACITY);
            c.wstart[sh] = -1;
        }
    }
}

// Staging of the quantize kernel: each CTA copies the fp16 K and V rows of T tokens x HG
// heads (at most kWqHalves values per tensor) into shared memory with two bulk copies.
#ifndef KVQ_WQ_LPV
#define KVQ_WQ_LPV 2
#endif
#ifndef KVQ_WQ_THREADS
#define KVQ_WQ_THREADS (128 * KVQ_WQ_LPV)
#endif
#ifndef KVQ_WQ_HALVES
#define KVQ_WQ_HALVES 8192
#endif
constexpr int kWqThreads = KVQ_WQ_THREADS;
constexpr int kWqLanesPerVec = KVQ_WQ_LPV;   // lanes per vector at head_dim 128 (64: one)
constexpr int kWqHalves = KVQ_WQ_HALVES; // fp16 values of K (and of V) staged per CTA
constexpr int kWqMaxPairs = kWqHalves / 64;
static_assert(kWqMaxPairs <= kWqThreads, "one (token, head) pair per thread");

struct WqPair {                          // one (token, head) of the CTA
    int64_t slot;                        // side-table slot
    uint32_t meta;                       // record offset in the stream | width code
    int32_t s;                           // sequence; -1: not written (rejected write or bad call)
    int32_t h;
    int32_t pad;
};

#ifndef KVQ_WQ_MIXED_SUB
#define KVQ_WQ_MIXED_SUB 1
#endif

// fl(x - z) for an fp16 x and an fp32 z: one instruction with the fp16 operand widened
// exactly (sm_100 mixed-precision subtract), or the explicit conversion then the subtract.
__device__ __forceinline__ float sub_h(uint32_t hbits, float z)
{
#if KVQ_WQ_MIXED_SUB
    float d;
    asm("sub.rn.f32.f16 %0, %1, %2;" : "=f"(d) : "h"((unsigned short)hbits), "f"(z));
    return d;
#else
    return __fsub_rn(__half2float(__ushort_as_half((unsigned short)hbits)), z);
#endif
}

// Codes of one chunk of 8 fp16 values (BITS = 2, 4, 8), packed LSB-first into w (BITS
// bytes), with the arithmetic of quant_store: u = fl(x - z), Markstein's correctly rounded
// quotient fl(u / s), rint by the 1.5 * 2^23 addition; `probe` sums the quotients.
template <int BITS>
__device__ __forceinline__ void chunk_codes(const uint4 &raw, float z, float2 y2, float2 ns2, float2 &probe,
                                            uint32_t (&w)[2])
{
    const uint32_t hw[4] = {raw.x, raw.y, raw.z, raw.w};
    const float2 mg2 = make_float2(kRoundMagic, kRoundMagic);
    w[0] = w[1] = 0u;
#pragma unroll
    for (int e = 0; e < 4; ++e) {                     // values 2e, 2e + 1
        const float2 u = make_float2(sub_h(hw[e] & 0xFFFFu, z), sub_h(hw[e] >> 16, z));
        const float2 q0 = __fmul2_rn(u, y2);
        const float2 r = __ffma2_rn(ns2, q0, u);      // u - s * q0, exact
        const float2 q = __ffma2_rn(r, y2, q0);       // RN(u / s)
        const float2 t = __fadd2_rn(q, mg2);
        probe = __fadd2_rn(probe, q);
        w[(2 * e * BITS) >> 5] += __float_as_uint(t.x) << ((2 * e * BITS) & 31);
        w[((2 * e + 1) * BITS) >> 5] += __float_as_uint(t.y) << (((2 * e + 1) * BITS) & 31);
    }
    constexpr int kWordBits = BITS * 8 < 32 ? BITS * 8 : 32;
    uint32_t magic = 0u;
#pragma unroll
    for (int sh = 0; sh < kWordBits; sh += BITS) magic += kRoundMagicBits << sh;
    w[0] -= magic;
    if (BITS == 8) w[1] -= magic;
}

// The plain formula for one chunk (taken only when a quotient was NaN: NaN or infinite
// inputs), which gives code 0 for a NaN quotient.
template <int BITS>
__device__ __forceinline__ void chunk_codes_plain(const uint4 &raw, float z, float sc, uint32_t (&w)[2])
{
    const uint32_t hw[4] = {raw.x, raw.y, raw.z, raw.w};
    const float top = (float)((1u << BITS) - 1u);
    w[0] = w[1] = 0u;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        const float x = __half2float(__ushort_as_half((unsigned short)((e & 1) ? hw[e >> 1] >> 16 : hw[e >> 1] & 0xFFFFu)));
        const float cv = fminf(fmaxf(rintf(__fdiv_rn(__fsub_rn(x, z), sc)), 0.0f), top);
        w[(e * BITS) >> 5] |= __float2uint_rz(cv) << ((e * BITS) & 31);
    }
}

// A record part's bytes [0, n): rel < split at p0 + rel, else at p1 + rel (a paged part
// crosses at most one page boundary, never inside a 16-byte group; contiguous parts never
// split).
struct PartDst {
    uint8_t *p0, *p1;
    uint32_t split;
    __device__ __forceinline__ uint8_t *at(uint32_t rel) const { return (rel < split ? p0 : p1) + rel; }
};

__device__ __forceinline__ PartDst part_dst(const RecLoc &L, uint32_t n)
{
    PartDst d;
    d.p0 = L.at(0);
    d.p1 = d.p0;
    d.split = 0xFFFFFFFFu;
    if (L.pt) {
        const uint32_t page = 1u << L.shift;
        const uint32_t room = page - (L.off & (page - 1u));
        if (room < n) {
            d.split = room;
            d.p1 = L.at(room) - room;
        }
    }
    return d;
}

__device__ __forceinline__ void swap_if(bool c, uint32_t &a, uint32_t &b)
{
    const uint32_t t = c ? b : a;
    b = c ? a : b;
    a = t;
}

// One lane writes the codes of NCHL chunks of 8 fp16 values held in shared memory (a whole
// vector, or its half when two lanes share a vector), a 16-byte group (G = 16/BITS chunks)
// per store at byte rel0 + 16 * group of the record part. With x = lane mod 8 (x < NCHL),
// step j reads chunk j ^ x: the eight lanes of a shared-memory phase read eight different
// bank groups (every vector starts on a 128-byte boundary), and the G steps k*G .. k*G + G - 1
// cover the chunks of group k ^ (x / G), chunk slot i ^ (x mod G) filled at step k*G + i;
// the slots are put in place by conditional swaps before the store. PLAIN selects the
// plain formula (taken only when a quotient was NaN: NaN or infinite inputs). Returns the
// sum of the quotients.
template <int NCHL, int BITS, bool PLAIN>
__device__ __forceinline__ float lane_codes(const uint4 *src, float z, float sc, const PartDst &dst, uint32_t rel0,
                                            int x)
{
    constexpr int G = 16 / BITS, NG = NCHL / G;
    static_assert(NCHL >= G, "a lane covers whole 16-byte groups");
    const float y = __frcp_rn(sc);
    const float2 y2 = make_float2(y, y), ns2 = make_float2(-sc, -sc);
    float2 probe = make_float2(0.0f, 0.0f);
    const int m = x & (G - 1);
#pragma unroll 1
    for (int k = 0; k < NG; ++k) {
        uint32_t o[4] = {0u, 0u, 0u, 0u};
#pragma unroll
        for (int i = 0; i < G; ++i) {
            uint32_t w[2];
            const uint4 raw = src[(k * G + i) ^ x];
            if (PLAIN) chunk_codes_plain<BITS>(raw, z, sc, w);
            else chunk_codes<BITS>(raw, z, y2, ns2, probe, w);
            if (BITS == 8) {
                o[2 * i] = w[0];
                o[2 * i + 1] = w[1];
            } else if (BITS == 4) {
                o[i] = w[0];
            } else {
                o[i >> 1] |= (w[0] & 0xFFFFu) << (16 * (i & 1));
            }
        }
        if (BITS == 8) {
            swap_if(m & 1, o[0], o[2]);
            swap_if(m & 1, o[1], o[3]);
        } else if (BITS == 4) {
            swap_if(m & 1, o[0], o[1]);
            swap_if(m & 1, o[2], o[3]);
            swap_if(m & 2, o[0], o[2]);
            swap_if(m & 2, o[1], o[3]);
        } else {
            const uint32_t sel = (m & 1) ? 0x1032u : 0x3210u;     // halves swapped or kept
#pragma unroll
            for (int e = 0; e < 4; ++e) o[e] = __byte_perm(o[e], 0u, sel);
            swap_if(m & 2, o[0], o[1]);
            swap_if(m & 2, o[2], o[3]);
            swap_if(m & 4, o[0], o[2]);
            swap_if(m & 4, o[1], o[3]);
        }
        *reinterpret_cast<uint4 *>(dst.at(rel0 + 16u * (uint32_t)(k ^ (x / G)))) = make_uint4(o[0], o[1], o[2], o[3]);
    }
    return probe.x + probe.y;
}

template <int NCHL, int BITS>
__device__ __forceinline__ void lane_quant(const uint4 *src, float z, float sc, const PartDst &dst, uint32_t rel0,
                                           int x)
{
    const float nan_probe = lane_codes<NCHL, BITS, false>(src, z, sc, dst, rel0, x);
    if (nan_probe != nan_probe) lane_codes<NCHL, BITS, true>(src, z, sc, dst, rel0, x);   // same lane, same bytes
}

// LPV lanes (1 or 2, adjacent) quantize one vector: min/max (combined across the pair with
// one shuffle), then each lane its share of the record part (the raw fp16 bits for
// b = 16); the first lane writes the (s, z) side entry.
template <int D, int LPV>
__device__ __forceinline__ void lane_vector(const CacheView &c, const uint4 *vsrc, int b, const RecLoc &L,
                                            int64_t slot, int part, int x, int half)
{
    constexpr int NCHL = D / 8 / LPV;            // chunks per lane
    const PartDst dst = part_dst(L, (uint32_t)(b * D / 8));
    const uint4 *src = vsrc + half * NCHL;
    const uint32_t rel0 = (uint32_t)(half * (b * D / 8 / LPV));
    float sc = 1.0f, z = 0.0f;
    if (b == 16) {
#pragma unroll 4
        for (int j = 0; j < NCHL; ++j)
            *reinterpret_cast<uint4 *>(dst.at(16u * (uint32_t)(half * NCHL + (j ^ x)))) = src[j ^ x];
    } else {
        // min and max in fp16 (exact); -0 and +0 are one value, stored as +0 below
        __half2 lo2 = *reinterpret_cast<const __half2 *>(&src[x].x), hi2 = lo2;
#pragma unroll 4
        for (int j = 0; j < NCHL; ++j) {
            const uint4 r = src[j ^ x];
            const uint32_t hw[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                lo2 = __hmin2(lo2, *reinterpret_cast<const __half2 *>(&hw[e]));
                hi2 = __hmax2(hi2, *reinterpret_cast<const __half2 *>(&hw[e]));
            }
        }
        __half2 mm = __halves2half2(__hmin(__low2half(lo2), __high2half(lo2)),
                                    __hneg(__hmax(__low2half(hi2), __high2half(hi2))));
        if (LPV == 2) {                          // (min, -max) of the pair's halves
            const unsigned pair = 3u << (threadIdx.x & 30);
            const uint32_t o = __shfl_xor_sync(pair, *reinterpret_cast<uint32_t *>(&mm), 1);
            mm = __hmin2(mm, *reinterpret_cast<const __half2 *>(&o));
        }
        const float mn = __low2float(mm), mx = -__high2float(mm);
        const float top = (float)((1u << b) - 1u);
        sc = __fadd_rn(__fdiv_rn(__fsub_rn(mx, mn), top), 0.0f);
        z = __fadd_rn(mn, 0.0f);
        if (sc != 0.0f) {
            if (b == 8) lane_quant<NCHL, 8>(src, z, sc, dst, rel0, x);
            else if (b == 4) lane_quant<NCHL, 4>(src, z, sc, dst, rel0, x);
            else lane_quant<NCHL, 2>(src, z, sc, dst, rel0, x);
        } else {                                   // a constant vector: every code is 0
            for (uint32_t o = 0; o < (uint32_t)(b * D / 8 / LPV); o += 16u)
                *reinterpret_cast<uint4 *>(dst.at(rel0 + o)) = make_uint4(0u, 0u, 0u, 0u);
        }
    }
    if (half == 0) reinterpret_cast<float2 *>(&c.side[slot])[part] = make_float2(sc, z);
}

// One CTA per tile of T tokens x HG heads. Warp 0 starts two bulk copies (the tile's K and
// V rows are contiguous when HG = H, else one copy per token and tensor); meanwhile every
// thread resolves the destination of one (token, head): its sequence (binary search of
// cu_seqlens), the call's verdict, the write start, and the record offset the scan kernel
// assigned. Then each vector of D values is quantized by one lane from shared memory.
template <int D>
__global__ void __launch_bounds__(kWqThreads)
write_quant_kernel(CacheView c, const __half *__restrict__ k, const __half *__restrict__ v,
                   const int32_t *__restrict__ cu, int64_t n_tok, uint32_t gen, int T, int HG)
{
    extern __shared__ __align__(128) uint8_t wq_smem[];
    __shared__ uint64_t bar;
    __shared__ WqPair pairs[kWqMaxPairs];
    __shared__ uint8_t order[kWqMaxPairs];   // written pairs sorted by width
    __shared__ int n_written;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // Launched right after the scan kernel: the K/V copies and the sequence lookup read only
    // the call's inputs and start before the scan has finished; pdl_wait() below comes
    // before the first read of what the scan writes (widths verdict, write start, offsets).
    pdl_trigger();
    const int H = c.H;
    const int64_t t0 = (int64_t)blockIdx.x * T;
    const int h0 = blockIdx.y * HG;
    const int Tc = (int)(n_tok - t0 < T ? n_tok - t0 : T);
    const int HGc = min(HG, H - h0);
    const uint32_t tensor_bytes = (uint32_t)(Tc * HGc * D * 2);
    __half *sk = reinterpret_cast<__half *>(wq_smem);
    __half *sv = sk + kWqHalves;

    if (tid == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (warp == 0) {
        if (lane == 0) mbar_arrive_expect_tx(&bar, 2 * tensor_bytes);
        __syncwarp();
        if (HGc == H) {
            if (lane < 2)
                bulk_g2s(lane ? sv : sk, (lane ? v : k) + t0 * H * D, tensor_bytes, &bar);
        } else {
            for (int i = lane; i < 2 * Tc; i += 32) {
                const int j = i >> 1;
                bulk_g2s((i & 1 ? sv : sk) + j * HGc * D,
                         (i & 1 ? v : k) + ((t0 + j) * H + h0) * D, HGc * D * 2, &bar);
            }
        }
    }

    // one (token, head) pair per thread (at most kWqMaxPairs <= kWqThreads pairs per tile)
    const int i = tid;
    const bool has_pair = i < Tc * HGc;
    const int64_t tk = t0 + i / max(HGc, 1);
    const int h = h0 + i % max(HGc, 1);
    int s = 0;
    if (has_pair) {
        int lo = 0, hi = c.B;                // cu[lo] <= tk < cu[hi]
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (cu[mid] <= tk) lo = mid;
            else hi = mid;
        }
        s = lo;
    }
    pdl_wait();
    if (has_pair) {
        WqPair pr;
        pr.slot = 0;
        pr.meta = 0;
        pr.s = -1;
        pr.h = h;
        pr.pad = 0;
        if (tk < cu[s + 1] && c.bad[s] != gen) {
            const int st = c.wstart[s * H + h];
            if (st >= 0) {
                const int64_t t_in_seq = tk - cu[s];
                pr.slot = slot_of(c, s, h, st + t_in_seq);
                pr.meta = c.meta[pr.slot];
                pr.s = s;
                if (t_in_seq == 0) {          // commit the new length and stream end
                    c.len[s * H + h] = st + (cu[s + 1] - cu[s]);
                    c.end[s * H + h] = c.wend[s * H + h];
                }
            }
        }
        pairs[i] = pr;
    }
    __syncthreads();
    // Sort the written pairs by width, so the lanes of a warp mostly share one code path.
    if (warp == 0) {
        const int n_pairs = Tc * HGc;
        int base = 0;
        for (int cls = 0; cls < 4; ++cls) {
            for (int i0 = 0; i0 < n_pairs; i0 += 32) {
                const int ii = i0 + lane;
                const bool in = ii < n_pairs && pairs[ii].s >= 0 && (int)(pairs[ii].meta & 3u) == cls;
                const uint32_t m = __ballot_sync(0xffffffffu, in);
                if (in) order[base + __popc(m & ((1u << lane) - 1u))] = (uint8_t)ii;
                base += __popc(m);
            }
        }
        if (lane == 0) n_written = base;
    }
    __syncthreads();
    if (!mbar_wait(&bar, 0, c.status)) return;

    // LPV adjacent lanes per vector: vector vi is pair order[vi / 2], K (even) or V (odd);
    // the lanes of a warp take consecutive vectors of the width-sorted list
    constexpr int LPV = (D == 128) ? kWqLanesPerVec : 1;
    const int n_vec = 2 * n_written;
    for (int t = tid; t < n_vec * LPV; t += kWqThreads) {
        const int vi = t / LPV, half = t % LPV;
        const int pi = order[vi >> 1], part = vi & 1;
        const WqPair pr = pairs[pi];
        const int b = 2 << (pr.meta & 3u);
        const uint4 *src = reinterpret_cast<const uint4 *>((part ? sv : sk) + pi * D);
        lane_vector<D, LPV>(c, src, b, rec_loc(c, pr.s, pr.h, (pr.meta & ~15u) + part * (b * D / 8)), pr.slot, part,
                            lane & 7, half);
    }
}

// Short appends (decode steps): one CTA of 256 threads per sequence does the scan and the
// quantization of all the sequence's new (token, head) pairs in one launch (append_seq).
// Same results as the scan + quantize pair of kernels.
template <int D>
__global__ void __launch_bounds__(256)
write_append_kernel(CacheView c, const __half *__restrict__ k, const __half *__restrict__ v,
                    const uint8_t *__restrict__ bits, const int32_t *__restrict__ cu, int64_t n_tok,
                    uint32_t gen)
{
    __shared__ AppendShared as;
    pdl_wait();
    pdl_trigger();
    append_seq<D>(c, k, v, bits, cu, n_tok, gen, nullptr, blockIdx.x, as);
}

} // namespace

cudaError_t launch_write(kvq_cache *cache, const __half *k, const __half *v,
                         const uint8_t *bits, const int32_t *cu, int64_t n_tok, cudaStream_t st)
{
    const CacheView &c = cache->view;
    const uint32_t gen = ++cache->write_gen;
    cudaError_t le = cudaSuccess;
    profile_before(st);
    if (n_tok > 0 && n_tok <= 2 * (int64_t)c.B && n_tok <= 4096) {
        // short append (decode steps): scan and quantize in one launch, a CTA per sequence
        if (c.D == 128)
            le = launch_pdl(write_append_kernel<128>, dim3(c.B), dim3(256), 0, st, c, k, v, bits, cu, n_tok, gen);
        else
            le = launch_pdl(write_append_kernel<64>, dim3(c.B), dim3(256), 0, st, c, k, v, bits, cu, n_tok, gen);
        profile_after(st);
        return le != cudaSuccess ? le : cudaGetLastError();
    }
    {
        const int64_t groups = (int64_t)c.B * c.H;
        // a warp per (sequence, head) for short appends (decode steps), a block for long ones
        if (n_tok <= 64 * (int64_t)c.B) {
            const int64_t blocks = (groups + 7) / 8;
            le = launch_pdl(write_scan_kernel<32>, dim3((unsigned)blocks), dim3(256), 0, st, c, bits, cu, n_tok, gen);
        } else {
            // chunks of 1024 tokens per (sequence, head); no sequence has more chunks than
            // the cache's largest capacity allows (a longer write fails its capacity check)
            const int n_chunks = (int)std::max<int64_t>(1, std::min<int64_t>((n_tok + kScanChunk - 1) / kScanChunk,
                                                                                 cache->scan_chunks));
            le = launch_pdl(write_scan_chunk_kernel, dim3((unsigned)(groups * n_chunks)), dim3(kScanChunkThreads), 0, st,
                            c, bits, cu, n_tok, gen, cache->scan_flags, n_chunks);
        }
        if (le != cudaSuccess) return le;
    }
    if (n_tok > 0) {
        // tiles of T tokens x HG heads, at most kWqHalves values per tensor; one token per
        // tile when the call is too short to give every SM a few tiles
        const int HG = std::min(c.H, kWqHalves / c.D);
        int T = std::max(1, kWqHalves / (HG * c.D));
        if (n_tok < (int64_t)T * 2 * num_sms()) T = 1;
        const dim3 grid((unsigned)((n_tok + T - 1) / T), (unsigned)((c.H + HG - 1) / HG));

        const size_t smem = 2 * kWqHalves * sizeof(__half);
        le = (c.D == 128) ? ensure_smem_attr((const void *)write_quant_kernel<128>, smem)
                          : ensure_smem_attr((const void *)write_quant_kernel<64>, smem);
        if (le != cudaSuccess) return le;
        if (c.D == 128)
            le = launch_pdl(write_quant_kernel<128>, grid, dim3(kWqThreads), smem, st, c, k, v, cu, n_tok, gen, T, HG);
        else
            le = launch_pdl(write_quant_kernel<64>, grid, dim3(kWqThreads), smem, st, c, k, v, cu, n_tok, gen, T, HG);
        if (le != cudaSuccess) return le;
    }
    profile_after(st);
    return cudaGetLastError();
}

} // namespace kvq
