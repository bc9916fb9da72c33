// Quantize-on-write (TriRoute paper review page, section 3, Eq. 4).
//
// Two launches per kvq_write call:
//   write_scan_kernel   a warp (short appends) or a block (long ones) per (sequence, head):
//                       validates capacity and widths (a bad width rejects the sequence's
//                       write for every head) and assigns each new token's record offset
//                       (prefix sum of record sizes b*D/4 in token order).
//   write_quant_kernel  one warp per (token, head): for K and for V, min/max over the
//                       head_dim values, s = (max - min)/(2^b - 1), z = min, codes
//                       rint((x - z)/s) in IEEE fp32 round-to-nearest-even (s == 0 -> 0),
//                       packed LSB-first into the record; (s, z) into the side table;
//                       commits the new length and stream end of accepted sequences.
// HBM traffic per (token, head): reads 2*D*2 bytes, writes b*D/4 + 16 + 4 bytes.
#include "kvq_internal.cuh"

namespace kvq {
namespace {

// TPS threads per (sequence, head): validates the call's widths of its head (a bad entry
// marks the sequence bad for this call, so no head of it is written), checks capacity,
// and assigns the new tokens' record offsets with a parallel prefix sum of the record
// sizes b*D/4. The new length/end are committed by the quantize kernel, which sees the
// per-sequence verdict of every head.
template <int TPS>
__global__ void __launch_bounds__(256)
write_scan_kernel(CacheView c, const uint8_t *__restrict__ bits, const int32_t *__restrict__ cu,
                  int64_t n_tok, uint32_t gen)
{
    constexpr int PER = 8;                       // tokens per thread per pass
    constexpr int WARPS = TPS / 32;
    __shared__ uint32_t wsum[256 / 32];
    const int tid = threadIdx.x % TPS, lane = threadIdx.x & 31;
    const int grp = threadIdx.x / TPS, wig = tid >> 5;     // group in block, warp in group
    const int64_t gsh = (int64_t)blockIdx.x * (256 / TPS) + grp;
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
        c.wstart[sh] = L0;
        c.wend[sh] = off;
    }
}

// D/4 lanes quantize one vector (4 channels per lane); a warp covers K and V of one
// (token, head): sequentially for D = 128, side by side for D = 64.
template <int D>
__global__ void write_quant_kernel(CacheView c, const __half *__restrict__ k,
                                   const __half *__restrict__ v, const uint8_t *__restrict__ bits,
                                   const int32_t *__restrict__ cu, int64_t n_tok, uint32_t gen)
{
    constexpr int VL = D / 4;            // lanes per vector
    constexpr int PER_ITER = 32 / VL;    // vectors per warp iteration
    const int lane = threadIdx.x & 31;
    const int li = lane % VL;
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int H = c.H;
    if (warp >= n_tok * H) return;
    const int64_t tk = warp / H;
    const int h = (int)(warp % H);

    // sequence of token tk: last s with cu[s] <= tk
    int lo = 0, hi = c.B;            // invariant: cu[lo] <= tk < cu[hi]
    while (hi - lo > 1) {
        int mid = (lo + hi) >> 1;
        if (cu[mid] <= tk) lo = mid;
        else hi = mid;
    }
    const int s = lo;
    if (tk >= cu[s + 1]) return;     // cu_seqlens violated its contract (flagged by the scan)
    const int start = c.wstart[s * H + h];
    if (start < 0 || c.bad[s] == gen) return;     // this sequence's write was rejected
    if (tk == cu[s] && lane == 0) {               // commit the new length and stream end
        c.len[s * H + h] = start + (cu[s + 1] - cu[s]);
        c.end[s * H + h] = c.wend[s * H + h];
    }
    const int64_t j = start + (tk - cu[s]);
    const int64_t slot = slot_of(c, s, h, j);
    const uint32_t meta = c.meta[slot];
    const int wc = meta & 3u;
    const int b = 2 << wc;           // 2, 4, 8, 16
    uint8_t *rec = stream_of(c, s, h) + (meta & ~15u);
    const int part_bytes = b * D / 8;

    float s_part[2] = {1.0f, 1.0f}, z_part[2] = {0.0f, 0.0f};
#pragma unroll
    for (int it = 0; it < 2 / PER_ITER; ++it) {
        const int part = it * PER_ITER + lane / VL;   // 0 = K, 1 = V
        const __half *src = (part == 0 ? k : v) + (tk * H + h) * D + 4 * li;
        const uint2 raw = *reinterpret_cast<const uint2 *>(src);
        uint8_t *dst = rec + part * part_bytes;
        if (b == 16) {
            *reinterpret_cast<uint2 *>(dst + 8 * li) = raw;
            continue;
        }
        const __half2 h01 = *reinterpret_cast<const __half2 *>(&raw.x);
        const __half2 h23 = *reinterpret_cast<const __half2 *>(&raw.y);
        float x[4] = {__low2float(h01), __high2float(h01), __low2float(h23), __high2float(h23)};
        float mn = fminf(fminf(x[0], x[1]), fminf(x[2], x[3]));
        float mx = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
#pragma unroll
        for (int d = VL / 2; d >= 1; d >>= 1) {
            mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, d));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, d));
        }
        const float top = (float)((1u << b) - 1u);
        // zeros are stored as +0 (the min scan may meet -0 or +0 first)
        const float sc = __fadd_rn(__fdiv_rn(__fsub_rn(mx, mn), top), 0.0f);
        const float z = __fadd_rn(mn, 0.0f);
        uint32_t packed = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            uint32_t code = 0;
            if (sc != 0.0f) {
                float r = rintf(__fdiv_rn(__fsub_rn(x[e], z), sc));
                r = fminf(fmaxf(r, 0.0f), top);
                code = (uint32_t)r;
            }
            packed |= code << (e * b);
        }
        if (b == 2) dst[li] = (uint8_t)packed;
        else if (b == 4) reinterpret_cast<uint16_t *>(dst)[li] = (uint16_t)packed;
        else reinterpret_cast<uint32_t *>(dst)[li] = packed;
        s_part[it] = sc;
        z_part[it] = z;
    }
    // side entry (s_K, z_K, s_V, z_V): K values live in lane 0, V values in lane 0 (D = 128,
    // second iteration) or lane VL (D = 64)
    float sK, zK, sV, zV;
    if (PER_ITER == 1) {
        sK = s_part[0];
        zK = z_part[0];
        sV = s_part[1 % (2 / PER_ITER)];
        zV = z_part[1 % (2 / PER_ITER)];
    } else {
        sK = __shfl_sync(0xffffffffu, s_part[0], 0);
        zK = __shfl_sync(0xffffffffu, z_part[0], 0);
        sV = __shfl_sync(0xffffffffu, s_part[0], VL);
        zV = __shfl_sync(0xffffffffu, z_part[0], VL);
    }
    if (lane == 0) c.side[slot] = make_float4(sK, zK, sV, zV);
}

} // namespace

cudaError_t launch_write(kvq_cache *cache, const __half *k, const __half *v,
                         const uint8_t *bits, const int32_t *cu, int64_t n_tok, cudaStream_t st)
{
    const CacheView &c = cache->view;
    const uint32_t gen = ++cache->write_gen;
    profile_before(st);
    {
        const int64_t groups = (int64_t)c.B * c.H;
        // a warp per (sequence, head) for short appends (decode steps), a block for long ones
        if (n_tok <= 64 * (int64_t)c.B) {
            const int64_t blocks = (groups + 7) / 8;
            write_scan_kernel<32><<<(unsigned)blocks, 256, 0, st>>>(c, bits, cu, n_tok, gen);
        } else {
            write_scan_kernel<256><<<(unsigned)groups, 256, 0, st>>>(c, bits, cu, n_tok, gen);
        }
    }
    if (n_tok > 0) {
        const int64_t warps = n_tok * c.H;
        const int threads = 256;
        const int64_t blocks = (warps * 32 + threads - 1) / threads;
        if (c.D == 128)
            write_quant_kernel<128><<<(unsigned)blocks, threads, 0, st>>>(c, k, v, bits, cu, n_tok, gen);
        else
            write_quant_kernel<64><<<(unsigned)blocks, threads, 0, st>>>(c, k, v, bits, cu, n_tok, gen);
    }
    profile_after(st);
    return cudaGetLastError();
}

} // namespace kvq
