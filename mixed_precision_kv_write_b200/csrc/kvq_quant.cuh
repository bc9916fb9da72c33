// Quantize-on-write helpers shared by the write kernels and the fused decode step
// (TriRoute paper review page, section 3, Eq. 4): per (token, head) vector of D fp16
// values, min/max, s = (max - min)/(2^b - 1), z = min, codes rint((x - z)/s) in IEEE fp32
// round-to-nearest-even (s == 0 -> 0), packed LSB-first; b = 16 keeps the fp16 bits.
#pragma once

#include "kvq_internal.cuh"

namespace kvq {

// Codes are rint(fl(u / s)) with u = fl(x - z), clamped to [0, 2^b - 1].
// The correctly rounded quotient fl(u / s) is formed with Markstein's correction
// (P. Markstein, "Computation of elementary functions on the IBM RISC System/6000
// processor", IBM J. Res. Dev. 34(1), 1990): with y = RN(1/s) and the faithful q0 = RN(u y),
// the remainder r = u - s q0 is exact in one FMA, and RN(q0 + r y) = RN(u / s). Because
// 0 <= u <= fl(max - min) the quotient lies in [0, 2^b - 1 + 2^-14], so rint never leaves the
// code range. rint is taken by adding 1.5 * 2^23: for 0 <= q < 2^22 the sum is
// 1.5 * 2^23 + rint(q) exactly (round-to-nearest-even), the integer in the low mantissa bits.
// A NaN quotient (NaN or infinite inputs) is caught by a running sum and the lane falls
// back to the plain clamped formula, which maps it to code 0.
constexpr float kRoundMagic = 12582912.0f;          // 1.5 * 2^23
constexpr uint32_t kRoundMagicBits = 0x4B400000u;

// Quantizes a lane's NC chunks of 8 fp16 values to BITS-bit codes. Chunk j holds channels
// 8 * (j * VL + li) .. + 7 of the vector, so its 8 codes fill BITS bytes of the part at byte
// BITS * (j * VL + li), and the VL lanes of a vector store adjacent chunks.
template <int BITS, int NC, int VL>
__device__ __forceinline__ void quant_store(const uint4 (&raw)[NC], float z, float sc,
                                            const RecLoc &dst, int li)
{
    uint32_t w[NC][2];
#pragma unroll
    for (int j = 0; j < NC; ++j) w[j][0] = w[j][1] = 0u;
    if (sc != 0.0f) {
        // Two values per instruction: the packed fp32 operations (FADD2/FMUL2/FFMA2) round
        // each half exactly as the scalar operation would, so the codes are unchanged.
        const float y = __frcp_rn(sc);
        const float2 y2 = make_float2(y, y), nz2 = make_float2(-z, -z), ns2 = make_float2(-sc, -sc);
        const float2 mg2 = make_float2(kRoundMagic, kRoundMagic);
        float2 probe = make_float2(0.0f, 0.0f);
#pragma unroll
        for (int j = 0; j < NC; ++j) {
            const __half2 *h2 = reinterpret_cast<const __half2 *>(&raw[j]);
#pragma unroll
            for (int e = 0; e < 4; ++e) {                 // channels 2e, 2e + 1 of the chunk
                const float2 x = __half22float2(h2[e]);
                const float2 u = __fadd2_rn(x, nz2);         // x - z
                const float2 q0 = __fmul2_rn(u, y2);
                const float2 r = __ffma2_rn(ns2, q0, u);     // u - s * q0, exact
                const float2 q = __ffma2_rn(r, y2, q0);      // RN(u / s)
                const float2 t = __fadd2_rn(q, mg2);
                probe = __fadd2_rn(probe, q);
                // code << shift; the 1.5 * 2^23 bits are taken off below
                w[j][(2 * e * BITS) >> 5] += __float_as_uint(t.x) << ((2 * e * BITS) & 31);
                w[j][((2 * e + 1) * BITS) >> 5] += __float_as_uint(t.y) << (((2 * e + 1) * BITS) & 31);
            }
        }
        const float nan_probe = probe.x + probe.y;
        constexpr int kWordBits = BITS * 8 < 32 ? BITS * 8 : 32;   // code bits per word
        uint32_t magic = 0u;
#pragma unroll
        for (int sh = 0; sh < kWordBits; sh += BITS) magic += kRoundMagicBits << sh;
#pragma unroll
        for (int j = 0; j < NC; ++j) {
            w[j][0] -= magic;
            if (BITS == 8) w[j][1] -= magic;
        }
        if (nan_probe != nan_probe) {
            const float top = (float)((1u << BITS) - 1u);
#pragma unroll
            for (int j = 0; j < NC; ++j) {
                const __half2 *h2 = reinterpret_cast<const __half2 *>(&raw[j]);
                w[j][0] = w[j][1] = 0u;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float x = (e & 1) ? __high2float(h2[e >> 1]) : __low2float(h2[e >> 1]);
                    const float c = fminf(fmaxf(rintf(__fdiv_rn(__fsub_rn(x, z), sc)), 0.0f), top);
                    w[j][(e * BITS) >> 5] |= __float2uint_rz(c) << ((e * BITS) & 31);
                }
            }
        }
    }
#pragma unroll
    for (int j = 0; j < NC; ++j) {
        const int chunk = j * VL + li;
        uint8_t *d = dst.at((uint32_t)(BITS * chunk));
        if (BITS == 8) *reinterpret_cast<uint2 *>(d) = make_uint2(w[j][0], w[j][1]);
        else if (BITS == 4) *reinterpret_cast<uint32_t *>(d) = w[j][0];
        else *reinterpret_cast<uint16_t *>(d) = (uint16_t)w[j][0];
    }
}

// min and max of a vector spread over VL adjacent lanes (NC 8-value chunks per lane), in
// fp16 (exact); (min, -max) travel as one half2 through the shuffles. Every lane of the
// warp takes part.
template <int NC, int VL>
__device__ __forceinline__ __half2 vec_minmax(const uint4 (&raw)[NC])
{
    const __half2 (&h2)[4 * NC] = *reinterpret_cast<const __half2 (*)[4 * NC]>(raw);
    __half2 lo2 = h2[0], hi2 = h2[0];
#pragma unroll
    for (int e = 1; e < 4 * NC; ++e) {
        lo2 = __hmin2(lo2, h2[e]);
        hi2 = __hmax2(hi2, h2[e]);
    }
    __half2 mm = __halves2half2(__hmin(__low2half(lo2), __high2half(lo2)),
                                __hneg(__hmax(__low2half(hi2), __high2half(hi2))));
#pragma unroll
    for (int d = VL / 2; d >= 1; d >>= 1) {
        const uint32_t o = __shfl_xor_sync(0xffffffffu, *reinterpret_cast<uint32_t *>(&mm), d);
        mm = __hmin2(mm, *reinterpret_cast<const __half2 *>(&o));
    }
    return mm;
}

// This lane's share of one vector's record part at `dst` (b-bit codes, or the fp16 values
// for b = 16) and, from the vector's first lane, its (s, z) side entry.
template <int NC, int VL>
__device__ __forceinline__ void vec_store(const CacheView &c, const uint4 (&raw)[NC], __half2 mm, int b,
                                          const RecLoc &dst, int64_t slot, int part, int li)
{
    float sc = 1.0f, z = 0.0f;
    if (b == 16) {
#pragma unroll
        for (int j = 0; j < NC; ++j) *reinterpret_cast<uint4 *>(dst.at(16u * (j * VL + li))) = raw[j];
    } else {
        const float mn = __low2float(mm), mx = -__high2float(mm);
        const float top = (float)((1u << b) - 1u);
        // zeros are stored as +0 (the min scan may meet -0 or +0 first)
        sc = __fadd_rn(__fdiv_rn(__fsub_rn(mx, mn), top), 0.0f);
        z = __fadd_rn(mn, 0.0f);
        if (b == 8) quant_store<8, NC, VL>(raw, z, sc, dst, li);
        else if (b == 4) quant_store<4, NC, VL>(raw, z, sc, dst, li);
        else quant_store<2, NC, VL>(raw, z, sc, dst, li);
    }
    if (li == 0) reinterpret_cast<float2 *>(&c.side[slot])[part] = make_float2(sc, z);
}

// Per-head results of append_seq, in shared memory (heads beyond kAppendHeads use the
// cache's arrays in global memory).
constexpr int kAppendHeads = 64;
constexpr int kAppendMeta = 512;                 // (token, head) record offsets kept on chip
struct AppendShared {
    int bad;                                     // a bad width in the sequence's new tokens
    int32_t wstart[kAppendHeads];                // write start (-1: refused), per head
    uint32_t wend[kAppendHeads];                 // stream end after the write, per head
    int32_t len[kAppendHeads];                   // length on return, per head
    uint32_t end[kAppendHeads];                  // stream end on return, per head
    uint32_t meta[kAppendMeta];                  // token i, head h at i * H + h, when n * H fits
};

// Appends the call's tokens of sequence s (rows cu[s] .. cu[s+1]-1 of k, v, bits) for
// every head; called by all threads of a block of 256 (it synchronizes the block).
// Every load that does not depend on another goes out first: the sequence's range,
// roll-back position and slot geometry, each head's length and stream end, the first 32
// widths of each head and this thread's first K/V chunks. Phase 1, a warp per head: the
// optional roll-back to positions[s] (the sequence keeps its first min(len, positions[s])
// tokens, as kvq_cache_truncate), then capacity, widths and record offsets (warp prefix
// sum) of the new tokens. Phase 2, after the block has seen every head's verdict: D/8
// lanes per vector quantize from the prefetched rows. A bad width refuses the sequence's
// write for every head; a capacity overflow refuses that head. On return the new lengths
// and stream ends are committed, visible to the whole block, and (heads below
// kAppendHeads) also in `as`. Inconsistent cu_seqlens leave the sequence untouched (status
// set; as.wstart[h] = -1).
template <int D>
__device__ __forceinline__ void append_seq(const CacheView &c, const __half *__restrict__ k,
                                           const __half *__restrict__ v, const uint8_t *__restrict__ bits,
                                           const int32_t *__restrict__ cu, int64_t n_tok, uint32_t gen,
                                           const int32_t *__restrict__ positions, int s, AppendShared &as)
{
    constexpr int VL = D / 8, VPW = 32 / VL;
    constexpr int kPre = 2;                      // vector passes whose rows are loaded up front
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int H = c.H;
    const int64_t t0 = cu[s], t1 = cu[s + 1];
    const int roll = positions ? positions[s] : -1;
    const int cap = c.cap[s];
    const int64_t sbase = c.slot_base[s];
    const int cpad = c.cap_pad[s];
    if (t0 < 0 || t1 < t0 || t1 > n_tok || (s == 0 && t0 != 0)) {   // block-uniform
        if (tid == 0) set_status(c.status, KVQ_ERR_DEVICE_CHECK);
        for (int h = tid; h < min(H, kAppendHeads); h += blockDim.x) {
            as.wstart[h] = -1;
            as.len[h] = c.len[s * H + h];
            as.end[h] = c.end[s * H + h];
        }
        __syncthreads();
        return;
    }
    const int n = (int)(t1 - t0);
    const int n_vec = 2 * n * H;                 // vector vi: pair vi / 2 = i * H + h, K or V
    const int li = lane % VL;
    const bool meta_on_chip = n * H <= kAppendMeta;
    // this thread's first kPre vector chunks
    uint4 pre[kPre];
#pragma unroll
    for (int p = 0; p < kPre; ++p) {
        const int vi = warp * VPW + lane / VL + p * 8 * VPW;
        pre[p] = make_uint4(0u, 0u, 0u, 0u);
        if (vi < n_vec) {
            const int pp = vi >> 1;
            pre[p] = reinterpret_cast<const uint4 *>((vi & 1 ? v : k) + ((t0 + pp / H) * H + pp % H) * D)[li];
        }
    }
    if (tid == 0) as.bad = 0;
    __syncthreads();
    for (int h = warp; h < H; h += 8) {
        const int sh = s * H + h;
        int L0 = c.len[sh];
        uint32_t off = c.end[sh];
        // the first 32 widths go out with the length
        int b_first = 0;
        if (lane < n) b_first = bits[(t0 + lane) * H + h];
        if (roll >= 0 && roll < L0) {             // roll back first (truncate semantics)
            off = c.meta[sbase + (int64_t)h * cpad + roll] & ~15u;
            L0 = roll;
        }
        __syncwarp();
        if (lane == 0) {
            c.len[sh] = L0;
            c.end[sh] = off;
            c.wstart[sh] = -1;
            if (h < kAppendHeads) {
                as.wstart[h] = -1;
                as.len[h] = L0;
                as.end[h] = off;
            }
        }
        if (n == 0) continue;
        if ((int64_t)L0 + n > cap) {
            if (lane == 0) set_status(c.status, KVQ_ERR_CAPACITY);
            continue;
        }
        const int64_t slot0 = sbase + (int64_t)h * cpad + L0;
        bool bad = false;
        for (int base = 0; base < n; base += 32) {
            const int i = base + lane;
            uint32_t sz = 0, wc = 0;
            if (i < n) {
                const int b = base == 0 ? b_first : bits[(t0 + i) * H + h];
                const int wcode = width_code(b);
                if (wcode < 0) bad = true;
                else {
                    wc = (uint32_t)wcode;
                    sz = (uint32_t)(b * D / 4);
                }
            }
            uint32_t incl = sz;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const uint32_t y = __shfl_up_sync(0xffffffffu, incl, d);
                if (lane >= d) incl += y;
            }
            if (i < n) {
                const uint32_t m = (off + incl - sz) | wc;
                c.meta[slot0 + i] = m;
                if (meta_on_chip) as.meta[i * H + h] = m;
            }
            off += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(&as.bad, 1);
        if (lane == 0) {
            if (map_pages(c, s, h, off)) {       // paged caches: pages for the new bytes
                c.wstart[sh] = L0;
                c.wend[sh] = off;
                if (h < kAppendHeads) {
                    as.wstart[h] = L0;
                    as.wend[h] = off;
                }
            } else {
                set_status(c.status, KVQ_ERR_CAPACITY);
            }
        }
    }
    __syncthreads();
    if (n == 0) return;                          // block-uniform
    if (as.bad) {                                // the sequence's write is refused for every head
        if (tid == 0) {
            c.bad[s] = gen;
            set_status(c.status, KVQ_ERR_BITS);
        }
        for (int h = tid; h < min(H, kAppendHeads); h += blockDim.x) as.wstart[h] = -1;
        __syncthreads();
        return;
    }
    int p = 0;
    for (int vb = warp * VPW; vb < n_vec; vb += 8 * VPW, ++p) {
        const int vi = vb + lane / VL;
        const bool in_range = vi < n_vec;
        const int pp = vi >> 1, part = vi & 1;
        const int i = pp / H, h = pp % H;
        uint4 raw[1] = {make_uint4(0u, 0u, 0u, 0u)};
        if (p < kPre) {
#pragma unroll
            for (int q = 0; q < kPre; ++q)
                if (q == p) raw[0] = pre[q];
        } else if (in_range) {
            raw[0] = reinterpret_cast<const uint4 *>((part ? v : k) + ((t0 + i) * H + h) * D)[li];
        }
        const __half2 mm = vec_minmax<1, VL>(raw);
        if (!in_range) continue;
        const int st = (h < kAppendHeads) ? as.wstart[h] : c.wstart[s * H + h];
        if (st < 0) continue;
        const int64_t slot = sbase + (int64_t)h * cpad + st + i;
        const uint32_t meta = meta_on_chip ? as.meta[i * H + h] : c.meta[slot];
        const int b = 2 << (meta & 3u);
        vec_store<1, VL>(c, raw, mm, b, rec_loc(c, s, h, (meta & ~15u) + part * (b * D / 8)), slot, part, li);
    }
    __syncthreads();
    for (int h = tid; h < H; h += blockDim.x) {  // commit the new lengths and stream ends
        const int st = (h < kAppendHeads) ? as.wstart[h] : c.wstart[s * H + h];
        if (st >= 0) {
            const uint32_t e = (h < kAppendHeads) ? as.wend[h] : c.wend[s * H + h];
            c.len[s * H + h] = st + n;
            c.end[s * H + h] = e;
            if (h < kAppendHeads) {
                as.len[h] = st + n;
                as.end[h] = e;
            }
        }
    }
    __syncthreads();
}

} // namespace kvq
