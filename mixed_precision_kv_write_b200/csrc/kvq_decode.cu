// Routed decode attention (TriRoute paper review page, section 3, Eq. 2) over the
// mixed-precision cache of Eq. 4: one query per (sequence, head) at t = len - 1.
//
// Three launches:
//   decode_sched_kernel   mode-aware scheduler: skip heads and empty sequences get no
//                         work, local heads are clamped to keys [max(0, t - w), t], full
//                         heads read [0, t]; each range is cut into near-equal items of at
//                         most 512 keys, listed on the device (no host round trip).
//   decode_splitk_kernel  three CTAs per SM. A producer warp walks the CTA's items in
//                         stages of at most 128 keys and 24 KB of records: it keeps a ring
//                         of record-offset windows fetched ahead, cuts each stage at the
//                         byte budget, sorts the stage's keys by width once (so the
//                         consumers' 4-key steps rarely mix widths), and streams the stage's
//                         contiguous record bytes, side entries and (for a new item) the
//                         query into shared memory with 1-D bulk copies (2-stage mbarrier
//                         pipeline). Five consumer warps split each stage's keys: 8 lanes
//                         per key, 16 channels per lane, K dot product -> logit -> online
//                         softmax kept per 8-lane group -> V accumulation, all in registers;
//                         the groups' states are merged once per item into a partial
//                         (m, l, o[D]).
//   decode_combine_kernel log-sum-exp merge of the item partials of each (sequence, head),
//                         one thread per channel; zeros for skip heads and empty sequences.
//
// Arithmetic. With codes c, scale s and zero z (Eq. 4):
//   q . deq(k_j) = s_j * (q . c_j) + z_j * sum(q)         (one dot product on integer codes)
//   sum_j p_j deq(v_j) = sum_j (p_j s_j) c_j + (sum_j p_j z_j) * 1
// Codes are never converted with an int->float instruction: a b-bit field masked in place
// inside a 32-bit word (bits below 23) IS the fp32 subnormal c * 2^(pos - 149), and FFMA
// multiplies subnormal operands exactly at full rate. The position scale 2^(pos - 149) is
// folded into the other operand (q for K, the softmax weight for V), which keeps the
// unpack at one LOP3 per code. fp32 subnormals must not be flushed: build without
// -ftz / fast-math.
#include <cstdio>
#include <mutex>

#include "kvq_internal.cuh"

namespace kvq {
namespace {

constexpr int kConsumerWarps = 5;
constexpr int kThreads = 32 * (kConsumerWarps + 1);
constexpr int kStages = 2;                        // record stages in flight per CTA
constexpr int kWin = kDecodeWindowKeys;           // keys per window of record offsets
constexpr uint32_t kStageRecBytes = 24576;        // record bytes per stage, at most
constexpr int kPermSlots = kWin + 32;             // width-sorted keys padded to whole chunks
constexpr int kMetaSlots = 6;                     // windows of record offsets fetched ahead
constexpr int kMetaWords = kWin + 8;
constexpr int kNewItem = 1, kLastSub = 2;         // stage flags
constexpr uint32_t kReadEndFromMeta = 0xFFFFFFFFu;
constexpr uint32_t kValid = 0x80000000u;

// q'_b[k] = q[k] * 2^(60 - pos_b(k)); the code field of channel k sits at pos_b(k) after
// unpack: b = 2 -> 2*(k % 8), b = 4 -> 4*(k % 4), b = 8 -> 0. Dot products over codes
// come out scaled by 2^(60 - 149) = 2^-89; over native fp16 values by 2^60.
constexpr float kQScale = 1152921504606846976.0f;      // 2^60
constexpr float kDotCodeUnscale = 618970019642690137449562112.0f;  // 2^89
constexpr float kDotNativeUnscale = 8.673617379884035e-19f;        // 2^-60
// V weights: w' = p * s * 2^(100 - pos); accumulators hold o * 2^-49.
constexpr float kWScale = 1267650600228229401496703205376.0f;      // 2^100
constexpr float kONativeScale = 1.7763568394002505e-15f;           // 2^-49
constexpr float kOUnscale = 562949953421312.0f;                    // 2^49

template <int D>
struct Stage {
    // width-sorted keys in class-pure chunks: kValid | (key << 16) | offset in rec;
    // padding entries are 0
    uint32_t perm[kPermSlots];
    int32_t info[4];         // item index, keys in the stage, flags, chunks
    int32_t cls_chunk[8];    // first chunk of each width class (b = 2, 4, 8, 16), [4] = chunks
    __half q[D];             // the item's query (copied with the item's first stage)
    float4 side[kWin];       // (s_K, z_K, s_V, z_V) per key, token order
    alignas(16) uint8_t rec[kStageRecBytes];
};

// one window of record offsets: meta of keys [ja, ...) of an item's stream
struct alignas(16) MetaSlot {
    uint32_t meta[kMetaWords];
    int32_t it, j, j1, ja;
    uint32_t end_off, first;
    int64_t sbase;
    int32_t sh, pad;
};

template <int D>
struct DecodeSmem {
    Stage<D> st[kStages];
    MetaSlot ms[kMetaSlots];
    float red_o[kConsumerWarps][D];
    float red_m[kConsumerWarps], red_l[kConsumerWarps], red_pz[kConsumerWarps];
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t mfull[kMetaSlots];
};

__device__ __forceinline__ float fld(uint32_t bits) { return __uint_as_float(bits); }

__global__ void decode_sched_kernel(CacheView c, const uint8_t *__restrict__ modes, int w,
                                    DecodeWork wk)
{
    __shared__ int warp_tot[32];
    __shared__ int carry_sh;
    pdl_wait();
    pdl_trigger();
    const int HQ = c.H * c.G;                 // query heads; query head hq reads KV head hq / G
    const int BH = c.B * HQ;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    if (tid == 0) carry_sh = 0;
    __syncthreads();
    for (int base = 0; base < BH; base += blockDim.x) {
        const int i = base + tid;
        int cnt = 0, lo = 0, hi = 0, L = 0;
        int64_t sb = 0;
        uint32_t end_i = 0;
        if (i < BH) {
            // every load of this head up front: one round trip before the scan
            const int s = i / HQ, h = (i % HQ) / c.G, shk = s * c.H + h;
            const int m = modes[i];
            L = c.len[shk];
            end_i = c.end[shk];
            sb = slot_of(c, s, h, 0);
            if (m > KVQ_MODE_FULL) {
                set_status(c.status, KVQ_ERR_MODE);
            } else if (m != KVQ_MODE_SKIP && L > 0) {
                hi = L;
                lo = (m == KVQ_MODE_LOCAL) ? max(0, L - 1 - w) : 0;
                cnt = (hi - lo + kDecodeItemKeys - 1) / kDecodeItemKeys;
            }
        }
        int incl = cnt;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, incl, d);
            if (lane >= d) incl += y;
        }
        if (lane == 31) warp_tot[wid] = incl;
        __syncthreads();
        if (wid == 0) {
            int t = (lane < (int)(blockDim.x >> 5)) ? warp_tot[lane] : 0;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                int y = __shfl_up_sync(0xffffffffu, t, d);
                if (lane >= d) t += y;
            }
            warp_tot[lane] = t;   // inclusive over warps
        }
        __syncthreads();
        const int carry = carry_sh;
        const int first = carry + (wid > 0 ? warp_tot[wid - 1] : 0) + incl - cnt;
        if (i < BH) {
            wk.head_first[i] = first;
            wk.head_cnt[i] = cnt;
            if (cnt > 0) {
                const int n = hi - lo, per = n / cnt, rem = n % cnt;
                int j0 = lo;
                for (int k = 0; k < cnt; ++k) {               // near-equal, non-empty items
                    DecodeItem it;
                    it.sh = i;
                    it.j0 = j0;
                    it.j1 = j0 + per + (k < rem ? 1 : 0);
                    j0 = it.j1;
                    // the stream end for the item ending at the last token; else the
                    // producer reads the offset of key j1 itself
                    it.end_off = (it.j1 < L) ? kReadEndFromMeta : end_i;
                    it.sbase = sb;
                    wk.items[first + k] = it;
                }
            }
        }
        __syncthreads();
        if (tid == 0) carry_sh = carry + warp_tot[(blockDim.x >> 5) - 1];
        __syncthreads();
    }
    if (tid == 0) *wk.count = carry_sh;
}

// ---- per-width dot products and accumulations for one lane's 16 channels ----------
// Channels c and c + 8 of the lane travel as one float2, so every FMA is a packed FFMA2
// (two fp32 FMAs, each with the rounding of fmaf, subnormal operands kept).
struct QRegs {
    float2 q2[8], q4[8], q8[8];   // (q[j], q[j + 8]) * 2^(60 - pos_b)
};

__device__ __forceinline__ float2 fpair(uint32_t a, uint32_t b) { return make_float2(fld(a), fld(b)); }
__device__ __forceinline__ float2 bcast(float a) { return make_float2(a, a); }

__device__ __forceinline__ float dot_codes2(const QRegs &q, uint32_t x)
{
    const uint32_t y = x >> 16;                 // channels 8..15
    float2 a[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const uint32_t m = 3u << (2 * k);
        a[k & 1] = __ffma2_rn(q.q2[k], fpair(x & m, y & m), a[k & 1]);
    }
    return (a[0].x + a[1].x) + (a[0].y + a[1].y);
}

__device__ __forceinline__ float dot_codes4(const QRegs &q, uint2 x)
{
    const uint32_t lo0 = x.x, hi0 = x.x >> 16, lo1 = x.y, hi1 = x.y >> 16;
    float2 a[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const uint32_t m = 15u << (4 * k);
        a[0] = __ffma2_rn(q.q4[k], fpair(lo0 & m, lo1 & m), a[0]);          // channels k, 8 + k
        a[1] = __ffma2_rn(q.q4[4 + k], fpair(hi0 & m, hi1 & m), a[1]);      // 4 + k, 12 + k
    }
    return (a[0].x + a[1].x) + (a[0].y + a[1].y);
}

__device__ __forceinline__ float dot_codes8(const QRegs &q, uint4 x)
{
    float2 a[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const uint32_t sel = 0x4440 + e;
        a[0] = __ffma2_rn(q.q8[e], fpair(__byte_perm(x.x, 0u, sel), __byte_perm(x.z, 0u, sel)), a[0]);
        a[1] = __ffma2_rn(q.q8[4 + e], fpair(__byte_perm(x.y, 0u, sel), __byte_perm(x.w, 0u, sel)), a[1]);
    }
    return (a[0].x + a[1].x) + (a[0].y + a[1].y);
}

__device__ __forceinline__ float dot_native(const QRegs &q, uint4 x0, uint4 x1)
{
    const uint32_t w[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
    float2 a[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
    for (int h = 0; h < 4; ++h) {               // word h: channels 2h, 2h + 1; word h + 4: + 8
        const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&w[h]));
        const float2 g = __half22float2(*reinterpret_cast<const __half2 *>(&w[h + 4]));
        a[0] = __ffma2_rn(q.q8[2 * h], make_float2(f.x, g.x), a[0]);
        a[1] = __ffma2_rn(q.q8[2 * h + 1], make_float2(f.y, g.y), a[1]);
    }
    return (a[0].x + a[1].x) + (a[0].y + a[1].y);
}

__device__ __forceinline__ void acc_codes2(float2 (&o)[8], float wv, uint32_t x)
{
    const uint32_t y = x >> 16;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const float wk = wv * __uint_as_float((127u - 2u * k) << 23);   // wv * 2^-2k
        const uint32_t m = 3u << (2 * k);
        o[k] = __ffma2_rn(bcast(wk), fpair(x & m, y & m), o[k]);
    }
}

__device__ __forceinline__ void acc_codes4(float2 (&o)[8], float wv, uint2 x)
{
    const uint32_t hi0 = x.x >> 16, hi1 = x.y >> 16;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const float2 wk = bcast(wv * __uint_as_float((127u - 4u * k) << 23));   // wv * 2^-4k
        const uint32_t m = 15u << (4 * k);
        o[k] = __ffma2_rn(wk, fpair(x.x & m, x.y & m), o[k]);
        o[4 + k] = __ffma2_rn(wk, fpair(hi0 & m, hi1 & m), o[4 + k]);
    }
}

__device__ __forceinline__ void acc_codes8(float2 (&o)[8], float wv, uint4 x)
{
    const float2 w2 = bcast(wv);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const uint32_t sel = 0x4440 + e;
        o[e] = __ffma2_rn(w2, fpair(__byte_perm(x.x, 0u, sel), __byte_perm(x.z, 0u, sel)), o[e]);
        o[4 + e] = __ffma2_rn(w2, fpair(__byte_perm(x.y, 0u, sel), __byte_perm(x.w, 0u, sel)), o[4 + e]);
    }
}

__device__ __forceinline__ void acc_native(float2 (&o)[8], float wv, uint4 x0, uint4 x1)
{
    const uint32_t w[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
    const float2 w2 = bcast(wv);
#pragma unroll
    for (int h = 0; h < 4; ++h) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&w[h]));
        const float2 g = __half22float2(*reinterpret_cast<const __half2 *>(&w[h + 4]));
        o[2 * h] = __ffma2_rn(w2, make_float2(f.x, g.x), o[2 * h]);
        o[2 * h + 1] = __ffma2_rn(w2, make_float2(f.y, g.y), o[2 * h + 1]);
    }
}

// merge the online-softmax state (m, l, pz, o) of this lane with the lane `mask` away
__device__ __forceinline__ void merge_state(float &m, float &l, float &pz, float2 (&o)[8], int mask)
{
    const float mp = __shfl_xor_sync(0xffffffffu, m, mask);
    const float lp = __shfl_xor_sync(0xffffffffu, l, mask);
    const float zp = __shfl_xor_sync(0xffffffffu, pz, mask);
    const float M = fmaxf(m, mp);
    const float fa = (m == -INFINITY) ? 0.f : exp2f(m - M);
    const float fb = (mp == -INFINITY) ? 0.f : exp2f(mp - M);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const float2 op = make_float2(__shfl_xor_sync(0xffffffffu, o[k].x, mask),
                                      __shfl_xor_sync(0xffffffffu, o[k].y, mask));
        o[k] = __ffma2_rn(op, bcast(fb), __fmul2_rn(o[k], bcast(fa)));
    }
    l = l * fa + lp * fb;
    pz = pz * fa + zp * fb;
    m = M;
}

struct KeyState {
    float m, l, pz;
    float2 o[8];      // (o[j], o[j + 8]) of the lane's 16 channels
};

// One key per 8-lane group (16 lanes x 4 groups for head_dim 64: 4 lanes x 8 groups), all
// of width class CLS (warp-uniform): K dot product on the codes, logit, online-softmax
// update of the group's state, V accumulation. Lanes of invalid entries only take part in
// the shuffles.
template <int D, int CLS>
__device__ __forceinline__ void process_key(KeyState &st, const QRegs &qr, float qsum, float qk_scale,
                                            const Stage<D> &sg, uint32_t ent, int gl)
{
    constexpr int GROUP = D / 16;
    const bool valid = (ent & kValid) != 0;
    const uint8_t *r = sg.rec + (ent & 0x7FFFu);
    float part = 0.f;
    if (valid) {
        if (CLS == 0) part = dot_codes2(qr, reinterpret_cast<const uint32_t *>(r)[gl]);
        else if (CLS == 1) part = dot_codes4(qr, reinterpret_cast<const uint2 *>(r)[gl]);
        else if (CLS == 2) part = dot_codes8(qr, reinterpret_cast<const uint4 *>(r)[gl]);
        else part = dot_native(qr, reinterpret_cast<const uint4 *>(r)[2 * gl],
                               reinterpret_cast<const uint4 *>(r)[2 * gl + 1]);
    }
#pragma unroll
    for (int d = 1; d < GROUP; d <<= 1) part += __shfl_xor_sync(0xffffffffu, part, d);
    if (!valid) return;
    const float4 sd = sg.side[(ent >> 16) & 127u];
    const float dot = (CLS == 3) ? part * kDotNativeUnscale : fmaf(sd.x, part * kDotCodeUnscale, sd.y * qsum);
    const float lg = dot * qk_scale;
    if (lg > st.m) {                          // new running max of this key group
        const float corr = exp2f(st.m - lg);
        st.l *= corr;
        st.pz *= corr;
#pragma unroll
        for (int k = 0; k < 8; ++k) st.o[k] = __fmul2_rn(st.o[k], bcast(corr));
        st.m = lg;
    }
    const float p = exp2f(lg - st.m);
    st.l += p;
    const uint8_t *rv = r + (D * (2 << CLS)) / 8;
    if (CLS == 3) {
        acc_native(st.o, p * kONativeScale, reinterpret_cast<const uint4 *>(rv)[2 * gl],
                   reinterpret_cast<const uint4 *>(rv)[2 * gl + 1]);
    } else {
        st.pz = fmaf(p, sd.w, st.pz);
        const float wv = p * sd.z * kWScale;
        if (CLS == 0) acc_codes2(st.o, wv, reinterpret_cast<const uint32_t *>(rv)[gl]);
        else if (CLS == 1) acc_codes4(st.o, wv, reinterpret_cast<const uint2 *>(rv)[gl]);
        else acc_codes8(st.o, wv, reinterpret_cast<const uint4 *>(rv)[gl]);
    }
}

// This warp's chunks ch, ch + kConsumerWarps, ... below `end`, all of width class CLS.
template <int D, int CLS>
__device__ __forceinline__ int run_class(KeyState &st, const QRegs &qr, float qsum, float qk_scale,
                                         const Stage<D> &sg, int ch, int end, int g, int gl)
{
    constexpr int KEYS_PER_STEP = 32 / (D / 16);
    for (; ch < end; ch += kConsumerWarps)
        process_key<D, CLS>(st, qr, qsum, qk_scale, sg, sg.perm[KEYS_PER_STEP * ch + g], gl);
    return ch;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 3)
decode_splitk_kernel(CacheView c, const __half *__restrict__ q, DecodeWork wk)
{
    constexpr int GROUP = D / 16;                 // lanes per key (16 channels per lane)
    constexpr int KEYS_PER_STEP = 32 / GROUP;     // keys per chunk step of a warp

    extern __shared__ __align__(128) uint8_t smem_raw[];
    DecodeSmem<D> &sm = *reinterpret_cast<DecodeSmem<D> *>(smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    pdl_wait();
    pdl_trigger();
    const int n_items = *wk.count;

    if (tid == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&sm.full[i], 1);
            mbar_init(&sm.empty[i], kConsumerWarps);
        }
        for (int i = 0; i < kMetaSlots; ++i) mbar_init(&sm.mfull[i], 1);
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == kConsumerWarps) {
        // ------------------------------ producer ---------------------------------
        // A filler cursor runs up to kMetaSlots windows ahead and bulk-copies each window of
        // 128 record offsets into a shared ring; the record cursor reads a window from shared
        // memory, cuts it into stages of at most kStageRecBytes, sorts each stage's keys by
        // width and issues the stage's copies.
        constexpr int KPL = kWin / 32;                // window keys per lane: lane + 32 r
        int f_it = blockIdx.x;
        if (f_it >= n_items) return;
        DecodeItem f_d = wk.items[f_it];
        int f_j = f_d.j0;
        bool f_valid = true;
        int filled = 0, consumed = 0, stage = 0;
        uint32_t phase = 0;
        const uint32_t lt = (1u << lane) - 1u;
        while (true) {
            while (f_valid && filled < consumed + kMetaSlots) {
                const int slot = filled % kMetaSlots;
                MetaSlot &ms = sm.ms[slot];
                const int ja = f_j & ~3;
                const int jb = (min(f_j + kWin + 1, f_d.j1 + 1) + 3) & ~3;
                if (lane == 0) {
                    ms.it = f_it;
                    ms.j = f_j;
                    ms.j1 = f_d.j1;
                    ms.ja = ja;
                    ms.end_off = f_d.end_off;
                    ms.first = (f_j == f_d.j0);
                    ms.sbase = f_d.sbase;
                    ms.sh = f_d.sh;
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    mbar_arrive_expect_tx(&sm.mfull[slot], 4u * (uint32_t)(jb - ja));
                    bulk_g2s(ms.meta, c.meta + f_d.sbase + ja, 4u * (uint32_t)(jb - ja), &sm.mfull[slot]);
                }
                ++filled;
                f_j += kWin;
                if (f_j >= f_d.j1) {
                    f_it += gridDim.x;
                    if (f_it < n_items) {
                        f_d = wk.items[f_it];
                        f_j = f_d.j0;
                    } else {
                        f_valid = false;
                    }
                }
            }
            if (consumed == filled) break;
            const int slot = consumed % kMetaSlots;
            if (!mbar_wait(&sm.mfull[slot], (uint32_t)(consumed / kMetaSlots) & 1u, c.status)) return;
            const MetaSlot &ms = sm.ms[slot];
            const int j = ms.j, it = ms.it;
            const int nwin = min(kWin, ms.j1 - j);
            const bool lastwin = (j + nwin == ms.j1), first = ms.first != 0;
            const uint32_t *mw = ms.meta + (j - ms.ja);
            uint32_t m[KPL], nx[KPL];
#pragma unroll
            for (int r = 0; r < KPL; ++r) m[r] = (lane + 32 * r < nwin) ? mw[lane + 32 * r] : 0u;
            const uint32_t bnd = ((!lastwin || ms.end_off == kReadEndFromMeta) ? mw[nwin] : ms.end_off) & ~15u;
            const int64_t sbase = ms.sbase;
            const int sh = ms.sh;
            // nx[r]: offset right after key lane + 32 r (the next key's offset, or the bound)
#pragma unroll
            for (int r = 0; r < KPL; ++r) {
                const uint32_t dn = __shfl_down_sync(0xffffffffu, m[r], 1) & ~15u;
                const uint32_t wrap = (r + 1 < KPL) ? (__shfl_sync(0xffffffffu, m[(r + 1) % KPL], 0) & ~15u) : bnd;
                nx[r] = (lane == 31) ? wrap : dn;
                if (lane + 32 * r + 1 >= nwin) nx[r] = bnd;
            }
            ++consumed;

            for (int w0 = 0; w0 < nwin;) {
                // the stage: keys [w0, w1) of the window, at most kStageRecBytes of records
                const uint32_t mstart = __shfl_sync(0xffffffffu, (w0 / 32 == 0) ? m[0] : (w0 / 32 == 1) ? m[1 % KPL]
                                                                   : (w0 / 32 == 2) ? m[2 % KPL] : m[3 % KPL], w0 & 31);
                const uint32_t off0 = mstart & ~15u;
                int n = 0;
#pragma unroll
                for (int r = 0; r < KPL; ++r) {
                    const int k = lane + 32 * r;
                    n += __popc(__ballot_sync(0xffffffffu, k >= w0 && k < nwin && nx[r] - off0 <= kStageRecBytes));
                }
                if (n < 1) {          // only with corrupt offsets: flag it, keep making progress
                    if (lane == 0) set_status(c.status, KVQ_ERR_DEVICE_CHECK);
                    n = 1;
                }
                const int w1 = w0 + n;
                const int kl = w1 - 1;
                const uint32_t nxl = __shfl_sync(0xffffffffu, (kl / 32 == 0) ? nx[0] : (kl / 32 == 1) ? nx[1 % KPL]
                                                             : (kl / 32 == 2) ? nx[2 % KPL] : nx[3 % KPL], kl & 31);
                const bool last = lastwin && w1 == nwin;
                const bool new_item = first && w0 == 0;
                uint32_t rec_bytes = nxl - off0;
                if (nxl < off0 || rec_bytes > kStageRecBytes) {   // corrupt offsets
                    if (lane == 0) set_status(c.status, KVQ_ERR_DEVICE_CHECK);
                    rec_bytes = 0;
                }
                // counting sort by width, each width's run padded to whole chunks of KEYS_PER_STEP
                constexpr int PADL = KEYS_PER_STEP - 1;       // pad entries per width, at most
                int cl_of[KPL], pos_of[KPL];
#pragma unroll
                for (int r = 0; r < KPL; ++r) {
                    const int k = lane + 32 * r;
                    cl_of[r] = (k >= w0 && k < w1) ? (int)(m[r] & 3u) : 4;
                    pos_of[r] = 0;
                }
                int pstart = 0, pad_pos = -1, cls_chunk[4];
#pragma unroll
                for (int cl = 0; cl < 4; ++cl) {
                    cls_chunk[cl] = pstart / KEYS_PER_STEP;
                    int before = 0;
#pragma unroll
                    for (int r = 0; r < KPL; ++r) {
                        const uint32_t b = __ballot_sync(0xffffffffu, cl_of[r] == cl);
                        if (cl_of[r] == cl) pos_of[r] = pstart + before + __popc(b & lt);
                        before += __popc(b);
                    }
                    const int padded = (before + PADL) / KEYS_PER_STEP * KEYS_PER_STEP;
                    if (lane / PADL == cl && before + lane % PADL < padded)     // PADL lanes per width
                        pad_pos = pstart + before + lane % PADL;
                    pstart += padded;
                }

                if (!mbar_wait(&sm.empty[stage], phase ^ 1u, c.status)) return;
                Stage<D> &sg = sm.st[stage];
#pragma unroll
                for (int r = 0; r < KPL; ++r) {
                    if (cl_of[r] < 4) {
                        // offset inside the stage; the clamp only bites on corrupt offsets and
                        // keeps every shared-memory read of the consumers inside the stage
                        const uint32_t ro = min((m[r] & ~15u) - off0,
                                                kStageRecBytes - (uint32_t)(D * (2 << cl_of[r])) / 4u);
                        sg.perm[pos_of[r]] = kValid | ((uint32_t)(lane + 32 * r - w0) << 16) | ro;
                    }
                }
                if (pad_pos >= 0) sg.perm[pad_pos] = 0u;
                if (lane == 0) {
                    sg.info[0] = it;
                    sg.info[1] = n;
                    sg.info[2] = (new_item ? kNewItem : 0) | (last ? kLastSub : 0);
                    sg.info[3] = pstart / KEYS_PER_STEP;
#pragma unroll
                    for (int cl = 0; cl < 4; ++cl) sg.cls_chunk[cl] = cls_chunk[cl];
                    sg.cls_chunk[4] = pstart / KEYS_PER_STEP;
                }
                __syncwarp();
                if (lane == 0) {
                    const uint32_t q_bytes = new_item ? 2u * D : 0u;
                    mbar_arrive_expect_tx(&sm.full[stage], 16u * n + rec_bytes + q_bytes);
                    bulk_g2s(sg.side, c.side + sbase + j + w0, 16u * n, &sm.full[stage]);
                    if (rec_bytes)
                        bulk_g2s(sg.rec, c.rec + sbase * (int64_t)(4 * D) + off0, rec_bytes, &sm.full[stage]);
                    if (q_bytes) bulk_g2s(sg.q, q + (int64_t)sh * D, q_bytes, &sm.full[stage]);
                }
                if (++stage == kStages) {
                    stage = 0;
                    phase ^= 1u;
                }
                w0 = w1;
            }
        }
        return;
    }

    // -------------------------------- consumers -------------------------------------
    const int g = lane / GROUP;          // key slot within a chunk step
    const int gl = lane % GROUP;         // channel block: channels [16 gl, 16 gl + 16)
    const float qk_scale = kLog2e * rsqrtf((float)D);   // logits in log2 units
    int stage = 0, rot = 0;
    uint32_t phase = 0;
    QRegs qr;
    float qsum = 0.f;
    for (int it = blockIdx.x; it < n_items; it += gridDim.x) {
        KeyState ks;
        ks.m = -INFINITY;
        ks.l = 0.f;
        ks.pz = 0.f;
#pragma unroll
        for (int k = 0; k < 8; ++k) ks.o[k] = make_float2(0.f, 0.f);
        bool last = false;
        while (!last) {
            if (!mbar_wait(&sm.full[stage], phase, c.status)) return;
            Stage<D> &sg = sm.st[stage];
            const int flags = sg.info[2];
            last = (flags & kLastSub) != 0;
            if (flags & kNewItem) {
                // query: this lane's 16 channels, scaled per width; sum(q) over all D
                const uint4 a = reinterpret_cast<const uint4 *>(sg.q + 16 * gl)[0];
                const uint4 bq = reinterpret_cast<const uint4 *>(sg.q + 16 * gl)[1];
                const uint32_t hw[8] = {a.x, a.y, a.z, a.w, bq.x, bq.y, bq.z, bq.w};
                qsum = 0.f;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&hw[e]));
                    const float fv[2] = {f.x, f.y};
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const int k = 2 * e + u;        // channel 16 gl + k -> pair k % 8, half k / 8
                        qsum += fv[u];
                        const float v8 = fv[u] * kQScale;
                        const float v4 = v8 * __uint_as_float((127u - 4u * (k % 4)) << 23);
                        const float v2 = v8 * __uint_as_float((127u - 2u * (k % 8)) << 23);
                        if (k < 8) {
                            qr.q8[k].x = v8;
                            qr.q4[k].x = v4;
                            qr.q2[k].x = v2;
                        } else {
                            qr.q8[k - 8].y = v8;
                            qr.q4[k - 8].y = v4;
                            qr.q2[k - 8].y = v2;
                        }
                    }
                }
#pragma unroll
                for (int d = 1; d < GROUP; d <<= 1) qsum += __shfl_xor_sync(0xffffffffu, qsum, d);
            }
            // class-pure chunks, dealt to the warps round-robin (rotated every stage); the
            // chunks are sorted by width, so the warp walks one run per width class
            int ch = (warp + kConsumerWarps - rot) % kConsumerWarps;
            ch = run_class<D, 0>(ks, qr, qsum, qk_scale, sg, ch, sg.cls_chunk[1], g, gl);
            ch = run_class<D, 1>(ks, qr, qsum, qk_scale, sg, ch, sg.cls_chunk[2], g, gl);
            ch = run_class<D, 2>(ks, qr, qsum, qk_scale, sg, ch, sg.cls_chunk[3], g, gl);
            run_class<D, 3>(ks, qr, qsum, qk_scale, sg, ch, sg.cls_chunk[4], g, gl);
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.empty[stage]);
            rot = (rot + 1) % kConsumerWarps;
            if (++stage == kStages) {
                stage = 0;
                phase ^= 1u;
            }
        }

        // merge the key groups of the warp, then the warps, into the item's partial
#pragma unroll
        for (int mask = GROUP; mask < 32; mask <<= 1) merge_state(ks.m, ks.l, ks.pz, ks.o, mask);
        if (g == 0) {
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                sm.red_o[warp][16 * gl + k] = ks.o[k].x;
                sm.red_o[warp][16 * gl + 8 + k] = ks.o[k].y;
            }
            if (gl == 0) {
                sm.red_m[warp] = ks.m;
                sm.red_l[warp] = ks.l;
                sm.red_pz[warp] = ks.pz;
            }
        }
        named_bar_sync(1, 32 * kConsumerWarps);
        if (warp == 0) {
            float M = -INFINITY;
#pragma unroll
            for (int wv = 0; wv < kConsumerWarps; ++wv) M = fmaxf(M, sm.red_m[wv]);
            float f[kConsumerWarps];
            float L = 0.f, PZ = 0.f;
#pragma unroll
            for (int wv = 0; wv < kConsumerWarps; ++wv) {
                f[wv] = (sm.red_m[wv] == -INFINITY) ? 0.f : exp2f(sm.red_m[wv] - M);
                L = fmaf(sm.red_l[wv], f[wv], L);
                PZ = fmaf(sm.red_pz[wv], f[wv], PZ);
            }
            float *part = wk.partials + (int64_t)it * (D + 4);
            for (int chn = lane; chn < D; chn += 32) {
                float acc = 0.f;
#pragma unroll
                for (int wv = 0; wv < kConsumerWarps; ++wv) acc = fmaf(sm.red_o[wv][chn], f[wv], acc);
                part[4 + chn] = fmaf(acc, kOUnscale, PZ);
            }
            if (lane == 0) {
                part[0] = M;
                part[1] = L;
            }
        }
        named_bar_sync(1, 32 * kConsumerWarps);   // red_* are reused by the next item
    }
}

// One CTA of D threads per (sequence, head): thread = channel.
template <int D>
__global__ void __launch_bounds__(D)
decode_combine_kernel(CacheView c, DecodeWork wk, float *__restrict__ out)
{
    __shared__ float red[D / 32];
    pdl_wait();
    pdl_trigger();
    const int sh = blockIdx.x, ch = threadIdx.x, lane = ch & 31, wid = ch >> 5;
    const int first = wk.head_first[sh], cnt = wk.head_cnt[sh];
    const float *P = wk.partials + (int64_t)first * (D + 4);
    float res = 0.f;
    if (cnt > 0) {
        float M = -INFINITY;
        for (int i = ch; i < cnt; i += D) M = fmaxf(M, P[(int64_t)i * (D + 4)]);
#pragma unroll
        for (int d = 16; d >= 1; d >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, d));
        if (lane == 0) red[wid] = M;
        __syncthreads();
        M = red[0];
#pragma unroll
        for (int w = 1; w < D / 32; ++w) M = fmaxf(M, red[w]);
        float L = 0.f, acc = 0.f;
        int i = 0;
        for (; i + 4 <= cnt; i += 4) {
            float mm[4], ll[4], oo[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float *p = P + (int64_t)(i + u) * (D + 4);
                mm[u] = p[0];
                ll[u] = p[1];
                oo[u] = p[4 + ch];
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float f = exp2f(mm[u] - M);
                L = fmaf(ll[u], f, L);
                acc = fmaf(oo[u], f, acc);
            }
        }
        for (; i < cnt; ++i) {
            const float *p = P + (int64_t)i * (D + 4);
            const float f = exp2f(p[0] - M);
            L = fmaf(p[1], f, L);
            acc = fmaf(p[4 + ch], f, acc);
        }
        res = acc / L;
    }
    out[(int64_t)sh * D + ch] = res;
}

template <int D>
cudaError_t launch_decode_t(const kvq_cache *cache, const __half *q, const uint8_t *modes, int w,
                            float *out, cudaStream_t st)
{
    const CacheView &c = cache->view;
    cudaError_t le = launch_pdl(decode_sched_kernel, dim3(1), dim3(1024), 0, st, c, modes, w, cache->work);
    if (le != cudaSuccess) return le;
    const size_t smem = sizeof(DecodeSmem<D>);
    static bool attr_done = false;
    if (!attr_done) {
        cudaError_t e = cudaFuncSetAttribute(decode_splitk_kernel<D>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        attr_done = true;
    }
    const int grid = (int)std::min<int64_t>(cache->work.max_items, 3 * (int64_t)num_sms());
    profile_before(st);
    le = launch_pdl(decode_splitk_kernel<D>, dim3(grid), dim3(kThreads), smem, st, c, q, cache->work);
    if (le != cudaSuccess) return le;
    profile_after(st);
    le = launch_pdl(decode_combine_kernel<D>, dim3(c.B * c.H * c.G), dim3(D), 0, st, c, cache->work, out);
    if (le != cudaSuccess) return le;
    return cudaGetLastError();
}

} // namespace

cudaError_t launch_decode(const kvq_cache *cache, const __half *q, const uint8_t *modes, int w,
                          float *out, cudaStream_t st)
{
    if (cache->D == 128) return launch_decode_t<128>(cache, q, modes, w, out, st);
    return launch_decode_t<64>(cache, q, modes, w, out, st);
}

} // namespace kvq

// ---- allocation-free decode -------------------------------------------------------------
// routed_attn_decode_noalloc runs the same three kernels as routed_attn_decode, but its
// per-call scratch (the scheduler's work list and the split-K partials) lives in the
// file-scope array below instead of the cache's workspace, and the call allocates
// nothing. Host code must never hand `g_decode_scratch` itself to a kernel: on the host
// that name is only a stand-in. The device address is looked up once per device, with that
// device current, by cudaGetSymbolAddress.
namespace {
constexpr size_t kStaticScratchBytes = size_t(16) << 20;   // 16 MiB on every device
}
static __device__ __align__(256) unsigned char g_decode_scratch[kStaticScratchBytes];

namespace kvq {
namespace {

std::mutex g_scratch_mu;
void *g_scratch_addr[256] = {};   // device address of g_decode_scratch, per device ordinal

cudaError_t static_scratch(int dev, unsigned char **out)
{
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (dev < 0 || dev >= 256) return cudaErrorInvalidDevice;
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_addr[dev] = p;
    }
    *out = static_cast<unsigned char *>(g_scratch_addr[dev]);
    return cudaSuccess;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

template <int D>
cudaError_t launch_decode_static(const kvq_cache *cache, const DecodeWork &wk, const __half *q,
                                 const uint8_t *modes, int w, float *out, cudaStream_t st)
{
    const CacheView &c = cache->view;
    cudaError_t e = launch_pdl(decode_sched_kernel, dim3(1), dim3(1024), 0, st, c, modes, w, wk);
    if (e != cudaSuccess) return e;
    const size_t smem = sizeof(DecodeSmem<D>);
    e = cudaFuncSetAttribute(decode_splitk_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int grid = (int)std::min<int64_t>(wk.max_items, 3 * (int64_t)num_sms());
    e = launch_pdl(decode_splitk_kernel<D>, dim3(grid), dim3(kThreads), smem, st, c, q, wk);
    if (e != cudaSuccess) return e;
    e = launch_pdl(decode_combine_kernel<D>, dim3(c.B * c.H * c.G), dim3(D), 0, st, c, wk, out);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

} // namespace
} // namespace kvq

extern "C" int routed_attn_decode_noalloc(const void *q, const kvq_cache *cache, const uint8_t *modes,
                                          int w, float *out, kvq_stream_t stream)
{
    using namespace kvq;
    if (!cache || cache->B <= 0 || cache->H <= 0)
        return report_error(KVQ_ERR_ARG, "routed_attn_decode_noalloc: bad cache");
    if (w < 0) return report_error(KVQ_ERR_ARG, "routed_attn_decode_noalloc: w < 0");
    if (!q || !modes || !out) return report_error(KVQ_ERR_ARG, "routed_attn_decode_noalloc: q, modes or out is NULL");
    if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(out)) & 15u)
        return report_error(KVQ_ERR_ARG, "routed_attn_decode_noalloc: q and out must be 16-byte aligned");
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return report_error(KVQ_ERR_CUDA, "routed_attn_decode_noalloc: cudaGetDevice failed");
    if (dev != cache->device)
        return report_error(KVQ_ERR_ARG, "routed_attn_decode_noalloc: the cache's device is not the current device");

    // scratch layout: count | head_first | head_cnt | items | partials, each 256-byte aligned,
    // sized for the cache's worst case (every head full at capacity)
    const int BH = cache->B * cache->H * cache->view.G;     // query heads
    const int64_t items = cache->work.max_items;
    const size_t o_first = 256;
    const size_t o_cnt = o_first + align256(sizeof(int32_t) * (size_t)BH);
    const size_t o_items = o_cnt + align256(sizeof(int32_t) * (size_t)BH);
    const size_t o_part = o_items + align256(sizeof(DecodeItem) * (size_t)items);
    const size_t need = o_part + sizeof(float) * (size_t)items * (cache->D + 4);
    if (need > kStaticScratchBytes) {
        char msg[256];
        snprintf(msg, sizeof(msg),
                 "routed_attn_decode_noalloc: this cache needs %zu bytes of scratch, more than the %zu "
                 "bytes of static scratch; use routed_attn_decode",
                 need, kStaticScratchBytes);
        return report_error(KVQ_ERR_ARG, msg);
    }
    unsigned char *base = nullptr;
    e = static_scratch(dev, &base);
    if (e != cudaSuccess) return report_error(KVQ_ERR_CUDA, "routed_attn_decode_noalloc: cudaGetSymbolAddress failed");
    DecodeWork wk;
    wk.count = reinterpret_cast<int32_t *>(base);
    wk.head_first = reinterpret_cast<int32_t *>(base + o_first);
    wk.head_cnt = reinterpret_cast<int32_t *>(base + o_cnt);
    wk.items = reinterpret_cast<DecodeItem *>(base + o_items);
    wk.partials = reinterpret_cast<float *>(base + o_part);
    wk.max_items = items;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    e = (cache->D == 128) ? launch_decode_static<128>(cache, wk, static_cast<const __half *>(q), modes, w, out, st)
                          : launch_decode_static<64>(cache, wk, static_cast<const __half *>(q), modes, w, out, st);
    if (e != cudaSuccess) return report_error(KVQ_ERR_CUDA, "routed_attn_decode_noalloc: kernel launch failed");
    return report_error(KVQ_OK, "");
}
