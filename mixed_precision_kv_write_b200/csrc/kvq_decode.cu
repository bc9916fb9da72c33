// Routed decode attention (TriRoute paper review page, section 3, Eq. 2) over the
// mixed-precision cache of Eq. 4: one query per (sequence, head) at t = len - 1.
//
// Three launches:
//   decode_sched_kernel   mode-aware scheduler: skip heads and empty sequences get no
//                         work, local heads are clamped to keys [max(0, t - w), t], full
//                         heads read [0, t]; each range is cut into items of up to 512
//                         keys, listed on the device (no host round trip).
//   decode_splitk_kernel  persistent CTAs: one producer warp streams each item's
//                         contiguous record bytes, side entries and offsets into shared
//                         memory with 1-D bulk copies (64-key stages, mbarrier pipeline);
//                         eight consumer warps dequantize in registers and run an online
//                         softmax; each item leaves a partial (m, l, o[D]).
//   decode_combine_kernel log-sum-exp merge of an item list per (sequence, head).
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
#include "kvq_internal.cuh"

namespace kvq {
namespace {

constexpr int kConsumerWarps = 8;
constexpr int kThreads = 32 * (kConsumerWarps + 1);
constexpr int kStages = 4;
constexpr int kSub = kDecodeSubKeys;              // 64 keys per stage


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
    uint32_t meta[kSub + 4];
    float4 side[kSub];
    alignas(16) uint8_t rec[kSub * 4 * D];
};

template <int D>
struct DecodeSmem {
    Stage<D> st[kStages];
    float logit[kStages][kSub];
    uint8_t perm[kConsumerWarps][kSub];
    float red[kConsumerWarps][D];
    uint64_t full[kStages];
    uint64_t empty[kStages];
};

__device__ __forceinline__ float fld(uint32_t bits) { return __uint_as_float(bits); }

__global__ void decode_sched_kernel(CacheView c, const uint8_t *__restrict__ modes, int w,
                                    DecodeWork wk)
{
    __shared__ int warp_tot[32];
    __shared__ int carry_sh;
    const int BH = c.B * c.H;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    if (tid == 0) carry_sh = 0;
    __syncthreads();
    for (int base = 0; base < BH; base += blockDim.x) {
        const int i = base + tid;
        int cnt = 0, lo = 0, hi = 0;
        if (i < BH) {
            const int m = modes[i];
            const int L = c.len[i];
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
            for (int k = 0; k < cnt; ++k)
                wk.items[first + k] = make_int4(i, lo + k * kDecodeItemKeys,
                                                min(hi, lo + (k + 1) * kDecodeItemKeys), 0);
        }
        __syncthreads();
        if (tid == 0) carry_sh = carry + warp_tot[(blockDim.x >> 5) - 1];
        __syncthreads();
    }
    if (tid == 0) *wk.count = carry_sh;
}

// ---- per-width dot products and accumulations for one lane's 16 channels ----------
struct QRegs {
    float q2[16], q4[16], q8[16];   // q * 2^(60 - pos_b)
};

__device__ __forceinline__ float dot_codes2(const QRegs &q, uint32_t x)
{
    const uint32_t y = x >> 16;
    float a0 = 0.f, a1 = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        a0 = fmaf(q.q2[k], fld(x & (3u << (2 * k))), a0);
        a1 = fmaf(q.q2[k + 8], fld(y & (3u << (2 * k))), a1);
    }
    return a0 + a1;
}

__device__ __forceinline__ float dot_codes4(const QRegs &q, uint2 x)
{
    float a0 = 0.f, a1 = 0.f;
    const uint32_t w[2] = {x.x, x.y};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const uint32_t lo = w[h], hi = w[h] >> 16;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            a0 = fmaf(q.q4[8 * h + k], fld(lo & (15u << (4 * k))), a0);
            a1 = fmaf(q.q4[8 * h + 4 + k], fld(hi & (15u << (4 * k))), a1);
        }
    }
    return a0 + a1;
}

__device__ __forceinline__ float dot_codes8(const QRegs &q, uint4 x)
{
    float a0 = 0.f, a1 = 0.f;
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int h = 0; h < 4; ++h) {
        a0 = fmaf(q.q8[4 * h + 0], fld(__byte_perm(w[h], 0u, 0x4440)), a0);
        a1 = fmaf(q.q8[4 * h + 1], fld(__byte_perm(w[h], 0u, 0x4441)), a1);
        a0 = fmaf(q.q8[4 * h + 2], fld(__byte_perm(w[h], 0u, 0x4442)), a0);
        a1 = fmaf(q.q8[4 * h + 3], fld(__byte_perm(w[h], 0u, 0x4443)), a1);
    }
    return a0 + a1;
}

__device__ __forceinline__ float dot_native(const QRegs &q, uint4 x0, uint4 x1)
{
    const uint32_t w[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
    float a0 = 0.f, a1 = 0.f;
#pragma unroll
    for (int h = 0; h < 8; ++h) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&w[h]));
        a0 = fmaf(q.q8[2 * h], f.x, a0);
        a1 = fmaf(q.q8[2 * h + 1], f.y, a1);
    }
    return a0 + a1;
}

__device__ __forceinline__ void acc_codes2(float (&o)[16], float wv, uint32_t x)
{
    const uint32_t y = x >> 16;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const float wk = wv * __uint_as_float((127u - 2u * k) << 23);   // wv * 2^-2k
        o[k] = fmaf(wk, fld(x & (3u << (2 * k))), o[k]);
        o[k + 8] = fmaf(wk, fld(y & (3u << (2 * k))), o[k + 8]);
    }
}

__device__ __forceinline__ void acc_codes4(float (&o)[16], float wv, uint2 x)
{
    const uint32_t w[2] = {x.x, x.y};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const float wk = wv * __uint_as_float((127u - 4u * k) << 23);   // wv * 2^-4k
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            o[8 * h + k] = fmaf(wk, fld(w[h] & (15u << (4 * k))), o[8 * h + k]);
            o[8 * h + 4 + k] = fmaf(wk, fld((w[h] >> 16) & (15u << (4 * k))), o[8 * h + 4 + k]);
        }
    }
}

__device__ __forceinline__ void acc_codes8(float (&o)[16], float wv, uint4 x)
{
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int h = 0; h < 4; ++h) {
#pragma unroll
        for (int e = 0; e < 4; ++e)
            o[4 * h + e] = fmaf(wv, fld(__byte_perm(w[h], 0u, 0x4440 + e)), o[4 * h + e]);
    }
}

__device__ __forceinline__ void acc_native(float (&o)[16], float wv, uint4 x0, uint4 x1)
{
    const uint32_t w[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
#pragma unroll
    for (int h = 0; h < 8; ++h) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&w[h]));
        o[2 * h] = fmaf(wv, f.x, o[2 * h]);
        o[2 * h + 1] = fmaf(wv, f.y, o[2 * h + 1]);
    }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
decode_splitk_kernel(CacheView c, const __half *__restrict__ q, int w, DecodeWork wk)
{
    constexpr int GROUP = D / 16;                 // lanes per key (16 channels per lane)
    constexpr int KEYS_PER_STEP = 32 / GROUP;     // keys a warp handles at once
    constexpr int KEYS_PER_WARP = kSub / kConsumerWarps;
    constexpr int STEPS = KEYS_PER_WARP / KEYS_PER_STEP;
    static_assert(STEPS * KEYS_PER_STEP == KEYS_PER_WARP, "sub-chunk split");

    extern __shared__ __align__(128) uint8_t smem_raw[];
    DecodeSmem<D> &sm = *reinterpret_cast<DecodeSmem<D> *>(smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int n_items = *wk.count;

    if (tid == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&sm.full[i], 1);
            mbar_init(&sm.empty[i], kConsumerWarps);
        }
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == kConsumerWarps) {
        // ------------------------------ producer ---------------------------------
        if (lane != 0) return;
        int stage = 0;
        uint32_t phase = 0;
        for (int it = blockIdx.x; it < n_items; it += gridDim.x) {
            const int4 item = wk.items[it];
            const int sh = item.x, s = sh / c.H, h = sh % c.H;
            const int L = c.len[sh];
            const int64_t sbase = slot_of(c, s, h, 0);
            const uint8_t *stream = stream_of(c, s, h);
            for (int j = item.y; j < item.z; j += kSub) {
                const int je = min(j + kSub, item.z);
                if (!mbar_wait(&sm.empty[stage], phase ^ 1u, c.status)) return;
                const uint32_t off0 = c.meta[sbase + j] & ~15u;
                const uint32_t off1 = (je < L) ? (c.meta[sbase + je] & ~15u) : c.end[sh];
                const int ja = j & ~3, jb = (je + 3) & ~3;
                const uint32_t meta_bytes = 4u * (uint32_t)(jb - ja);
                const uint32_t side_bytes = 16u * (uint32_t)(je - j);
                uint32_t rec_bytes = off1 - off0;
                if (off1 < off0 || rec_bytes > (uint32_t)(kSub * 4 * D)) {   // corrupt offsets
                    set_status(c.status, KVQ_ERR_DEVICE_CHECK);
                    rec_bytes = 0;
                }
                Stage<D> &sg = sm.st[stage];
                mbar_arrive_expect_tx(&sm.full[stage], meta_bytes + side_bytes + rec_bytes);
                bulk_g2s(sg.meta, c.meta + sbase + ja, meta_bytes, &sm.full[stage]);
                bulk_g2s(sg.side, c.side + sbase + j, side_bytes, &sm.full[stage]);
                if (rec_bytes) bulk_g2s(sg.rec, stream + off0, rec_bytes, &sm.full[stage]);
                if (++stage == kStages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        return;
    }

    // -------------------------------- consumers -------------------------------------
    const int g = lane / GROUP;          // key slot within a step
    const int gl = lane % GROUP;         // channel block: channels [16 gl, 16 gl + 16)
    const float qk_scale = kLog2e * rsqrtf((float)D);   // logits in log2 units
    int stage = 0;
    uint32_t phase = 0;
    for (int it = blockIdx.x; it < n_items; it += gridDim.x) {
        const int4 item = wk.items[it];
        const int sh = item.x;

        // query: this lane's 16 channels, scaled per width; sum(q) over all D
        QRegs qr;
        float qsum = 0.f;
        {
            const uint4 *qp = reinterpret_cast<const uint4 *>(q + (int64_t)sh * D + 16 * gl);
            const uint4 a = qp[0], bq = qp[1];
            const uint32_t hw[8] = {a.x, a.y, a.z, a.w, bq.x, bq.y, bq.z, bq.w};
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&hw[e]));
                const float fv[2] = {f.x, f.y};
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int k = 2 * e + u;
                    qsum += fv[u];
                    qr.q8[k] = fv[u] * kQScale;
                    qr.q4[k] = qr.q8[k] * __uint_as_float((127u - 4u * (k % 4)) << 23);
                    qr.q2[k] = qr.q8[k] * __uint_as_float((127u - 2u * (k % 8)) << 23);
                }
            }
#pragma unroll
            for (int d = 1; d < GROUP; d <<= 1) qsum += __shfl_xor_sync(0xffffffffu, qsum, d);
        }

        float m_run = -INFINITY, l_run = 0.f, pz_run = 0.f;
        float o[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) o[k] = 0.f;

        for (int j = item.y; j < item.z; j += kSub) {
            const int n = min(kSub, item.z - j);
            if (!mbar_wait(&sm.full[stage], phase, c.status)) return;
            Stage<D> &sg = sm.st[stage];
            const int mo = j & 3;                      // meta copy starts at j & ~3
            const uint32_t off0 = sg.meta[mo] & ~15u;

            // order the stage's keys by width (warp-redundant counting sort via ballots)
            {
                const int k0 = lane, k1 = lane + 32;
                const int c0 = (k0 < n) ? (int)(sg.meta[mo + k0] & 3u) : 4;
                const int c1 = (k1 < n) ? (int)(sg.meta[mo + k1] & 3u) : 4;
                const uint32_t lt = (1u << lane) - 1u;
                int base = 0, p0 = 0, p1 = 0;
#pragma unroll
                for (int cl = 0; cl < 4; ++cl) {
                    const uint32_t b0 = __ballot_sync(0xffffffffu, c0 == cl);
                    const uint32_t b1 = __ballot_sync(0xffffffffu, c1 == cl);
                    if (c0 == cl) p0 = base + __popc(b0 & lt);
                    if (c1 == cl) p1 = base + __popc(b0) + __popc(b1 & lt);
                    base += __popc(b0) + __popc(b1);
                }
                if (k0 < n) sm.perm[warp][p0] = (uint8_t)k0;
                if (k1 < n) sm.perm[warp][p1] = (uint8_t)k1;
                __syncwarp();
            }

            // K pass: logits of this warp's keys
#pragma unroll
            for (int stp = 0; stp < STEPS; ++stp) {
                const int pos = warp * KEYS_PER_WARP + stp * KEYS_PER_STEP + g;
                float part = 0.f;
                int key = -1;
                int cls = 0;
                if (pos < n) {
                    key = sm.perm[warp][pos];
                    const uint32_t mt = sg.meta[mo + key];
                    cls = mt & 3u;
                    const uint8_t *r = sg.rec + ((mt & ~15u) - off0);
                    if (cls == 0) part = dot_codes2(qr, reinterpret_cast<const uint32_t *>(r)[gl]);
                    else if (cls == 1) part = dot_codes4(qr, reinterpret_cast<const uint2 *>(r)[gl]);
                    else if (cls == 2) part = dot_codes8(qr, reinterpret_cast<const uint4 *>(r)[gl]);
                    else part = dot_native(qr, reinterpret_cast<const uint4 *>(r)[2 * gl],
                                           reinterpret_cast<const uint4 *>(r)[2 * gl + 1]);
                }
#pragma unroll
                for (int d = 1; d < GROUP; d <<= 1) part += __shfl_xor_sync(0xffffffffu, part, d);
                if (key >= 0 && gl == 0) {
                    const float4 sd = sg.side[key];
                    float dot;
                    if (cls == 3) dot = part * kDotNativeUnscale;
                    else dot = fmaf(sd.x, part * kDotCodeUnscale, sd.y * qsum);
                    sm.logit[stage][key] = dot * qk_scale;
                }
            }
            named_bar_sync(1, 32 * kConsumerWarps);

            // softmax over the stage (every warp redundantly, so no second barrier)
            const float l0 = (lane < n) ? sm.logit[stage][lane] : -INFINITY;
            const float l1 = (lane + 32 < n) ? sm.logit[stage][lane + 32] : -INFINITY;
            float cmax = fmaxf(l0, l1);
#pragma unroll
            for (int d = 16; d >= 1; d >>= 1) cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, d));
            const float m_new = fmaxf(m_run, cmax);
            const float corr = exp2f(m_run - m_new);
            const float p0 = (lane < n) ? exp2f(l0 - m_new) : 0.f;
            const float p1 = (lane + 32 < n) ? exp2f(l1 - m_new) : 0.f;
            float psum = p0 + p1;
            float pz = 0.f;
            if (lane < n && (sg.meta[mo + lane] & 3u) != 3u) pz = p0 * sg.side[lane].w;
            if (lane + 32 < n && (sg.meta[mo + lane + 32] & 3u) != 3u) pz = fmaf(p1, sg.side[lane + 32].w, pz);
#pragma unroll
            for (int d = 16; d >= 1; d >>= 1) {
                psum += __shfl_xor_sync(0xffffffffu, psum, d);
                pz += __shfl_xor_sync(0xffffffffu, pz, d);
            }
            l_run = fmaf(l_run, corr, psum);
            pz_run = fmaf(pz_run, corr, pz);
            m_run = m_new;
#pragma unroll
            for (int k = 0; k < 16; ++k) o[k] *= corr;

            // V pass
#pragma unroll
            for (int stp = 0; stp < STEPS; ++stp) {
                const int pos = warp * KEYS_PER_WARP + stp * KEYS_PER_STEP + g;
                const int key = (pos < n) ? sm.perm[warp][pos] : 0;
                const float pa = __shfl_sync(0xffffffffu, p0, key & 31);
                const float pb = __shfl_sync(0xffffffffu, p1, key & 31);
                if (pos < n) {
                    const float p = (key < 32) ? pa : pb;
                    const uint32_t mt = sg.meta[mo + key];
                    const int cls = mt & 3u;
                    const uint8_t *r = sg.rec + ((mt & ~15u) - off0) + (D * (2 << cls)) / 8;
                    if (cls == 3) {
                        acc_native(o, p * kONativeScale, reinterpret_cast<const uint4 *>(r)[2 * gl],
                                   reinterpret_cast<const uint4 *>(r)[2 * gl + 1]);
                    } else {
                        const float wv = p * sg.side[key].z * kWScale;
                        if (cls == 0) acc_codes2(o, wv, reinterpret_cast<const uint32_t *>(r)[gl]);
                        else if (cls == 1) acc_codes4(o, wv, reinterpret_cast<const uint2 *>(r)[gl]);
                        else acc_codes8(o, wv, reinterpret_cast<const uint4 *>(r)[gl]);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.empty[stage]);
            if (++stage == kStages) {
                stage = 0;
                phase ^= 1u;
            }
        }

        // reduce o over the key slots of the warp, then over the consumer warps
#pragma unroll
        for (int k = 0; k < 16; ++k) {
#pragma unroll
            for (int d = GROUP; d < 32; d <<= 1) o[k] += __shfl_xor_sync(0xffffffffu, o[k], d);
        }
        if (g == 0) {
#pragma unroll
            for (int k = 0; k < 16; ++k) sm.red[warp][16 * gl + k] = o[k];
        }
        named_bar_sync(1, 32 * kConsumerWarps);
        float *part = wk.partials + (int64_t)it * (D + 4);
        for (int ch = tid; ch < D; ch += 32 * kConsumerWarps) {
            float acc = 0.f;
#pragma unroll
            for (int wv = 0; wv < kConsumerWarps; ++wv) acc += sm.red[wv][ch];
            part[4 + ch] = fmaf(acc, kOUnscale, pz_run);
        }
        if (tid == 0) {
            part[0] = m_run;
            part[1] = l_run;
        }
        named_bar_sync(1, 32 * kConsumerWarps);   // red[] is reused by the next item
    }
}

template <int D>
__global__ void decode_combine_kernel(CacheView c, DecodeWork wk, float *__restrict__ out)
{
    constexpr int PER_LANE = D / 32;
    const int lane = threadIdx.x & 31;
    const int sh = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (sh >= c.B * c.H) return;
    const int first = wk.head_first[sh], cnt = wk.head_cnt[sh];
    float acc[PER_LANE];
#pragma unroll
    for (int e = 0; e < PER_LANE; ++e) acc[e] = 0.f;
    if (cnt > 0) {
        float M = -INFINITY;
        for (int i = 0; i < cnt; ++i) M = fmaxf(M, wk.partials[(int64_t)(first + i) * (D + 4)]);
        float L = 0.f;
        for (int i = 0; i < cnt; ++i) {
            const float *p = wk.partials + (int64_t)(first + i) * (D + 4);
            const float f = exp2f(p[0] - M);
            L = fmaf(p[1], f, L);
#pragma unroll
            for (int e = 0; e < PER_LANE; ++e) acc[e] = fmaf(p[4 + lane + 32 * e], f, acc[e]);
        }
        const float inv = 1.0f / L;
#pragma unroll
        for (int e = 0; e < PER_LANE; ++e) acc[e] *= inv;
    }
    float *o = out + (int64_t)sh * D;
#pragma unroll
    for (int e = 0; e < PER_LANE; ++e) o[lane + 32 * e] = acc[e];
}

template <int D>
cudaError_t launch_decode_t(const kvq_cache *cache, const __half *q, const uint8_t *modes, int w,
                            float *out, cudaStream_t st)
{
    const CacheView &c = cache->view;
    decode_sched_kernel<<<1, 1024, 0, st>>>(c, modes, w, cache->work);
    const size_t smem = sizeof(DecodeSmem<D>);
    static bool attr_done = false;
    if (!attr_done) {
        cudaError_t e = cudaFuncSetAttribute(decode_splitk_kernel<D>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        attr_done = true;
    }
    const int grid = (int)std::min<int64_t>(cache->work.max_items, (int64_t)num_sms());
    profile_before(st);
    decode_splitk_kernel<D><<<grid, kThreads, smem, st>>>(c, q, w, cache->work);
    profile_after(st);
    const int BH = c.B * c.H;
    decode_combine_kernel<D><<<(BH * 32 + 255) / 256, 256, 0, st>>>(c, cache->work, out);
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
