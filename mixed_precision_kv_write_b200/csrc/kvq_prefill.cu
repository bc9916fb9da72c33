// Routed causal prefill attention (TriRoute paper review page, section 3, Eq. 2) over the
// mixed-precision cache of Eq. 4, CUDA-core version.
//
// One CTA per (sequence, head, tile of 32 consecutive queries). The CTA walks the union
// of its queries' key ranges in 32-key tiles; each tile is dequantized once into shared
// memory (fp32, deq = code * s + z, b = 16 -> the fp16 value) and shared by the CTA's
// queries. Each warp owns 8 queries with an online softmax; a query skips every key tile
// outside its own range [lo, t] (lo = max(0, t - w) for local, 0 for full), and skip
// queries do no work and write zeros.
#include "kvq_internal.cuh"

namespace kvq {
namespace {

constexpr int kQT = 32;   // queries per CTA
constexpr int kKT = 32;   // keys per tile
constexpr int kWarps = 4;
constexpr int kQPW = kQT / kWarps;

template <int D>
__global__ void __launch_bounds__(32 * kWarps)
prefill_simple_kernel(CacheView c, const __half *__restrict__ q, const uint8_t *__restrict__ modes,
                      int w, const int32_t *__restrict__ cu, float *__restrict__ out)
{
    constexpr int PL = D / 32;   // channels per lane
    extern __shared__ __align__(16) float psm[];
    float (*qf)[D] = reinterpret_cast<float (*)[D]>(psm);
    float (*kT)[kKT + 1] = reinterpret_cast<float (*)[kKT + 1]>(psm + kQT * D);
    float (*vs)[D] = reinterpret_cast<float (*)[D]>(psm + kQT * D + D * (kKT + 1));
    __shared__ int q_lo[kQT], q_t[kQT], q_mode[kQT];
    __shared__ int range_sh[2];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int H = c.H;
    const int h = blockIdx.y;
    int bx = blockIdx.x, s = -1;
    for (int ss = 0; ss < c.B; ++ss) {
        const int nt = (cu[ss + 1] - cu[ss] + kQT - 1) / kQT;
        if (bx < nt) {
            s = ss;
            break;
        }
        bx -= nt;
    }
    if (s < 0) return;
    const int n_s = cu[s + 1] - cu[s];
    const int L = c.len[s * H + h];
    const int pos0 = L - n_s;                 // position of this sequence's first query
    const int i0 = bx * kQT;
    if (pos0 < 0) {
        if (tid == 0) set_status(c.status, KVQ_ERR_DEVICE_CHECK);
        return;
    }

    if (tid == 0) {
        range_sh[0] = INT32_MAX;
        range_sh[1] = -1;
    }
    __syncthreads();
    if (tid < kQT) {
        const int i = i0 + tid;
        int m = KVQ_MODE_SKIP, t = -1, lo = 0;
        if (i < n_s) {
            m = modes[(int64_t)(cu[s] + i) * H + h];
            t = pos0 + i;
            if (m > KVQ_MODE_FULL) {
                set_status(c.status, KVQ_ERR_MODE);
                m = KVQ_MODE_SKIP;
            }
            lo = (m == KVQ_MODE_LOCAL) ? max(0, t - w) : 0;
            if (m != KVQ_MODE_SKIP) {
                atomicMin(&range_sh[0], lo);
                atomicMax(&range_sh[1], t);
            }
        }
        q_mode[tid] = m;
        q_t[tid] = t;
        q_lo[tid] = lo;
    }
    for (int idx = tid; idx < kQT * D; idx += blockDim.x) {
        const int r = idx / D, ch = idx % D;
        const int i = i0 + r;
        qf[r][ch] = (i < n_s) ? __half2float(q[((int64_t)(cu[s] + i) * H + h) * D + ch]) : 0.f;
    }
    __syncthreads();
    const int klo = range_sh[0], khi = range_sh[1];

    const float scale = kLog2e * rsqrtf((float)D);
    float m_run[kQPW], l_run[kQPW], o[kQPW][PL];
#pragma unroll
    for (int r = 0; r < kQPW; ++r) {
        m_run[r] = -INFINITY;
        l_run[r] = 0.f;
#pragma unroll
        for (int e = 0; e < PL; ++e) o[r][e] = 0.f;
    }
    const int64_t sbase = slot_of(c, s, h, 0);
    const uint8_t *stream = stream_of(c, s, h);

    for (int kt = (khi >= 0 ? (klo / kKT) * kKT : 0); kt <= khi; kt += kKT) {
        __syncthreads();
        // dequantize keys kt .. kt + 31 into kT (transposed) and vs
        for (int kk = warp; kk < kKT; kk += kWarps) {
            const int j = kt + kk;
            if (j <= khi) {
                const uint32_t mt = c.meta[sbase + j];
                const int b = 2 << (mt & 3u);
                const float4 sd = c.side[sbase + j];
                const uint8_t *r = stream + (mt & ~15u);
#pragma unroll
                for (int e = 0; e < PL; ++e) {
                    const int ch = lane + 32 * e;
                    float kv, vv;
                    if (b == 16) {
                        kv = __half2float(reinterpret_cast<const __half *>(r)[ch]);
                        vv = __half2float(reinterpret_cast<const __half *>(r + 2 * D)[ch]);
                    } else {
                        const int bit = b * ch;
                        const uint32_t mask = (1u << b) - 1u;
                        const uint32_t ck = (reinterpret_cast<const uint32_t *>(r)[bit >> 5] >> (bit & 31)) & mask;
                        const uint32_t cv = (reinterpret_cast<const uint32_t *>(r + b * D / 8)[bit >> 5] >> (bit & 31)) & mask;
                        kv = fmaf((float)ck, sd.x, sd.y);
                        vv = fmaf((float)cv, sd.z, sd.w);
                    }
                    kT[ch][kk] = kv;
                    vs[kk][ch] = vv;
                }
            } else {
#pragma unroll
                for (int e = 0; e < PL; ++e) {
                    kT[lane + 32 * e][kk] = 0.f;
                    vs[kk][lane + 32 * e] = 0.f;
                }
            }
        }
        __syncthreads();
#pragma unroll
        for (int r = 0; r < kQPW; ++r) {
            const int qi = warp * kQPW + r;
            const int m = q_mode[qi];
            const int t = q_t[qi], lo = q_lo[qi];
            if (m == KVQ_MODE_SKIP || kt > t || kt + kKT - 1 < lo) continue;
            const int j = kt + lane;
            float lg = 0.f;
#pragma unroll 8
            for (int d = 0; d < D; ++d) lg = fmaf(qf[qi][d], kT[d][lane], lg);
            const bool ok = (j >= lo) && (j <= t);
            lg = ok ? lg * scale : -INFINITY;
            float tmax = lg;
#pragma unroll
            for (int d = 16; d >= 1; d >>= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, d));
            const float m_new = fmaxf(m_run[r], tmax);
            const float corr = exp2f(m_run[r] - m_new);
            const float p = ok ? exp2f(lg - m_new) : 0.f;
            float ps = p;
#pragma unroll
            for (int d = 16; d >= 1; d >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, d);
            l_run[r] = fmaf(l_run[r], corr, ps);
            m_run[r] = m_new;
#pragma unroll
            for (int e = 0; e < PL; ++e) o[r][e] *= corr;
            for (int kk = 0; kk < kKT; ++kk) {
                const float pk = __shfl_sync(0xffffffffu, p, kk);
#pragma unroll
                for (int e = 0; e < PL; ++e) o[r][e] = fmaf(pk, vs[kk][lane + 32 * e], o[r][e]);
            }
        }
    }
#pragma unroll
    for (int r = 0; r < kQPW; ++r) {
        const int qi = warp * kQPW + r;
        const int i = i0 + qi;
        if (i >= n_s) continue;
        float *dst = out + ((int64_t)(cu[s] + i) * H + h) * D;
        const bool sk = q_mode[qi] == KVQ_MODE_SKIP || l_run[r] == 0.f;
        const float inv = sk ? 0.f : 1.0f / l_run[r];
#pragma unroll
        for (int e = 0; e < PL; ++e) dst[lane + 32 * e] = sk ? 0.f : o[r][e] * inv;
    }
}

template <int D>
cudaError_t run_simple(dim3 grid, const CacheView &c, const __half *q, const uint8_t *modes, int w,
                       const int32_t *cu, float *out, cudaStream_t st)
{
    const size_t smem = sizeof(float) * (kQT * D + D * (kKT + 1) + kKT * D);
    static bool attr_done = false;
    if (!attr_done) {
        cudaError_t e = cudaFuncSetAttribute(prefill_simple_kernel<D>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        attr_done = true;
    }
    profile_before(st);
    prefill_simple_kernel<D><<<grid, 32 * kWarps, smem, st>>>(c, q, modes, w, cu, out);
    profile_after(st);
    return cudaGetLastError();
}

} // namespace

cudaError_t launch_prefill(const kvq_cache *cache, const __half *q, const uint8_t *modes, int w,
                           const int32_t *cu, int64_t n_tok, float *out, cudaStream_t st)
{
    const CacheView &c = cache->view;
    if (n_tok == 0) return cudaSuccess;
    const int64_t tiles = (n_tok + kQT - 1) / kQT + c.B;   // >= sum_s ceil(n_s / 32)
    dim3 grid((unsigned)tiles, (unsigned)c.H);
    if (c.D == 128) return run_simple<128>(grid, c, q, modes, w, cu, out, st);
    return run_simple<64>(grid, c, q, modes, w, cu, out, st);
}

} // namespace kvq
