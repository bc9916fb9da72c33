// Inference-time router (TriRoute paper review page, section 3 item 5, Eq. 5; and the
// inference paragraph after the training procedure): the controller's attention head
// gives logits z^a over (skip, local, full) and its bit head logits z^b over the widths
// (2, 4, 8, 16) for each (token, head); at inference the router takes the hard argmax.
//
//   route_argmax_kernel  4 rows per thread: the rows' logits arrive as 16-byte loads
//                        (3 float4 for 4 rows of z^a, 4 for z^b), the argmax is a
//                        first-wins scan that passes over NaN, and the 4 results leave
//                        as one 4-byte store per output. Memory-bound: 28 bytes in and
//                        2 bytes out per row.
#include "kvq_internal.cuh"

namespace kvq {
namespace {

template <int K>
__device__ __forceinline__ uint32_t argmax_first(const float *z)
{
    int best = -1;
    float bv = 0.f;
#pragma unroll
    for (int i = 0; i < K; ++i) {
        if (isnan(z[i])) continue;
        if (best < 0 || z[i] > bv) {
            best = i;
            bv = z[i];
        }
    }
    return (uint32_t)(best < 0 ? 0 : best);
}

__device__ __forceinline__ uint32_t width_of(uint32_t idx) { return 2u << idx; }   // 2, 4, 8, 16

__global__ void __launch_bounds__(256)
route_argmax_kernel(const float *__restrict__ za, const float *__restrict__ zb, int64_t n,
                    uint8_t *__restrict__ modes, uint8_t *__restrict__ bits)
{
    pdl_wait();
    pdl_trigger();
    const int64_t r0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 4;
    if (r0 >= n) return;
    if (r0 + 4 <= n) {
        if (za) {
            const float4 *p = reinterpret_cast<const float4 *>(za + r0 * 3);
            float z[12];
            *reinterpret_cast<float4 *>(&z[0]) = p[0];
            *reinterpret_cast<float4 *>(&z[4]) = p[1];
            *reinterpret_cast<float4 *>(&z[8]) = p[2];
            uint32_t o = 0;
#pragma unroll
            for (int r = 0; r < 4; ++r) o |= argmax_first<3>(&z[3 * r]) << (8 * r);
            *reinterpret_cast<uint32_t *>(modes + r0) = o;
        }
        if (zb) {
            const float4 *p = reinterpret_cast<const float4 *>(zb + r0 * 4);
            uint32_t o = 0;
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const float4 v = p[r];
                const float z[4] = {v.x, v.y, v.z, v.w};
                o |= width_of(argmax_first<4>(z)) << (8 * r);
            }
            *reinterpret_cast<uint32_t *>(bits + r0) = o;
        }
    } else {
        for (int64_t r = r0; r < n; ++r) {
            if (za) modes[r] = (uint8_t)argmax_first<3>(za + r * 3);
            if (zb) bits[r] = (uint8_t)width_of(argmax_first<4>(zb + r * 4));
        }
    }
}

} // namespace

cudaError_t launch_route_argmax(const float *za, const float *zb, int64_t n, uint8_t *modes,
                                uint8_t *bits, cudaStream_t st)
{
    if (n == 0) return cudaSuccess;
    const int64_t threads = (n + 3) / 4;
    const int64_t blocks = (threads + 255) / 256;
    return launch_pdl(route_argmax_kernel, dim3((unsigned)blocks), dim3(256), 0, st, za, zb, n, modes, bits);
}

} // namespace kvq
