// Routed causal prefill attention (TriRoute paper review page, section 3, Eq. 2) over the
// mixed-precision cache of Eq. 4, on the sm_100a tensor cores (tcgen05 + TMEM).
//
// Three launches per call:
//   prefill_sched_kernel  one CTA per (sequence, head): compacts the call's queries by
//                         mode (stable) into a local list and a full list, cuts each into tiles of
//                         at most 128 queries, and writes zeros for skip queries. A local
//                         tile reads keys [min(t) - w, max(t)], a full tile [0, max(t)],
//                         so local rows do not pay for a full tile's range.
//   prefill_order_kernel  orders the tiles longest first (keys spanned, descending).
//   prefill_tc_kernel     one CTA per tile, 18 warps:
//     - warps 0-7, softmax: thread = (query row 32 (w % 4) + lane, key half w / 4). Per 64-key
//       tile the thread takes its 32 S values from TMEM, forms the logits
//       s_K * (q.c) + z_K * sum(q) (log2 units, scaled by 1/sqrt(D)) with the row's causal/window
//       mask, runs an online softmax with lazy rescaling over its half, and writes
//       P' = p * s_V as fp16 hi + lo parts to TMEM (fp16 rounding of P alone would cost ~1e-2
//       on outlier channels). Each key half has its own running max and its own O
//       accumulator in TMEM, so the two warps of a row never wait for each other; the halves
//       are merged once at the end.
//     - warps 8-15: unpack each 64-key tile's K and V codes into exact fp16 operands (codes
//       are integers <= 255; b = 16 keys are the fp16 values) in shared memory, three tiles
//       in flight; K 128B-swizzled K-major, V 128B-swizzled MN-major.
//     - warp 16: owns 512 TMEM columns (S double buffer, P', Q, O of each key half) and
//       issues the QK MMAs from one lane: S = Q C_K^T (M128 N64 K16 steps, A = Q in TMEM, B
//       in shared memory) once K(t) is unpacked and S(t-2) has been read; warp 18 issues
//       O_h += P'_h,hi V_h + P'_h,lo V_h per key half h (M128 ND K16, A in TMEM) once P'(t)
//       is written.
//     - warp 17: stages each key tile's records (one contiguous byte range of the stream)
//       with bulk copies and orders the unpack tasks by width, three tiles ahead.
//   All mbarrier waits are bounded; on a timeout the CTA records KVQ_ERR_DEVICE_CHECK,
//   leaves its loops, waits (bounded) for its MMAs and frees its TMEM before returning.
#include "kvq_internal.cuh"

namespace kvq {
namespace {

constexpr int kQRows = 128;     // queries per tile (MMA M)
constexpr int kKeys = 64;       // keys per key tile (QK MMA N, PV MMA K)
// 20 warps: 0-7 softmax (two per row, one per key half), 8-15 K/V unpack, 16 QK issuer,
// 17 record stager, 18 PV issuer (19 idle, present so that the last warpgroup is whole for the
// register split below)
constexpr int kSoftmaxWarps = 8, kSoftmaxThreads = 32 * kSoftmaxWarps;
constexpr int kUnpackWarps = 8, kUnpackThreads = 32 * kUnpackWarps;
constexpr int kMmaWarp = kSoftmaxWarps + kUnpackWarps;
constexpr int kQReadyBar = 3;                   // named barrier: Q in TMEM (softmax warps + QK issuer)
constexpr int kStageWarp = kMmaWarp + 1;
constexpr int kPvWarp = kMmaWarp + 2;
constexpr int kTcThreads = 32 * (kStageWarp + 3);
constexpr int kQP = kUnpackThreads / 64;   // unpack threads per key (the tile's 64 keys)
// Registers: the launch gives every thread kLaunchRegs (65536 / 640 rounded down to a
// multiple of 8); setmaxnreg at the head of each role then moves them between warpgroups:
// softmax kRegSoftmax, unpack kRegUnpack, MMA/stager warpgroup kRegMma per thread. The sum
// stays within the launch's allocation; the host refuses to launch when the compiled
// register count differs from kLaunchRegs.
constexpr int kLaunchRegs = 96, kRegSoftmax = 144, kRegUnpack = 80, kRegMma = 32;
static_assert(kTcThreads * kLaunchRegs <= 65536, "launch registers");
static_assert(kSoftmaxThreads * kRegSoftmax + kUnpackThreads * kRegUnpack + 128 * kRegMma <= kTcThreads * kLaunchRegs,
              "register split exceeds the launch");
constexpr int kRawBufs = 3;     // record staging buffers: a key tile's records land up to three tiles ahead
constexpr int kKvBufs = 3;      // unpacked K/V operand tiles in flight
constexpr uint32_t kTmemCols = 512;
// TMEM columns: S double buffer (fp32, 64 keys) at 0 and 64; P' at 128, holding per key half h
// the fp16 pairs of P'_hi (16 columns) then P'_lo (16) at 32 h; Q (fp16 pairs, D / 2 columns)
// at 192; O of key half h (fp32, D columns) at 256 + h D. S is double buffered so that QK(t+1)
// never waits for the softmax of tile t; one P' buffer suffices because PV(t-1) has long
// completed when the softmax of tile t writes P'(t).
constexpr uint32_t kTmemS = 0, kTmemP = 128, kTmemQ = 192, kTmemO = 256;

// ---- tcgen05 / UMMA helpers -------------------------------------------------------
// Shared-memory matrix descriptor, 128-byte swizzle (layout type 2), descriptor version 1.
__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes)
{
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor, kind::f16: fp16 A/B, fp32 accumulator, M = 128.
__host__ __device__ constexpr uint32_t umma_idesc(int n, bool b_mn_major)
{
    return (1u << 4) | ((b_mn_major ? 1u : 0u) << 16) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}

// D (TMEM) [+]= A (TMEM, K-major: row = lane, 2 fp16 per 32-bit column) * B (shared)
__device__ __forceinline__ void umma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b, uint32_t idesc, bool acc)
{
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
                 ::"r"(d_tmem), "r"(a_tmem), "l"(b), "r"(idesc), "r"((uint32_t)acc)
                 : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t *bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32])
{
    uint32_t r[32];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 "
                 "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
                 "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                   "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
                   "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
                   "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
                   "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
                 : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32])
{
    asm volatile("tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
                 "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
                 "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
                 ::"r"(taddr), "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])),
                   "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])),
                   "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
                   "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])),
                   "r"(__float_as_uint(v[11])), "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])),
                   "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])),
                   "r"(__float_as_uint(v[17])), "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])),
                   "r"(__float_as_uint(v[20])), "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])),
                   "r"(__float_as_uint(v[23])), "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])),
                   "r"(__float_as_uint(v[26])), "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])),
                   "r"(__float_as_uint(v[29])), "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
                 : "memory");
}

__device__ __forceinline__ void tmem_st32u(uint32_t taddr, const uint32_t (&v)[32])
{
    asm volatile("tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
                 "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
                 "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
                 ::"r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]),
                   "r"(v[7]), "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
                   "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]),
                   "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]),
                   "r"(v[29]), "r"(v[30]), "r"(v[31])
                 : "memory");
}

__device__ __forceinline__ void tmem_st16u(uint32_t taddr, const uint32_t (&v)[16])
{
    asm volatile("tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
                 "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
                 ::"r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]),
                   "r"(v[7]), "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
                   "r"(v[15])
                 : "memory");
}

// byte offset of the 16-byte chunk `cc` (0..7) of row r inside a 128B-swizzled K-major
// block of rows (rows of 128 bytes, 8-row atoms of 1024 bytes)
__device__ __forceinline__ uint32_t kmajor_off(int r, int cc)
{
    return (uint32_t)((r >> 3) * 1024 + (r & 7) * 128 + ((cc ^ (r & 7)) << 4));
}

// fp16 operands holding integer codes. A word whose two halves are 0x64cc (the fp16
// number 1024 + c for a code c < 1024) minus (1024, 1024) is the half2 (c0, c1), exactly.
__device__ __forceinline__ uint32_t h2_minus_1024(uint32_t h)
{
    uint32_t r;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(h), "r"(0x64006400u));
    return r;
}

// two codes sitting in bytes 0 and 2 of `t` (other bits arbitrary) -> half2 (c0, c1)
__device__ __forceinline__ uint32_t bytes02_to_h2(uint32_t t, uint32_t mask)
{
    return h2_minus_1024((t & mask) | 0x64006400u);
}

// 8 channels starting at channel 8*chunk of a packed part -> 16 bytes of fp16 (registers only)
__device__ __forceinline__ uint4 unpack8(const uint8_t *part, int bits, int chunk)
{
    if (bits == 16) return reinterpret_cast<const uint4 *>(part)[chunk];
    uint32_t w0, w1, w2, w3;
    if (bits == 8) {
        const uint2 x = reinterpret_cast<const uint2 *>(part)[chunk];
        // bytes (c0, 0x64, c1, 0x64) via byte permutes, then - 1024
        w0 = h2_minus_1024(__byte_perm(x.x, 0x64646464u, 0x5140));
        w1 = h2_minus_1024(__byte_perm(x.x, 0x64646464u, 0x5342));
        w2 = h2_minus_1024(__byte_perm(x.y, 0x64646464u, 0x5140));
        w3 = h2_minus_1024(__byte_perm(x.y, 0x64646464u, 0x5342));
    } else if (bits == 4) {
        const uint32_t x = reinterpret_cast<const uint32_t *>(part)[chunk];
        const uint32_t lo = x & 0x0F0F0F0Fu, hi = (x >> 4) & 0x0F0F0F0Fu;   // even / odd channels
        // pair k = (lo byte k, hi byte k) placed in bytes 0 and 2
        w0 = bytes02_to_h2(__byte_perm(lo, hi, 0x0400), 0x00FF00FFu);
        w1 = bytes02_to_h2(__byte_perm(lo, hi, 0x0501), 0x00FF00FFu);
        w2 = bytes02_to_h2(__byte_perm(lo, hi, 0x0602), 0x00FF00FFu);
        w3 = bytes02_to_h2(__byte_perm(lo, hi, 0x0703), 0x00FF00FFu);
    } else {
        const uint32_t x = reinterpret_cast<const uint16_t *>(part)[chunk];
        // channel 2k at bits 4k, channel 2k+1 at bits 4k+2: move the odd ones up by 14
        const uint32_t y = (x & 0x3333u) | ((x & 0xCCCCu) << 14);        // even: bits 4k, odd: bits 16+4k
        w0 = bytes02_to_h2(y, 0x00030003u);
        w1 = bytes02_to_h2(y >> 4, 0x00030003u);
        w2 = bytes02_to_h2(y >> 8, 0x00030003u);
        w3 = bytes02_to_h2(y >> 12, 0x00030003u);
    }
    return make_uint4(w0, w1, w2, w3);
}

// 2^x with the hardware's approximate exp2 (relative error of a few ulp), used for the
// softmax weights; 2^-inf = 0. Results below 2^-126 flush to zero: a weight that small is
// below 2^-118 of the row's sum (which holds a weight >= 2^-8), far under the tolerance.
__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

struct PfTile {
    int32_t sh, mode, start, count;   // (sequence, head), mode, first list entry, queries
    int32_t nkeys, pad[3];            // keys the tile's range spans (its work, for ordering)
};

template <int D>
struct alignas(1024) PfSmem {
    __half k[kKvBufs][kKeys * D];     // K-major SW128, D/64 blocks of 64 rows x 128 B
    __half v[kKvBufs][kKeys * D];     // MN-major SW128: atom (8 keys x 64 ch) at (key/8)*(D/64)+ch/64
    // side entries of key pairs (2j, 2j + 1), laid out for packed fp32 arithmetic:
    float4 side_k[kKvBufs][kKeys / 2];   // (s_K c, s_K c, z_K c, z_K c), c = log2(e)/sqrt(D)
    float4 side_v[kKvBufs][kKeys / 2];   // (s_V, s_V, z_V, z_V)
    uint8_t raw[kRawBufs][kKeys * 4 * D];   // a key tile's records as stored (one contiguous range
                                            // of the stream; at most 64 keys x 2 x D fp16 values)
    // the tile's keys ordered by width class (class 4: no key):
    // offset of the key's record in raw << 16 | class << 8 | key
    uint32_t task[kRawBufs][kKeys];
    float4 fin[2][kQRows];            // per key half: (running max, l, sum p z_V) of each row
    float qpart[2][kQRows];           // per half of the channels: partial sums of each Q row
    uint64_t raw_full[kRawBufs], raw_empty[kRawBufs], kv_full[kKvBufs], kv_empty[kKvBufs];
    uint64_t s_full[2], s_free[2], p_full, pv_done, drain;
    uint32_t tmem_base;
    int32_t klo, khi, abort_flag;
};

template <int D>
__global__ void __launch_bounds__(kTcThreads, 1)
prefill_tc_kernel(CacheView c, const __half *__restrict__ q, int w, const int32_t *__restrict__ cu,
                  const PfTile *__restrict__ tiles, const int32_t *__restrict__ tile_count,
                  const int32_t *__restrict__ qidx, float *__restrict__ out)
{
    if ((int)blockIdx.x >= *tile_count) return;
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned (the 128B-swizzled operand tiles): offset the shared pointer itself,
    // so that the compiler keeps every access in the shared address space
    PfSmem<D> &sm = *reinterpret_cast<PfSmem<D> *>(smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u));
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const PfTile tile = tiles[blockIdx.x];
    // tile.sh = (sequence, query head); query head hq reads KV head hq / G
    const int H = c.H * c.G, sh = tile.sh, s = sh / H, h = sh % H, hk = h / c.G;
    const int n_s = cu[s + 1] - cu[s];
    const int pos0 = c.len[s * c.H + hk] - n_s;
    const int64_t sbase = slot_of(c, s, hk, 0);
    const RecLoc stream = rec_loc(c, s, hk, 0);

    if (tid == 0) {
        for (int i = 0; i < kKvBufs; ++i) {
            mbar_init(&sm.kv_full[i], kUnpackWarps);
            mbar_init(&sm.kv_empty[i], 1);
        }
        for (int i = 0; i < kRawBufs; ++i) {
            mbar_init(&sm.raw_full[i], 1);
            mbar_init(&sm.raw_empty[i], kUnpackWarps);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sm.s_full[i], 1);
            mbar_init(&sm.s_free[i], kSoftmaxWarps);
        }
        mbar_init(&sm.p_full, kSoftmaxWarps);
        mbar_init(&sm.pv_done, 1);
        mbar_init(&sm.drain, 2);
        // the tile's key range, from its first and last query: a tile's query list is
        // monotonic (local queries ascending, full queries descending), so these hold the
        // smallest and the largest position; each row checks its own range below
        sm.klo = INT32_MAX;
        sm.khi = -1;
        if (tile.count > 0) {
            const int ia = qidx[tile.start], ib = qidx[tile.start + tile.count - 1];
            sm.khi = pos0 + max(ia, ib);
            sm.klo = (tile.mode == KVQ_MODE_LOCAL) ? max(0, pos0 + min(ia, ib) - w) : 0;
        }
        sm.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(&sm.tmem_base)), "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    // ---- prologue: query rows (softmax warps; the two warps of a row load half the
    // channels each into the Q columns of TMEM). The stager and the unpack warps start on
    // the first key tiles meanwhile; the QK issuer waits for Q at a named barrier. ----
    const int kh = warp / 4;                       // softmax: key half (and channel half of Q)
    const int row = 32 * (warp & 3) + lane;
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
    int row_t = -1, row_lo = 0, row_i = -1;
    if (warp < kSoftmaxWarps) {
        const bool valid = row < tile.count;
        if (valid) {
            row_i = qidx[tile.start + row];
            row_t = pos0 + row_i;
            row_lo = (tile.mode == KVQ_MODE_LOCAL) ? max(0, row_t - w) : 0;
            if (kh == 0 && (row_lo < sm.klo || row_t > sm.khi)) set_status(c.status, KVQ_ERR_DEVICE_CHECK);
        }
        const uint4 *src = reinterpret_cast<const uint4 *>(q + ((int64_t)(cu[s] + max(row_i, 0)) * H + h) * D) + kh * (D / 16);
        uint32_t words[D / 4];
        float part = 0.f;
#pragma unroll
        for (int ch = 0; ch < D / 16; ++ch) {
            const uint4 x = valid ? src[ch] : make_uint4(0, 0, 0, 0);
            words[4 * ch] = x.x;
            words[4 * ch + 1] = x.y;
            words[4 * ch + 2] = x.z;
            words[4 * ch + 3] = x.w;
            const __half2 *hx = reinterpret_cast<const __half2 *>(&x);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = __half22float2(hx[e]);
                part += f.x + f.y;
            }
        }
        if constexpr (D == 128) {
            tmem_st32u(tmem + lane_base + kTmemQ + 32 * kh, words);
        } else {
            tmem_st16u(tmem + lane_base + kTmemQ + 16 * kh, words);
        }
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
        sm.qpart[kh][row] = part;
        tc_fence_before();
        named_bar_sync(kQReadyBar, kSoftmaxThreads + 32);   // Q in TMEM, with the QK issuer
    }
    const int klo = sm.klo, khi = sm.khi;
    const int n_kt = (khi >= klo) ? (khi - klo + kKeys) / kKeys : 0;
    if (warp >= kMmaWarp) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegMma));
    }
    // ---- MMA issue (warp 16: QK, warp 18: PV), one lane each ----
    constexpr uint32_t idesc_qk = umma_idesc(kKeys, false);
    constexpr uint32_t idesc_pv = umma_idesc(D, true);
    constexpr uint32_t v_sbo = (D / 64) * 1024;       // next 8 keys
    auto issue_qk = [&](int t) {
        tc_fence_after();
        const uint32_t k0 = smem_u32(sm.k[t % kKvBufs]);
        if (lane == 0) {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint64_t db = umma_desc(k0 + (kk >> 2) * (kKeys * 128) + (kk & 3) * 32, 16, 1024);
                umma_f16_ts(tmem + kTmemS + 64 * (t & 1), tmem + kTmemQ + 8 * kk, db, idesc_qk, kk > 0);
            }
            umma_commit(&sm.s_full[t & 1]);
        }
        __syncwarp();
    };
    auto issue_pv = [&](int t) {
        tc_fence_after();
        const uint32_t v0 = smem_u32(sm.v[t % kKvBufs]);
        if (lane == 0) {
#pragma unroll
            for (int half = 0; half < 2; ++half) {
#pragma unroll
                for (int part = 0; part < 2; ++part) {
                    // P'_hi then P'_lo of key half `half`: 8 TMEM columns per 16 keys
                    const uint32_t pa = tmem + kTmemP + 32 * half + 16 * part;
#pragma unroll
                    for (int k2 = 0; k2 < 2; ++k2) {
                        const int kk = 2 * half + k2;         // 16-key step of the tile
                        const uint64_t db = umma_desc(v0 + 2 * kk * v_sbo, 1024, v_sbo);
                        umma_f16_ts(tmem + kTmemO + half * D, pa + 8 * k2, db, idesc_pv, part > 0 || t > 0 || k2 > 0);
                    }
                }
            }
            umma_commit(&sm.pv_done);
            umma_commit(&sm.kv_empty[t % kKvBufs]);
        }
        __syncwarp();
    };
    if (warp == kMmaWarp) {
        // QK(t) once K(t) is unpacked and the softmax has read S(t-2); the PV MMAs come from
        // their own warp. Both wait on their barriers (suspended, no polling).
        named_bar_sync(kQReadyBar, kSoftmaxThreads + 32);       // the query rows are in TMEM
        for (int t = 0; t < n_kt; ++t) {
            if (!__all_sync(0xffffffffu, mbar_wait(&sm.kv_full[t % kKvBufs], (t / kKvBufs) & 1, c.status) &&
                                             (t < 2 || mbar_wait(&sm.s_free[t & 1], ((t - 2) >> 1) & 1, c.status)) &&
                                             !*reinterpret_cast<volatile int *>(&sm.abort_flag))) {
                sm.abort_flag = 1;
                break;
            }
            issue_qk(t);
        }
        // every MMA this warp issued has completed before the TMEM is freed (bounded wait)
        if (lane == 0) umma_commit(&sm.drain);
        __syncwarp();
        mbar_wait(&sm.drain, 0, c.status);
    } else if (warp == kPvWarp) {
        // ------------------------------- PV issuer ---------------------------------
        // PV(t) once P'(t) is in TMEM (which implies that QK(t) has completed)
        for (int t = 0; t < n_kt; ++t) {
            if (!__all_sync(0xffffffffu, mbar_wait(&sm.p_full, t & 1, c.status) &&
                                             !*reinterpret_cast<volatile int *>(&sm.abort_flag))) {
                sm.abort_flag = 1;
                break;
            }
            issue_pv(t);
        }
        if (lane == 0) umma_commit(&sm.drain);
        __syncwarp();
        mbar_wait(&sm.drain, 0, c.status);
    } else if (warp == kStageWarp) {
        // ------------------------------ record stager ------------------------------------
        // Per key tile: the 64 keys' record words, the tile's byte range in the stream (the
        // records of consecutive keys are contiguous), one bulk copy of that range (cut at
        // page ends) into a staging buffer, and the conversion tasks ordered by width class
        // so that each unpack warp's lanes run one width's conversion.
        constexpr uint32_t kNone = 0xFFFFFFFFu;
        auto meta_of = [&](int t, int k) -> uint32_t {
            const int j = klo + t * kKeys + k;
            return (t < n_kt && j <= khi) ? c.meta[sbase + j] : kNone;
        };
        uint32_t ma = meta_of(0, lane), mb = meta_of(0, 32 + lane);
        const uint32_t lt = (1u << lane) - 1u;
        int issued = 0;
        for (int t = 0; t < n_kt; ++t) {
            const int st = t % kRawBufs;
            const uint32_t na = meta_of(t + 1, lane), nb = meta_of(t + 1, 32 + lane);   // next tile, in flight
            if (t >= kRawBufs &&
                !__all_sync(0xffffffffu, mbar_wait(&sm.raw_empty[st], ((t / kRawBufs) - 1) & 1, c.status) &&
                                             !*reinterpret_cast<volatile int *>(&sm.abort_flag))) {
                sm.abort_flag = 1;
                break;
            }
            const int ca = (ma == kNone) ? 4 : (int)(ma & 3u), cb = (mb == kNone) ? 4 : (int)(mb & 3u);
            // byte range: from the first key's record (always present) to the end of the last
            const uint32_t base = __shfl_sync(0xffffffffu, ma, 0) & ~15u;
            const uint32_t va = __ballot_sync(0xffffffffu, ma != kNone), vb = __ballot_sync(0xffffffffu, mb != kNone);
            const int last = vb ? 63 - __clz(vb) : 31 - __clz(va);
            const uint32_t ml = __shfl_sync(0xffffffffu, last >= 32 ? mb : ma, last & 31);
            const uint32_t end = (ml & ~15u) + (uint32_t)((2 << (ml & 3u)) * D / 4);    // K and V parts
            if (end - base > (uint32_t)sizeof(sm.raw[0])) {      // records not contiguous: corrupt cache
                if (lane == 0) set_status(c.status, KVQ_ERR_DEVICE_CHECK);
                sm.abort_flag = 1;
                break;
            }
            // stable order by class (none last): key position among the tile's keys
            int pa = 0, pb = 0, start = 0;
#pragma unroll
            for (int c2 = 0; c2 < 5; ++c2) {
                const uint32_t ba = __ballot_sync(0xffffffffu, ca == c2), bb = __ballot_sync(0xffffffffu, cb == c2);
                if (ca == c2) pa = start + __popc(ba & lt);
                if (cb == c2) pb = start + __popc(ba) + __popc(bb & lt);
                start += __popc(ba) + __popc(bb);
            }
            sm.task[st][pa] = ((ca < 4 ? (ma & ~15u) - base : 0u) << 16) | ((uint32_t)ca << 8) | (uint32_t)lane;
            sm.task[st][pb] = ((cb < 4 ? (mb & ~15u) - base : 0u) << 16) | ((uint32_t)cb << 8) | (uint32_t)(32 + lane);
            __syncwarp();
            if (lane == 0) {
                mbar_arrive_expect_tx(&sm.raw_full[st], end - base);
                for (uint32_t o = base; o < end;) {
                    uint32_t e2 = end;
                    if (stream.pt) {                          // not past the page holding o
                        const uint32_t pg_end = (((stream.off + o) >> stream.shift) + 1u) << stream.shift;
                        e2 = min(end, pg_end - stream.off);
                    }
                    bulk_g2s(sm.raw[st] + (o - base), stream.at(o), e2 - o, &sm.raw_full[st]);
                    o = e2;
                }
            }
            __syncwarp();
            ++issued;
            ma = na;
            mb = nb;
        }
        // the staging buffers must not receive bytes after the CTA ends: wait (bounded) for
        // the copies of the last tiles (earlier ones were consumed before their buffer came back)
        for (int t = max(0, issued - kRawBufs); t < issued; ++t)
            mbar_wait(&sm.raw_full[t % kRawBufs], (t / kRawBufs) & 1, c.status);
    } else if (warp >= kSoftmaxWarps && warp < kMmaWarp) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegUnpack));
        // ------------------------------ K/V unpack -----------------------------------
        // Each warp converts 8 keys of the class-ordered list, D/8 lanes per key and one
        // 8-channel chunk per lane, so that a quarter warp reads 128 consecutive staged bytes
        // and writes eight distinct 16-byte slots of a swizzled row (no bank conflicts). The
        // side entry of key kj = u / 4 is loaded three tiles ahead by one thread in four.
        const int u = tid - kSoftmaxThreads;
        const int kj = u / kQP, half = u % kQP;
        constexpr int kCpr = D / 8;                  // 8-channel chunks per row
        constexpr int kKpp = 32 / kCpr;              // keys per pass of a warp
        const int uw = u >> 5, chunk = lane % kCpr, kslot = lane / kCpr;
        auto load_side = [&](int t) -> float4 {
            const int j = klo + t * kKeys + kj;
            return (half == 0 && t < n_kt && j <= khi) ? c.side[sbase + j] : make_float4(0.f, 0.f, 0.f, 0.f);
        };
        float4 sd_cur = load_side(0), sd_n1 = load_side(1), sd_n2 = load_side(2);
        for (int t = 0; t < n_kt; ++t) {
            const int b = t % kKvBufs, st = t % kRawBufs;
            const float4 sd_n3 = load_side(t + 3);
            if (!__all_sync(0xffffffffu, mbar_wait(&sm.raw_full[st], (t / kRawBufs) & 1, c.status) &&
                                             mbar_wait(&sm.kv_empty[b], ((t / kKvBufs) & 1) ^ 1, c.status) &&
                                             !*reinterpret_cast<volatile int *>(&sm.abort_flag))) {
                sm.abort_flag = 1;
                break;
            }
            uint8_t *kb = reinterpret_cast<uint8_t *>(sm.k[b]);
            uint8_t *vb = reinterpret_cast<uint8_t *>(sm.v[b]);
            if (half == 0) {
                const float lsc = kLog2e * rsqrtf((float)D);
                float *sk = reinterpret_cast<float *>(&sm.side_k[b][kj >> 1]) + (kj & 1);
                float *sv = reinterpret_cast<float *>(&sm.side_v[b][kj >> 1]) + (kj & 1);
                sk[0] = sd_cur.x * lsc;
                sk[2] = sd_cur.y * lsc;
                sv[0] = sd_cur.z;
                sv[2] = sd_cur.w;
            }
#pragma unroll
            for (int pass = 0; pass < 8 / kKpp; ++pass) {
                const uint32_t task = sm.task[st][8 * uw + kKpp * pass + kslot];
                const int cls = (int)((task >> 8) & 7u), tkj = (int)(task & 63u);
                const int bits = (cls < 4) ? (2 << cls) : 0;
                const uint8_t *ksrc = sm.raw[st] + (task >> 16);
                const uint4 kx = bits ? unpack8(ksrc, bits, chunk) : make_uint4(0, 0, 0, 0);
                const uint4 vx = bits ? unpack8(ksrc + bits * D / 8, bits, chunk) : make_uint4(0, 0, 0, 0);
                *reinterpret_cast<uint4 *>(kb + (chunk >> 3) * (kKeys * 128) + kmajor_off(tkj, chunk & 7)) = kx;
                const int n = chunk * 8;
                const int atom = (tkj >> 3) * (D / 64) + (n >> 6);
                *reinterpret_cast<uint4 *>(vb + atom * 1024 + (tkj & 7) * 128 + ((((n & 63) >> 3) ^ (tkj & 7)) << 4)) = vx;
            }
            fence_async_smem();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&sm.kv_full[b]);
                mbar_arrive(&sm.raw_empty[st]);
            }
            sd_cur = sd_n1;
            sd_n1 = sd_n2;
            sd_n2 = sd_n3;
        }
    } else if (warp < kSoftmaxWarps) {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegSoftmax));
        // ------------------------------ softmax rows ---------------------------------
        // This thread: row `row`, keys 32 kh .. 32 kh + 31 of every tile.
        const float qsum = sm.qpart[0][row] + sm.qpart[1][row];
        const float2 qs2 = make_float2(qsum, qsum);
        const uint32_t o_col = kTmemO + kh * D;
        float m_run = -INFINITY;
        float2 l_run = make_float2(0.f, 0.f), pz_run = make_float2(0.f, 0.f);   // even / odd keys
        bool ok = true;
        for (int t = 0; t < n_kt; ++t) {
            const int st = t % kKvBufs;
            // warp-uniform outcome: the TMEM accesses below are .sync.aligned
            if (!__all_sync(0xffffffffu, mbar_wait(&sm.s_full[t & 1], (t >> 1) & 1, c.status) &&
                                             !*reinterpret_cast<volatile int *>(&sm.abort_flag))) {
                sm.abort_flag = 1;
                ok = false;
                break;
            }
            tc_fence_after();
            float sv[32];
            tmem_ld32(tmem + lane_base + kTmemS + 64 * (t & 1) + 32 * kh, sv);
            // S may now be overwritten by QK(t+1)
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.s_free[t & 1]);
            const int kt0 = klo + t * kKeys + 32 * kh;
            // the row's keys in this half tile: [max(row_lo, kt0), min(row_t, kt0 + 31)]
            const int c_lo = max(row_lo - kt0, 0), c_hi = min(row_t - kt0, 31);
            const bool interior = __all_sync(0xffffffffu, c_lo == 0 && c_hi == 31);
            // Logits in log2 units relative to the running max, in one pass over key pairs:
            // e = s_K c (q.c) + (z_K c Sum(q) - m). A half with no key yet uses m = 0.
            const float mref = (m_run == -INFINITY) ? 0.f : m_run;
            const float2 nm2 = make_float2(-mref, -mref);
            const float4 *skp = &sm.side_k[st][16 * kh];
            float2 e[16];
            float mx = -INFINITY;
            if (interior) {
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const float4 sk = skp[j];
                    e[j] = __ffma2_rn(make_float2(sk.x, sk.y), make_float2(sv[2 * j], sv[2 * j + 1]),
                                      __ffma2_rn(make_float2(sk.z, sk.w), qs2, nm2));
                    mx = fmaxf(mx, fmaxf(e[j].x, e[j].y));
                }
            } else {
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const float4 sk = skp[j];
                    float2 x = __ffma2_rn(make_float2(sk.x, sk.y), make_float2(sv[2 * j], sv[2 * j + 1]),
                                          __ffma2_rn(make_float2(sk.z, sk.w), qs2, nm2));
                    x.x = (2 * j >= c_lo && 2 * j <= c_hi) ? x.x : -INFINITY;
                    x.y = (2 * j + 1 >= c_lo && 2 * j + 1 <= c_hi) ? x.y : -INFINITY;
                    e[j] = x;
                    mx = fmaxf(mx, fmaxf(x.x, x.y));
                }
            }
            /*TRACE_MAX*/
            // Lazy rescaling: the half keeps its running max until a key exceeds it by more
            // than 8 (so p <= 2^8 fits fp16 after the s_V scale); then the logits, O, l and
            // pz move to the new max. The final merge uses each half's max, so the result
            // is unchanged.
            const bool bump = (m_run == -INFINITY) ? (mx > -INFINITY) : (mx > 8.f);
            float corr = 1.f;
            if (__any_sync(0xffffffffu, bump)) {
                const float d = bump ? mx : 0.f;
                const float2 nd2 = make_float2(-d, -d);
#pragma unroll
                for (int j = 0; j < 16; ++j) e[j] = __fadd2_rn(e[j], nd2);
                if (bump) {
                    corr = (m_run == -INFINITY) ? 0.f : ex2(-mx);
                    m_run = mref + mx;
                }
            }
            const float4 *svp = &sm.side_v[st][16 * kh];
            float2 psum = make_float2(0.f, 0.f), pz = make_float2(0.f, 0.f);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const float4 svz = svp[j];
                const float2 p = make_float2(ex2(e[j].x), ex2(e[j].y));   // 2^-inf = 0: masked keys
                psum = __fadd2_rn(psum, p);
                pz = __ffma2_rn(p, make_float2(svz.z, svz.w), pz);
                e[j] = __fmul2_rn(p, make_float2(svz.x, svz.y));           // P' = p * s_V
            }
            const float2 corr2 = make_float2(corr, corr);
            l_run = __ffma2_rn(l_run, corr2, psum);
            pz_run = __ffma2_rn(pz_run, corr2, pz);
            /*TRACE_EXP*/
            // P' was last read by PV(t-1), which a rescale of O also needs complete
            const bool rescale = t > 0 && __any_sync(0xffffffffu, bump);
            /*TRACE_RESC*/
            if (t > 0) {
                if (!__all_sync(0xffffffffu, mbar_wait(&sm.pv_done, (t - 1) & 1, c.status))) {
                    sm.abort_flag = 1;
                    ok = false;
                    break;
                }
                tc_fence_after();
            }
            /*TRACE_PVW*/
            if (rescale) {                                  // rescale this half's O rows
#pragma unroll
                for (int cb = 0; cb < D / 32; ++cb) {
                    float ov[32];
                    tmem_ld32(tmem + lane_base + o_col + cb * 32, ov);
#pragma unroll
                    for (int i = 0; i < 32; ++i) ov[i] *= corr;
                    tmem_st32(tmem + lane_base + o_col + cb * 32, ov);
                }
            }
            // P' = hi + lo, both fp16: column j of this half's 16 holds keys (2j, 2j + 1)
            {
                uint32_t hw[16], lw[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float2 a = e[i];
                    const __half2 hv = __float22half2_rn(a);
                    const float2 hfv = __half22float2(hv);
                    const __half2 lv = __float22half2_rn(__fadd2_rn(a, make_float2(-hfv.x, -hfv.y)));
                    hw[i] = *reinterpret_cast<const uint32_t *>(&hv);
                    lw[i] = *reinterpret_cast<const uint32_t *>(&lv);
                }
                tmem_st16u(tmem + lane_base + kTmemP + 32 * kh, hw);
                tmem_st16u(tmem + lane_base + kTmemP + 32 * kh + 16, lw);
            }
            asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.p_full);
        }
        // ---- merge the two key halves of each row; each warp writes half the channels ----
        const int t_last = n_kt - 1;
        if (ok && n_kt > 0 &&
            !__all_sync(0xffffffffu, mbar_wait(&sm.pv_done, t_last & 1, c.status)))
            ok = false;
        tc_fence_after();
        sm.fin[kh][row] = make_float4(m_run, l_run.x + l_run.y, pz_run.x + pz_run.y, 0.f);
        // every softmax warp reaches this barrier, aborted or not
        if (named_bar_or(1, kSoftmaxThreads, !ok)) {
            if (row_t >= 0) sm.abort_flag = 1;
        } else {
            const float4 fa = sm.fin[0][row], fb = sm.fin[1][row];
            const float m = fmaxf(fa.x, fb.x);
            const float wa = (fa.x == -INFINITY) ? 0.f : ex2(fa.x - m);
            const float wb = (fb.x == -INFINITY) ? 0.f : ex2(fb.x - m);
            const float l = fa.y * wa + fb.y * wb, pzs = fa.z * wa + fb.z * wb;
            const float inv = (l > 0.f) ? 1.0f / l : 0.f;
            const bool write = row_t >= 0;
            float *dst = out + ((int64_t)(cu[s] + max(row_i, 0)) * H + h) * D + kh * (D / 2);
#pragma unroll
            for (int cb = 0; cb < D / 64; ++cb) {
                float oa[32], ob[32];
                tmem_ld32(tmem + lane_base + kTmemO + kh * (D / 2) + cb * 32, oa);
                tmem_ld32(tmem + lane_base + kTmemO + D + kh * (D / 2) + cb * 32, ob);
                if (write) {
#pragma unroll
                    for (int e = 0; e < 32; e += 4)
                        *reinterpret_cast<float4 *>(dst + cb * 32 + e) =
                            make_float4((fmaf(oa[e], wa, ob[e] * wb) + pzs) * inv,
                                        (fmaf(oa[e + 1], wa, ob[e + 1] * wb) + pzs) * inv,
                                        (fmaf(oa[e + 2], wa, ob[e + 2] * wb) + pzs) * inv,
                                        (fmaf(oa[e + 3], wa, ob[e + 3] * wb) + pzs) * inv);
                }
            }
        }
    }

    // ---- teardown: every role ends here; TMEM is freed even after an abort ----
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
    }
}

// One CTA per (sequence, head): stable compaction of the call's queries by mode, 4096
// queries per pass (4 consecutive queries per thread, block prefix sum of the per-thread
// counts packed as local | full << 16). Skip rows are zeroed a whole row per warp store.
constexpr int kSchedThreads = 1024, kSchedPer = 4;

__global__ void __launch_bounds__(kSchedThreads)
prefill_sched_kernel(CacheView c, const uint8_t *__restrict__ modes, int w, const int32_t *__restrict__ cu,
                     int64_t n_tok, int D, float *__restrict__ out, PfTile *__restrict__ tiles,
                     int32_t *__restrict__ tile_count, int32_t *__restrict__ qidx)
{
    __shared__ int wsum[kSchedThreads / 32];
    __shared__ int carry_l, carry_f;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    // one CTA per (sequence, query head); query head h reads KV head h / G
    const int H = c.H * c.G, sh = blockIdx.x, s = sh / H, h = sh % H;
    const int64_t t0 = cu[s], t1 = cu[s + 1];
    if (t0 < 0 || t1 < t0 || t1 > n_tok) return;      // flagged by the write's checks
    const int n = (int)(t1 - t0);
    if (n == 0) return;
    if (c.len[s * c.H + h / c.G] - n < 0) {
        if (tid == 0) set_status(c.status, KVQ_ERR_DEVICE_CHECK);
        return;
    }
    int32_t *region = qidx + t0 * H + (int64_t)h * n;    // local from the front, full from the back
    if (tid == 0) {
        carry_l = 0;
        carry_f = 0;
    }
    constexpr int kPass = kSchedThreads * kSchedPer;
    for (int base = 0; base < n; base += kPass) {
        int m[kSchedPer];
        int cnt = 0;                                     // local | full << 16
#pragma unroll
        for (int k = 0; k < kSchedPer; ++k) {
            const int i = base + tid * kSchedPer + k;
            m[k] = -1;
            if (i < n) {
                m[k] = modes[(t0 + i) * H + h];
                if (m[k] > KVQ_MODE_FULL) {
                    set_status(c.status, KVQ_ERR_MODE);
                    m[k] = KVQ_MODE_SKIP;
                }
            }
            cnt += (m[k] == KVQ_MODE_LOCAL) ? 1 : (m[k] == KVQ_MODE_FULL) ? (1 << 16) : 0;
        }
        int incl = cnt;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int o = __shfl_up_sync(0xffffffffu, incl, d);
            if (lane >= d) incl += o;
        }
        if (lane == 31) wsum[wid] = incl;
        __syncthreads();
        if (wid == 0) {
            const int x = wsum[lane];
            int y = x;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const int o = __shfl_up_sync(0xffffffffu, y, d);
                if (lane >= d) y += o;
            }
            wsum[lane] = y - x;                          // exclusive prefix of the warps
        }
        __syncthreads();
        const int pre = wsum[wid] + incl - cnt;
        int pl = carry_l + (pre & 0xFFFF), pf = carry_f + (pre >> 16);
#pragma unroll
        for (int k = 0; k < kSchedPer; ++k) {
            const int i = base + tid * kSchedPer + k;
            if (m[k] == KVQ_MODE_LOCAL) region[pl++] = i;
            if (m[k] == KVQ_MODE_FULL) region[n - 1 - (pf++)] = i;
        }
        // zeros for skip rows: one row of D floats per warp store
#pragma unroll
        for (int k = 0; k < kSchedPer; ++k) {
            uint32_t skip = __ballot_sync(0xffffffffu, m[k] == KVQ_MODE_SKIP);
            while (skip) {
                const int src = __ffs(skip) - 1;
                skip &= skip - 1;
                const int64_t row = (t0 + base + (wid * 32 + src) * kSchedPer + k) * H + h;
                if (lane < D / 4)
                    reinterpret_cast<float4 *>(out + row * D)[lane] = make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
        __syncthreads();
        if (tid == kSchedThreads - 1) {                  // its pl, pf are the pass totals
            carry_l = pl;
            carry_f = pf;
        }
        __syncthreads();
    }
    if (tid == 0) {
        const int tot_l = carry_l, tot_f = carry_f;
        const int ntl = (tot_l + kQRows - 1) / kQRows, ntf = (tot_f + kQRows - 1) / kQRows;
        const int first = atomicAdd(tile_count, ntl + ntf);
        const int32_t off = (int32_t)(t0 * H + (int64_t)h * n);
        const int pos0 = c.len[s * c.H + h / c.G] - n;
        // local list: query indices ascending; full list (from the back): descending
        for (int k = 0; k < ntl; ++k) {
            const int cnt = min(kQRows, tot_l - k * kQRows);
            const int t_lo = pos0 + region[k * kQRows], t_hi = pos0 + region[k * kQRows + cnt - 1];
            tiles[first + k] = PfTile{sh, KVQ_MODE_LOCAL, off + k * kQRows, cnt, t_hi - max(0, t_lo - w) + 1, {0, 0, 0}};
        }
        for (int k = 0; k < ntf; ++k) {
            const int st = n - tot_f + k * kQRows;
            tiles[first + ntl + k] = PfTile{sh, KVQ_MODE_FULL, off + st, min(kQRows, tot_f - k * kQRows),
                                            pos0 + region[st] + 1, {0, 0, 0}};
        }
    }
}

// Longest tile first: one CTA orders the tile list by the keys each tile spans
// (descending, in buckets of 64 keys), so the long full-range tiles start in the first
// wave and the short ones fill in behind them.
constexpr int kSortBuckets = 1024;

__global__ void __launch_bounds__(1024)
prefill_order_kernel(const PfTile *__restrict__ in, const int32_t *__restrict__ tile_count, PfTile *__restrict__ out)
{
    __shared__ int hist[kSortBuckets];
    const int n = *tile_count, tid = threadIdx.x;
    for (int b = tid; b < kSortBuckets; b += blockDim.x) hist[b] = 0;
    __syncthreads();
    auto bucket = [](int nkeys) { return kSortBuckets - 1 - min(kSortBuckets - 1, (nkeys + 63) / 64); };
    for (int i = tid; i < n; i += blockDim.x) atomicAdd(&hist[bucket(in[i].nkeys)], 1);
    __syncthreads();
    if (tid < 32) {                              // exclusive prefix over the buckets, one warp
        int carry = 0;
        for (int b0 = 0; b0 < kSortBuckets; b0 += 32) {
            const int x = hist[b0 + tid];
            int incl = x;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, d);
                if (tid >= d) incl += y;
            }
            hist[b0 + tid] = carry + incl - x;
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
    }
    __syncthreads();
    for (int i = tid; i < n; i += blockDim.x) out[atomicAdd(&hist[bucket(in[i].nkeys)], 1)] = in[i];
}

template <int D>
cudaError_t run_tc(const kvq_cache *cache, const __half *q, const uint8_t *modes, int w, const int32_t *cu,
                   int64_t n_tok, float *out, cudaStream_t st)
{
    const CacheView &c = cache->view;
    PfTile *tiles = reinterpret_cast<PfTile *>(cache->pf_tiles);
    PfTile *ordered = tiles + cache->pf_max_tiles;
    cudaError_t e = cudaMemsetAsync(cache->pf_count, 0, sizeof(int32_t), st);
    if (e != cudaSuccess) return e;
    prefill_sched_kernel<<<c.B * c.H * c.G, kSchedThreads, 0, st>>>(c, modes, w, cu, n_tok, D, out, tiles,
                                                                    cache->pf_count, cache->pf_qidx);
    prefill_order_kernel<<<1, 1024, 0, st>>>(tiles, cache->pf_count, ordered);
    const int64_t max_tiles = n_tok * c.H * c.G / kQRows + 2LL * c.B * c.H * c.G;
    const size_t smem = sizeof(PfSmem<D>) + 1024;
    e = ensure_smem_attr((const void *)prefill_tc_kernel<D>, smem);
    if (e != cudaSuccess) return e;
    // the register split inside the kernel assumes the launch's count per thread
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, (const void *)prefill_tc_kernel<D>);
    if (e != cudaSuccess) return e;
    if (fa.numRegs != kLaunchRegs) return cudaErrorInvalidConfiguration;
    profile_before(st);
    prefill_tc_kernel<D><<<(unsigned)max_tiles, kTcThreads, smem, st>>>(c, q, w, cu, ordered, cache->pf_count,
                                                                        cache->pf_qidx, out);
    profile_after(st);
    return cudaGetLastError();
}

} // namespace

cudaError_t launch_prefill_tc(const kvq_cache *cache, const __half *q, const uint8_t *modes, int w,
                              const int32_t *cu, int64_t n_tok, float *out, cudaStream_t st)
{
    if (n_tok == 0) return cudaSuccess;
    if (cache->D == 128) return run_tc<128>(cache, q, modes, w, cu, n_tok, out, st);
    return run_tc<64>(cache, q, modes, w, cu, n_tok, out, st);
}

} // namespace kvq
