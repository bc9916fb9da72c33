// Routed decode attention (TriRoute paper review page, section 3, Eq. 2) over the
// mixed-precision cache of Eq. 4: one query per (sequence, query head) at t = len - 1.
//
// Three launches (programmatic dependent launch between them):
//   decode_plan_kernel    one CTA per sequence. Optionally first appends the step's tokens
//                         (Eq. 4 quantize-on-write, after an optional roll-back), so one
//                         decode step is three launches. Then the mode-aware schedule: skip
//                         queries get no work, local queries read keys [max(0, t - w), t],
//                         full queries [0, t]. A KV head's query group (grouped-query
//                         attention) is served in subgroups of up to 4 queries that share
//                         every record read: the key range is the union of the subgroup's
//                         ranges, cut where the local window starts, so within an item
//                         every active query reads every key. Ranges are cut into
//                         near-equal pieces of at most 1152 keys: the local window's pieces
//                         are back items, the other range's last piece a middle item and
//                         its other pieces, two at a time, front items. Each CTA reserves
//                         its items with one atomicAdd on each of the call's (generation,
//                         count) words of the three regions.
//   decode_splitk_kernel  three CTAs per SM, one producer and four consumer warps each. The
//                         producer claims items one at a time from the call's cursor, front
//                         items first, then middle, then back (a CTA that finishes early
//                         takes more; the short items come last and even out the CTAs' end
//                         times), and walks each in stages of at most 128 keys and 28 KB of
//                         records: a ring of record-offset windows is bulk-copied
//                         ahead, each stage's keys are sorted by width into chunks of one
//                         width (8 keys at head_dim 128), and the stage's contiguous record
//                         bytes, side entries and (for a new item) queries are bulk-copied
//                         into a 2-stage mbarrier pipeline. Consumer lanes: head_dim/32
//                         lanes per key, 32 channels per lane; K dot product on raw codes ->
//                         logit -> online softmax per key group (the running max moves only
//                         when a logit exceeds it by more than 8 in log2 units, a
//                         warp-uniform branch) -> V accumulation. Each warp serves one query
//                         of the item; at the item's end each warp deposits its state and
//                         the last warp to do so merges them into a partial per (item,
//                         query), while the others go on with the next item.
//   decode_combine_kernel log-sum-exp merge of the partials of each (sequence, query head),
//                         one thread per channel (decode_combine_warp_kernel, a warp per
//                         output, when there are at least 4 outputs per SM); zeros for skip
//                         heads and empty sequences.
//
// Arithmetic. With codes c, scale s and zero z (Eq. 4):
//   q . deq(k_j) = s_j * (q . c_j) + z_j * sum(q)         (one dot product on integer codes)
//   sum_j p_j deq(v_j) = sum_j (p_j s_j) c_j + (sum_j p_j z_j) * 1
// Codes are never converted with an int->float instruction: a b-bit field masked in place
// inside a 32-bit word (bits below 23) IS the fp32 subnormal c * 2^(pos - 149), and FFMA
// multiplies subnormal operands exactly at full rate. For K the products at each bit
// position accumulate separately and the position scales 2^-pos are applied once per key;
// for V the softmax weight is scaled by 2^-pos once per position. Channels c and c + 16 of
// a lane travel as one float2, so the FMAs are packed FFMA2 instructions (two fp32 FMAs,
// each rounded as fmaf, subnormal operands kept). fp32 subnormals must not be flushed:
// build without -ftz / fast-math.
#include <atomic>
#include <cstdio>
#include <mutex>

#include <nvtx3/nvToolsExt.h>

#include "kvq_quant.cuh"

namespace kvq {
namespace {

// Launch shape of the split-K kernel (build-time tunables; the defaults are the measured
// best on B200).
#ifndef KVQ_DECODE_CONSUMERS
#define KVQ_DECODE_CONSUMERS 4
#endif
#ifndef KVQ_DECODE_CTAS_PER_SM
#define KVQ_DECODE_CTAS_PER_SM 3
#endif
#ifndef KVQ_DECODE_STAGES
#define KVQ_DECODE_STAGES 2
#endif
#ifndef KVQ_DECODE_STAGE_BYTES
#define KVQ_DECODE_STAGE_BYTES 28672
#endif
#ifndef KVQ_DECODE_META_SLOTS
#define KVQ_DECODE_META_SLOTS 4
#endif
constexpr int kConsumerWarps = KVQ_DECODE_CONSUMERS;
constexpr int kThreads = 32 * (kConsumerWarps + 1);
constexpr int kCtasPerSm = KVQ_DECODE_CTAS_PER_SM;
constexpr int kStages = KVQ_DECODE_STAGES;        // record stages in flight per CTA
#ifndef KVQ_DECODE_WINDOW
#define KVQ_DECODE_WINDOW 128
#endif
constexpr int kWin = KVQ_DECODE_WINDOW;           // keys per window of record offsets
constexpr int KPL = kWin / 32;                    // window slots per producer lane
static_assert(kWin == 128, "windows of 128 keys: the width sort packs positions below 256 in bytes");
constexpr uint32_t kStageRecBytes = KVQ_DECODE_STAGE_BYTES;   // record bytes per stage, at most
constexpr int kPermSlots = kWin + 64;             // width-sorted keys padded to whole chunks
constexpr int kMetaSlots = KVQ_DECODE_META_SLOTS; // windows of record offsets fetched ahead
static_assert(kStageRecBytes <= 32768, "stage offsets are 15 bits");
constexpr int kMetaWords = kWin + 8;
// A consumer warp can run at most kStages items ahead of the slowest one (the stages are
// shared and every item has at least one), so kStages + 1 merge slots never collide.
constexpr int kMergeRing = kStages + 1;
constexpr int kNewItem = 1, kLastSub = 2, kStop = 4;   // stage flags (kStop: no more items)
constexpr uint32_t kReadEndFromMeta = 0xFFFFFFFFu;
// DecodeItem.role of a front item: kPairHead, the next list entry is the following piece of
// the same range; kPairTail, the entry before it is its head; kSolo, neither
constexpr int kSolo = 0, kPairHead = 1, kPairTail = 2;
// A call whose list has at least this many items per split-K CTA walks each pair of front
// items as one item (fewer item starts and merges); a shorter list keeps the finer items
#ifndef KVQ_DECODE_PAIR_ITEMS_PER_CTA
#define KVQ_DECODE_PAIR_ITEMS_PER_CTA 6
#endif
constexpr uint32_t kValid = 0x80000000u;
constexpr float kLazy = 8.f;                      // running-max slack, log2 units
constexpr float kMInit = -1e30f;                  // running max before the first key
constexpr int kPlanThreads = 256;

// q' = q * 2^60. A code field at bit position pos is c * 2^(pos - 149), so q' * field =
// q * c * 2^(pos - 89): per-position sums are unscaled by 2^(89 - pos). Native fp16 values
// give q * x * 2^60.
constexpr float kQScale = 1152921504606846976.0f;                   // 2^60
constexpr float kDotCodeUnscale = 618970019642690137449562112.0f;   // 2^89
constexpr float kDotNativeUnscale = 8.673617379884035e-19f;         // 2^-60
// V weights: w' = p * s * 2^(100 - pos); accumulators hold o * 2^-49.
constexpr float kWScale = 1267650600228229401496703205376.0f;       // 2^100
constexpr float kONativeScale = 1.7763568394002505e-15f;            // 2^-49
constexpr float kOUnscale = 562949953421312.0f;                     // 2^49

template <int D>
struct Geo {
    static constexpr int LPK = D / 32;             // lanes per key, 32 channels per lane
    static constexpr int KPS = 32 / LPK;           // keys per warp step (chunk)
};

struct AppendArgs {
    const __half *k, *v;
    const uint8_t *bits;
    const int32_t *cu, *positions;
    int64_t n_tok;
    uint32_t gen;
};

template <int D>
struct Stage {
    // width-sorted keys in chunks of one width: kValid | (key << 16) | offset in rec;
    // padding entries are a key of the same width without kValid
    uint32_t perm[kPermSlots];
    int32_t info[8];         // item index, keys in the stage, flags, chunks, qinfo
    int32_t cls_chunk[8];    // first chunk of each width class (b = 2, 4, 8, 16), [4] = chunks
    __half q[kDecodeMaxQ][D];  // the item's queries (copied with the item's first stage)
    float4 side[kWin];       // (s_K, z_K, s_V, z_V) per key, token order
    alignas(16) uint8_t rec[kStageRecBytes];
};

// one window of record offsets: meta of keys [ja, ...) of an item's stream
struct alignas(16) MetaSlot {
    uint32_t meta[kMetaWords];
    int32_t it, j, j1, ja;
    uint32_t end_off, first;
    int64_t sbase;
    int32_t sh, qinfo;
};

template <int D>
struct DecodeSmem {
    Stage<D> st[kStages];
    MetaSlot ms[kMetaSlots];
    // item merges: a ring of kMergeRing items (states deposited by each consumer warp)
    float red_o[kMergeRing][kConsumerWarps][D];
    float red_m[kMergeRing][kConsumerWarps], red_l[kMergeRing][kConsumerWarps], red_pz[kMergeRing][kConsumerWarps];
    int32_t merge_cnt[kMergeRing];
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t mfull[kMetaSlots];
    int32_t abort_flag;
};

__device__ __forceinline__ float fld(uint32_t bits) { return __uint_as_float(bits); }
__device__ __forceinline__ float2 fpair(uint32_t a, uint32_t b) { return make_float2(fld(a), fld(b)); }
__device__ __forceinline__ float2 bcast(float a) { return make_float2(a, a); }

// 2^x with the hardware's approximate exp2 (relative error of a few ulp; 2^-inf = 0,
// results below 2^-126 flush to 0): the softmax weights.
__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float h2f_lo(uint32_t w) { return __half2float(__ushort_as_half((unsigned short)(w & 0xFFFFu))); }
__device__ __forceinline__ float h2f_hi(uint32_t w) { return __half2float(__ushort_as_half((unsigned short)(w >> 16))); }

// ------------------------------------------------------------------ planning
// Appends the step's tokens of sequence blockIdx.x (APPEND), then lists the decode items of
// its (KV head, subgroup) units. A unit's key range outside the local window (all of it
// when no query of the subgroup is local) is cut into c near-equal pieces of at most
// kDecodeItemKeys keys; pieces 0 .. c - 2 are front items (consecutive in the list, marked
// as pairs (0, 1), (2, 3), ...), piece c - 1 a middle item; the window's pieces are back
// items. The split-K CTAs claim front, then middle, then back items, so the long items
// start first and the short ones even out the end of the launch. Which keys an item
// covers, and which items pair up, depend on the unit alone (not on the order in which
// the CTAs reserve), so the results do not depend on timing.
template <int D, bool APPEND>
__global__ void __launch_bounds__(kPlanThreads)
decode_plan_kernel(CacheView c, const uint8_t *__restrict__ modes, int w, DecodeWork wk, uint32_t gen,
                   AppendArgs ap)
{
    __shared__ AppendShared as;
    // counts packed as front items | back items << 32 (a pass lists fewer than 2^31 of
    // each), middle items apart
    __shared__ long long warp_tot[kPlanThreads / 32];
    __shared__ int warp_totm[kPlanThreads / 32];
    __shared__ long long cnt_sh[kPlanThreads];
    __shared__ int cntm_sh[kPlanThreads];
    __shared__ uint32_t base_sh[3];
    // per unit of the pass: first front, back and middle item (relative to the pass), keys
    // outside and inside the window, query masks and subgroup, length, stream end, first slot
    __shared__ int u_startF[kPlanThreads + 1], u_startB[kPlanThreads + 1], u_startM[kPlanThreads + 1];
    __shared__ int u_nF[kPlanThreads], u_nW[kPlanThreads], u_q[kPlanThreads], u_L[kPlanThreads];
    __shared__ uint32_t u_end[kPlanThreads];
    __shared__ int64_t u_sbase[kPlanThreads];
    pdl_wait();
    pdl_trigger();
    // the previous call's kernels have completed: its count words become the next call's
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        *wk.count_next = (unsigned long long)(gen + 1u) << 32;
        *wk.count_back_next = (unsigned long long)(gen + 1u) << 32;
        *wk.count_mid_next = (unsigned long long)(gen + 1u) << 32;
        *wk.cursor = 0u;                 // the split-K CTAs claim this call's items from 0
    }
    const int s = blockIdx.x;
    if (APPEND) append_seq<D>(c, ap.k, ap.v, ap.bits, ap.cu, ap.n_tok, ap.gen, ap.positions, s, as);
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int H = c.H, G = c.G, HQ = H * G;
    const int BH = c.B * H;
    const int nsub = (G + kDecodeMaxQ - 1) / kDecodeMaxQ;
    const int units = H * nsub;
    const int per_pass = (kPlanThreads / nsub) * nsub;      // whole KV heads per pass
    constexpr int K = kDecodeItemKeys;
    for (int u0 = 0; u0 < units; u0 += per_pass) {
        const int u = u0 + tid;
        const bool mine = tid < per_pass && u < units;
        int L = 0, nF = 0, nW = 0, mF = 0, mW = 0, g0 = 0, hk = 0;
        if (mine) {
            hk = u / nsub;
            g0 = (u % nsub) * kDecodeMaxQ;
            L = (APPEND && hk < kAppendHeads) ? as.len[hk] : c.len[s * H + hk];
            const int lo_loc = max(0, L - 1 - w);
            int full = 0, local = 0;
            for (int i = 0; i < kDecodeMaxQ && g0 + i < G; ++i) {
                const int m = modes[(int64_t)s * HQ + hk * G + g0 + i];
                if (m > KVQ_MODE_FULL) set_status(c.status, KVQ_ERR_MODE);
                else if (m == KVQ_MODE_FULL) full |= 1 << i;
                else if (m == KVQ_MODE_LOCAL) local |= 1 << i;
            }
            if (L > 0) {
                if (local) {                         // window [lo_loc, L): every active query;
                    mW = full | local;               // keys before it: the full ones alone
                    nW = L - lo_loc;
                    mF = full;
                    nF = full ? lo_loc : 0;
                } else if (full) {                   // one range [0, L)
                    mF = full;
                    nF = L;
                }
            }
        }
        const int pieces = (nF + K - 1) / K;
        const int cF = max(pieces - 1, 0), cM = pieces > 0 ? 1 : 0, cB = (nW + K - 1) / K;
        const long long cnt = (long long)cF | ((long long)cB << 32);
        cnt_sh[tid] = cnt;
        cntm_sh[tid] = cM;
        long long incl = cnt;
        int inclm = cM;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const long long y = __shfl_up_sync(0xffffffffu, incl, d);
            const int ym = __shfl_up_sync(0xffffffffu, inclm, d);
            if (lane >= d) {
                incl += y;
                inclm += ym;
            }
        }
        if (lane == 31) {
            warp_tot[wid] = incl;
            warp_totm[wid] = inclm;
        }
        __syncthreads();
        long long wpre = 0, tot = 0;
        int wprem = 0, totM = 0;
#pragma unroll
        for (int qq = 0; qq < kPlanThreads / 32; ++qq) {
            const long long t = warp_tot[qq];
            const int tm = warp_totm[qq];
            if (qq < wid) {
                wpre += t;
                wprem += tm;
            }
            tot += t;
            totM += tm;
        }
        const int totF = (int)(tot & 0xFFFFFFFFll), totB = (int)(tot >> 32);
        if (tid == 0) {
            // reserve [base, base + tot) of this call's front, back and middle regions (one
            // atomic each, no retries)
            const unsigned long long oF = atomicAdd(wk.count, (unsigned long long)totF);
            const unsigned long long oB = atomicAdd(wk.count_back, (unsigned long long)totB);
            const unsigned long long oM = atomicAdd(wk.count_mid, (unsigned long long)totM);
            const uint32_t tagF = (uint32_t)(oF >> 32), tagB = (uint32_t)(oB >> 32), tagM = (uint32_t)(oM >> 32);
            if ((tagF != gen && tagF != 0u) || (tagB != gen && tagB != 0u) || (tagM != gen && tagM != 0u)) {
                set_status(c.status, KVQ_ERR_DEVICE_CHECK);     // stale: list nothing
                base_sh[0] = 0xFFFFFFFFu;
            } else {
                base_sh[0] = (uint32_t)oF;
                base_sh[1] = (uint32_t)oB;
                base_sh[2] = (uint32_t)oM;
            }
            u_startF[kPlanThreads] = totF;
            u_startB[kPlanThreads] = totB;
            u_startM[kPlanThreads] = totM;
        }
        const long long rel = wpre + incl - cnt;      // the unit's first items within the pass
        const int relM = wprem + inclm - cM;
        u_startF[tid] = (int)(rel & 0xFFFFFFFFll);
        u_startB[tid] = (int)(rel >> 32);
        u_startM[tid] = relM;
        u_nF[tid] = nF;
        u_nW[tid] = nW;
        u_q[tid] = g0 | (mF << 8) | (mW << 12);
        u_L[tid] = L;
        if (mine && (pieces + cB) > 0) {
            u_end[tid] = (APPEND && hk < kAppendHeads) ? as.end[hk] : c.end[s * H + hk];
            u_sbase[tid] = slot_of(c, s, hk, 0);
        }
        __syncthreads();
        const bool stale = base_sh[0] == 0xFFFFFFFFu;
        const int64_t baseF = stale ? 0 : base_sh[0], baseB = stale ? 0 : base_sh[1], baseM = stale ? 0 : base_sh[2];
        const bool over = !stale && (baseF + totF > wk.mid_base || baseB + totB > wk.mid_base ||
                                     baseM + totM > wk.max_items - wk.mid_base);
        if (mine && u % nsub == 0) {                  // the KV head's items: its subgroups' runs
            int nFi = 0, nBi = 0, nMi = 0;
            for (int k = 0; k < nsub; ++k) {
                nFi += (int)(cnt_sh[tid + k] & 0xFFFFFFFFll);
                nBi += (int)(cnt_sh[tid + k] >> 32);
                nMi += cntm_sh[tid + k];
            }
            const int unit = s * H + hk;
            const bool none = stale || over;
            wk.head_first[unit] = (int32_t)(baseF + (rel & 0xFFFFFFFFll));
            wk.head_cnt[unit] = none ? 0 : nFi;
            // back items x .. x + nBi - 1 sit at mid_base - 1 - x down to mid_base - x - nBi
            wk.head_first[BH + unit] = (int32_t)(wk.mid_base - (baseB + (rel >> 32) + nBi));
            wk.head_cnt[BH + unit] = none ? 0 : nBi;
            wk.head_first[2 * BH + unit] = (int32_t)(wk.mid_base + baseM + relM);
            wk.head_cnt[2 * BH + unit] = none ? 0 : nMi;
        }
        if (stale) {
        } else if (over) {
            if (tid == 0) set_status(c.status, KVQ_ERR_DEVICE_CHECK);
        } else {
            // every thread writes items: item i of a region's pass belongs to the last unit
            // whose first item in that region is <= i (binary search over the pass's units)
            const int n_units = min(per_pass, units - u0);
            for (int t = tid; t < totF + totM + totB; t += kPlanThreads) {
                const int reg = (t < totF) ? 0 : (t < totF + totM) ? 1 : 2;   // front, middle, back
                const int i = (reg == 0) ? t : (reg == 1) ? t - totF : t - totF - totM;
                const int *ust = (reg == 0) ? u_startF : (reg == 1) ? u_startM : u_startB;
                int lo = 0, hi = n_units;                  // ust[lo] <= i < ust[hi]
                while (hi - lo > 1) {
                    const int mid = (lo + hi) >> 1;
                    if (ust[mid] <= i) lo = mid;
                    else hi = mid;
                }
                while (lo + 1 < n_units && ust[lo + 1] <= i) ++lo;   // skip units with no items
                const int k = i - ust[lo];
                const int Lu = u_L[lo], qv = u_q[lo];
                int j0, j1, mask, role = kSolo;
                if (reg < 2) {                             // pieces of [0, nF)
                    const int n = u_nF[lo], pc = (n + K - 1) / K;
                    const int per = n / pc, rem = n % pc;  // near-equal, non-empty pieces
                    const int pa = (reg == 0) ? k : pc - 1;
                    j0 = pa * per + min(pa, rem);
                    j1 = (pa + 1) * per + min(pa + 1, rem);
                    mask = (qv >> 8) & 0xF;
                    if (reg == 0) role = (k & 1) ? kPairTail : (k + 1 <= pc - 2) ? kPairHead : kSolo;
                } else {                                   // pieces of the window [Lu - nW, Lu)
                    const int n = u_nW[lo], pc = (n + K - 1) / K;
                    const int per = n / pc, rem = n % pc;
                    j0 = Lu - n + k * per + min(k, rem);
                    j1 = j0 + per + (k < rem ? 1 : 0);
                    mask = (qv >> 12) & 0xF;
                }
                DecodeItem d;
                d.sh = s * H + (u0 + lo) / nsub;
                d.j0 = j0;
                d.j1 = j1;
                // the stream end for the item ending at the last token; else the producer
                // reads the offset of key j1 itself
                d.end_off = (j1 < Lu) ? kReadEndFromMeta : u_end[lo];
                d.sbase = u_sbase[lo];
                d.qinfo = (qv & 0xFF) | (mask << 8);
                d.role = role;
                const int64_t ix = (reg == 0) ? baseF + i : (reg == 1) ? wk.mid_base + baseM + i
                                                                       : wk.mid_base - 1 - (baseB + i);
                wk.items[ix] = d;
            }
        }
        __syncthreads();                             // the per-unit arrays are reused by the next pass
    }
}

// ------------------------------------------------------------------ per-width lane math
// A lane holds 32 channels (c0 .. c0 + 31) of one key; its share of a record part is 4*b
// bytes starting at byte 4*b*li. Pairs (k, k + 16) of the lane's channels share a float2.
struct QRegs {
    float2 q[16];            // (q[k], q[k + 16]) * 2^60
};

// Lane partial of q . c (scaled as described above), by width class.
template <int CLS>
__device__ __forceinline__ float lane_dot(const QRegs &Q, const uint8_t *p)
{
    if (CLS == 0) {                                   // 2-bit: 2 words, 8 positions per half
        const uint2 x = *reinterpret_cast<const uint2 *>(p);
        const uint32_t y0 = x.x >> 16, y1 = x.y >> 16;
        float2 a[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const uint32_t m = 3u << (2 * j);
            a[j] = __fmul2_rn(Q.q[j], fpair(x.x & m, x.y & m));
            a[j] = __ffma2_rn(Q.q[8 + j], fpair(y0 & m, y1 & m), a[j]);
        }
        float r = a[7].x + a[7].y;
#pragma unroll
        for (int j = 6; j >= 0; --j) r = fmaf(r, 0.25f, a[j].x + a[j].y);   // sum_j 2^(-2j) a_j
        return r;
    } else if (CLS == 1) {                            // 4-bit: 4 words, 4 positions per half
        const uint4 x = *reinterpret_cast<const uint4 *>(p);
        const uint32_t h0 = x.x >> 16, h1 = x.y >> 16, h2 = x.z >> 16, h3 = x.w >> 16;
        float2 a[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t m = 15u << (4 * j);
            a[j] = __fmul2_rn(Q.q[j], fpair(x.x & m, x.z & m));
            a[j] = __ffma2_rn(Q.q[4 + j], fpair(h0 & m, h2 & m), a[j]);
            a[j] = __ffma2_rn(Q.q[8 + j], fpair(x.y & m, x.w & m), a[j]);
            a[j] = __ffma2_rn(Q.q[12 + j], fpair(h1 & m, h3 & m), a[j]);
        }
        float r = a[3].x + a[3].y;
#pragma unroll
        for (int j = 2; j >= 0; --j) r = fmaf(r, 0.0625f, a[j].x + a[j].y);
        return r;
    } else if (CLS == 2) {                            // 8-bit: 8 words, bytes moved to position 0
        const uint4 x0 = reinterpret_cast<const uint4 *>(p)[0];
        const uint4 x1 = reinterpret_cast<const uint4 *>(p)[1];
        const uint32_t wv[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
        float2 a[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
        for (int i = 0; i < 4; ++i) {                 // word i: channels 4i..4i+3; word i+4: +16
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const uint32_t sel = 0x4440 + e;
                a[e & 1] = __ffma2_rn(Q.q[4 * i + e], fpair(__byte_perm(wv[i], 0u, sel), __byte_perm(wv[i + 4], 0u, sel)),
                                      a[e & 1]);
            }
        }
        return (a[0].x + a[1].x) + (a[0].y + a[1].y);
    } else {                                          // 16-bit: 16 words of fp16 pairs
        uint32_t wv[16];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint4 x = reinterpret_cast<const uint4 *>(p)[i];
            wv[4 * i] = x.x;
            wv[4 * i + 1] = x.y;
            wv[4 * i + 2] = x.z;
            wv[4 * i + 3] = x.w;
        }
        float2 a[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
        for (int i = 0; i < 8; ++i) {                 // word i: channels 2i, 2i+1; word i+8: +16
            a[0] = __ffma2_rn(Q.q[2 * i], make_float2(h2f_lo(wv[i]), h2f_lo(wv[i + 8])), a[0]);
            a[1] = __ffma2_rn(Q.q[2 * i + 1], make_float2(h2f_hi(wv[i]), h2f_hi(wv[i + 8])), a[1]);
        }
        return (a[0].x + a[1].x) + (a[0].y + a[1].y);
    }
}

// o[k] += weight * (c_k, c_{k+16}) for the lane's 32 V values of width class CLS.
template <int CLS>
__device__ __forceinline__ void lane_acc(float2 (&o)[16], float wv, const uint8_t *p)
{
    if (CLS == 0) {
        const uint2 x = *reinterpret_cast<const uint2 *>(p);
        const uint32_t y0 = x.x >> 16, y1 = x.y >> 16;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float2 wj = bcast(wv * __uint_as_float((127u - 2u * j) << 23));   // wv * 2^-2j
            const uint32_t m = 3u << (2 * j);
            o[j] = __ffma2_rn(wj, fpair(x.x & m, x.y & m), o[j]);
            o[8 + j] = __ffma2_rn(wj, fpair(y0 & m, y1 & m), o[8 + j]);
        }
    } else if (CLS == 1) {
        const uint4 x = *reinterpret_cast<const uint4 *>(p);
        const uint32_t h0 = x.x >> 16, h1 = x.y >> 16, h2 = x.z >> 16, h3 = x.w >> 16;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 wj = bcast(wv * __uint_as_float((127u - 4u * j) << 23));   // wv * 2^-4j
            const uint32_t m = 15u << (4 * j);
            o[j] = __ffma2_rn(wj, fpair(x.x & m, x.z & m), o[j]);
            o[4 + j] = __ffma2_rn(wj, fpair(h0 & m, h2 & m), o[4 + j]);
            o[8 + j] = __ffma2_rn(wj, fpair(x.y & m, x.w & m), o[8 + j]);
            o[12 + j] = __ffma2_rn(wj, fpair(h1 & m, h3 & m), o[12 + j]);
        }
    } else if (CLS == 2) {
        const uint4 x0 = reinterpret_cast<const uint4 *>(p)[0];
        const uint4 x1 = reinterpret_cast<const uint4 *>(p)[1];
        const uint32_t wd[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
        const float2 w2 = bcast(wv);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const uint32_t sel = 0x4440 + e;
                o[4 * i + e] = __ffma2_rn(w2, fpair(__byte_perm(wd[i], 0u, sel), __byte_perm(wd[i + 4], 0u, sel)),
                                          o[4 * i + e]);
            }
        }
    } else {
        uint32_t wd[16];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint4 x = reinterpret_cast<const uint4 *>(p)[i];
            wd[4 * i] = x.x;
            wd[4 * i + 1] = x.y;
            wd[4 * i + 2] = x.z;
            wd[4 * i + 3] = x.w;
        }
        const float2 w2 = bcast(wv);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            o[2 * i] = __ffma2_rn(w2, make_float2(h2f_lo(wd[i]), h2f_lo(wd[i + 8])), o[2 * i]);
            o[2 * i + 1] = __ffma2_rn(w2, make_float2(h2f_hi(wd[i]), h2f_hi(wd[i + 8])), o[2 * i + 1]);
        }
    }
}

struct KeyState {
    float m, l, pz;
    float2 o[16];      // (o[c0 + k], o[c0 + k + 16]) of the lane's 32 channels
};

// merge the online-softmax state of this lane with the lane `mask` away
__device__ __forceinline__ void merge_state(KeyState &st, int mask)
{
    const float mp = __shfl_xor_sync(0xffffffffu, st.m, mask);
    const float lp = __shfl_xor_sync(0xffffffffu, st.l, mask);
    const float zp = __shfl_xor_sync(0xffffffffu, st.pz, mask);
    const float M = fmaxf(st.m, mp);
    const float fa = ex2(st.m - M), fb = ex2(mp - M);
#pragma unroll
    for (int k = 0; k < 16; ++k) {
        const float2 op = make_float2(__shfl_xor_sync(0xffffffffu, st.o[k].x, mask),
                                      __shfl_xor_sync(0xffffffffu, st.o[k].y, mask));
        st.o[k] = __ffma2_rn(op, bcast(fb), __fmul2_rn(st.o[k], bcast(fa)));
    }
    st.l = st.l * fa + lp * fb;
    st.pz = st.pz * fa + zp * fb;
    st.m = M;
}

// One chunk: a key per LPK-lane group, all of width class CLS (warp-uniform): K dot product
// on the codes, logit, online-softmax update of the group's state, V accumulation.
// Padding entries (no valid bit) read a real record of the same width and get weight 0.
template <int D, int CLS>
__device__ __forceinline__ void process_chunk(KeyState &st, const QRegs &Q, float qsum_l, float cdot,
                                              const Stage<D> &sg, uint32_t ent, int li)
{
    constexpr int LPK = Geo<D>::LPK;
    constexpr int BITS = 2 << CLS;
    const uint8_t *r = sg.rec + (ent & 0x7FFFu);
    float part = lane_dot<CLS>(Q, r + 4 * BITS * li);
#pragma unroll
    for (int d = 1; d < LPK; d <<= 1) part += __shfl_xor_sync(0xffffffffu, part, d);
    const float4 sd = sg.side[(ent >> 16) & 0xFFu];
    float lg = (CLS == 3) ? part * cdot : fmaf(sd.x * cdot, part, sd.y * qsum_l);
    lg = (ent & kValid) ? lg : -INFINITY;
    if (__any_sync(0xffffffffu, lg > st.m + kLazy)) {      // rare after an item's first keys
        const float m_new = (lg > st.m + kLazy) ? lg : st.m;
        const float corr = ex2(st.m - m_new);
        st.l *= corr;
        st.pz *= corr;
#pragma unroll
        for (int k = 0; k < 16; ++k) st.o[k] = __fmul2_rn(st.o[k], bcast(corr));
        st.m = m_new;
    }
    const float p = ex2(lg - st.m);
    st.l += p;
    const uint8_t *rv = r + (D * BITS) / 8 + 4 * BITS * li;
    if (CLS == 3) {
        lane_acc<3>(st.o, p * kONativeScale, rv);
    } else {
        st.pz = fmaf(p, sd.w, st.pz);
        lane_acc<CLS>(st.o, p * (sd.z * kWScale), rv);
    }
}

// This warp's chunks ch, ch + step, ... below `end`, all of width class CLS.
template <int D, int CLS>
__device__ __forceinline__ int run_class(KeyState &st, const QRegs &Q, float qsum_l, float cdot,
                                         const Stage<D> &sg, int ch, int end, int step, int g, int li)
{
    constexpr int KPS = Geo<D>::KPS;
    for (; ch < end; ch += step) process_chunk<D, CLS>(st, Q, qsum_l, cdot, sg, sg.perm[KPS * ch + g], li);
    return ch;
}

template <int D>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
decode_splitk_kernel(CacheView c, const __half *__restrict__ q, DecodeWork wk)
{
    constexpr int LPK = Geo<D>::LPK;
    constexpr int KPS = Geo<D>::KPS;

    extern __shared__ __align__(128) uint8_t smem_raw[];
    DecodeSmem<D> &sm = *reinterpret_cast<DecodeSmem<D> *>(smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    pdl_wait();
    pdl_trigger();
    // claims 0 .. n_front - 1 are the front items, then come the middle items, then the back
    // items from the end of the front/back zone down
    int n_front = 0, n_fm = 0, n_items = 0;
    {
        const unsigned long long cf = *wk.count, cb = *wk.count_back, cm = *wk.count_mid;
        const uint32_t tagF = (uint32_t)(cf >> 32), tagB = (uint32_t)(cb >> 32), tagM = (uint32_t)(cm >> 32);
        if ((tagF == wk.gen || tagF == 0u) && (tagB == wk.gen || tagB == 0u) && (tagM == wk.gen || tagM == 0u)) {
            const int64_t nf = (uint32_t)cf, nb = (uint32_t)cb, nm = (uint32_t)cm;
            if (nf + nb <= wk.mid_base && nm <= wk.max_items - wk.mid_base) {
                n_front = (int)nf;
                n_fm = (int)(nf + nm);
                n_items = (int)(nf + nm + nb);
            } else if (blockIdx.x == 0 && tid == 0) {
                set_status(c.status, KVQ_ERR_DEVICE_CHECK);
            }
        }
    }

    if (tid == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&sm.full[i], 1);
            mbar_init(&sm.empty[i], kConsumerWarps);
        }
        for (int i = 0; i < kMetaSlots; ++i) mbar_init(&sm.mfull[i], 1);
        for (int i = 0; i < kMergeRing; ++i) sm.merge_cnt[i] = 0;
        sm.abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == kConsumerWarps) {
        // ------------------------------ producer ---------------------------------
        // A filler cursor runs up to kMetaSlots windows ahead and bulk-copies each window of
        // 128 record offsets into a shared ring; the record cursor reads a window from shared
        // memory, cuts it into stages of at most kStageRecBytes, sorts each stage's keys by
        // width and issues the stage's copies. On a timed-out wait it stops issuing, waits
        // (bounded) for the copies already in flight and returns.
        // A window's record offsets sit in slots 0..kWin+3 of its ring entry, key ja + i in
        // slot i (ja = the window's first key rounded down to a multiple of 4); lane l holds
        // slots KPL*l .. KPL*l + KPL - 1 (16-byte shared loads). Windows after an item's first
        // end on 4-aligned keys, so a window's keys fit slots [d, d + nwin) with
        // d + nwin <= kWin. Items are claimed when the filler reaches them (CTAs that finish
        // early take more); after the last one the producer marks a stage kStop.
        // (Claiming the next item one item ahead, to hide the claim's latency, lengthened the
        // tail more than it saved.)
        // With a long list (a decision from the item count alone, the same in every CTA) a
        // pair head's claimer walks both pieces as one item and marks the tail's partials
        // empty (l = 0) for the combine; a claimed tail is then skipped.
        const bool pairs = n_items >= KVQ_DECODE_PAIR_ITEMS_PER_CTA * (int)gridDim.x;
        auto claim = [&](DecodeItem &d) {        // the next item's index (d: its range), or -1
            for (;;) {
                int v = 0;
                if (lane == 0) v = (int)atomicAdd(wk.cursor, 1u);
                v = __shfl_sync(0xffffffffu, v, 0);
                if (v >= n_items) return -1;
                const int it = v < n_front ? v
                             : v < n_fm    ? (int)wk.mid_base + (v - n_front)
                                           : (int)wk.mid_base - 1 - (v - n_fm);
                d = wk.items[it];
                if (!pairs || v >= n_front || d.role == kSolo) return it;
                if (d.role == kPairTail) continue;
                const DecodeItem d2 = wk.items[it + 1];     // the head's tail (a front item)
                d.j1 = d2.j1;
                d.end_off = d2.end_off;
                const int slot_q = lane;                  // lanes 0..3: the query slots
                if (slot_q < wk.qslots && ((d2.qinfo >> (8 + slot_q)) & 1))
                    wk.partials[((int64_t)(it + 1) * wk.qslots + slot_q) * (D + 4) + 1] = 0.f;
                return it;
            }
        };
        DecodeItem f_d = wk.items[0];
        int f_it = claim(f_d);
        bool f_valid = f_it >= 0, aborted = false;
        int f_j = f_d.j0;
        int filled = 0, consumed = 0, issued = 0;
        auto pick = [](const uint32_t (&a)[KPL], int i) {       // a[i], i warp-uniform
            uint32_t v = a[0];
#pragma unroll
            for (int r = 1; r < KPL; ++r) v = (i == r) ? a[r] : v;
            return v;
        };
        while (!aborted) {
            while (f_valid && filled < consumed + kMetaSlots) {
                const int slot = filled % kMetaSlots;
                MetaSlot &ms = sm.ms[slot];
                const int ja = f_j & ~3;
                const int nwin = min(kWin - (f_j - ja), f_d.j1 - f_j);
                const int jb = (f_j + nwin + 1 + 3) & ~3;    // includes the key after the window
                if (lane == 0) {
                    ms.it = f_it;
                    ms.j = f_j;
                    ms.j1 = f_j + nwin;
                    ms.ja = ja;
                    ms.end_off = (f_j + nwin == f_d.j1) ? f_d.end_off : kReadEndFromMeta;
                    ms.first = (f_j == f_d.j0) | ((f_j + nwin == f_d.j1) ? 2 : 0);
                    ms.sbase = f_d.sbase;
                    ms.sh = f_d.sh;
                    ms.qinfo = f_d.qinfo;
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    mbar_arrive_expect_tx(&sm.mfull[slot], 4u * (uint32_t)(jb - ja));
                    bulk_g2s(ms.meta, c.meta + f_d.sbase + ja, 4u * (uint32_t)(jb - ja), &sm.mfull[slot]);
                }
                ++filled;
                f_j += nwin;
                if (f_j >= f_d.j1) {
                    f_it = claim(f_d);
                    if (f_it >= 0) {
                        f_j = f_d.j0;
                    } else {
                        f_valid = false;
                    }
                }
            }
            if (consumed == filled) break;
            const int slot = consumed % kMetaSlots;
            if (!mbar_wait(&sm.mfull[slot], (uint32_t)(consumed / kMetaSlots) & 1u, c.status)) {
                aborted = true;
                break;
            }
            const MetaSlot &ms = sm.ms[slot];
            const int it = ms.it, qinfo = ms.qinfo, ja = ms.ja;
            const int d = ms.j - ja, dend = ms.j1 - ja;       // the window's keys: slots [d, dend)
            const bool first = (ms.first & 1) != 0, lastwin = (ms.first & 2) != 0;
            uint32_t m[KPL];
#pragma unroll
            for (int v4 = 0; v4 < KPL / 4; ++v4) {
                const uint4 mv = reinterpret_cast<const uint4 *>(ms.meta)[KPL / 4 * lane + v4];
                m[4 * v4] = mv.x;
                m[4 * v4 + 1] = mv.y;
                m[4 * v4 + 2] = mv.z;
                m[4 * v4 + 3] = mv.w;
            }
            const uint32_t bnd = (ms.end_off == kReadEndFromMeta ? ms.meta[dend] : ms.end_off) & ~15u;
            const int64_t sbase = ms.sbase;
            const int sh = ms.sh;
            // nx[r]: the offset right after the key in slot KPL lane + r (the next key's
            // offset, or the bound after the window's last key)
            uint32_t nx[KPL];
            const uint32_t next_lane = __shfl_down_sync(0xffffffffu, m[0], 1);
#pragma unroll
            for (int r = 0; r < KPL; ++r) {
                const int sl = KPL * lane + r;
                nx[r] = (sl + 1 == dend) ? bnd : ((r + 1 < KPL ? m[(r + 1) % KPL] : next_lane) & ~15u);
            }
            ++consumed;

            for (int s0 = d; s0 < dend;) {
                // the stage: slots [s0, s1), at most kStageRecBytes of records, at most 255
                // keys, and (paged caches) bytes in at most two pages
                const uint32_t off0 = __shfl_sync(0xffffffffu, pick(m, s0 % KPL), s0 / KPL) & ~15u;
                const uint32_t plast = (off0 >> c.page_shift) + 1u;
                int n;
                uint32_t nxl;
                if (dend - s0 <= 255 && bnd - off0 <= kStageRecBytes && bnd >= off0 &&
                    ((bnd - 1u) >> c.page_shift) <= plast) {
                    n = dend - s0;    // the rest of the window is one stage (the common case)
                    nxl = bnd;
                } else {
                    uint32_t cnt = 0;
#pragma unroll
                    for (int r = 0; r < KPL; ++r) {
                        const int sl = KPL * lane + r;
                        cnt += (sl >= s0 && sl < dend && sl < s0 + 255 && nx[r] - off0 <= kStageRecBytes &&
                                ((nx[r] - 1u) >> c.page_shift) <= plast) ? 1u : 0u;
                    }
                    n = (int)__reduce_add_sync(0xffffffffu, cnt);
                    if (n < 1) {      // only with corrupt offsets: flag it, keep making progress
                        if (lane == 0) set_status(c.status, KVQ_ERR_DEVICE_CHECK);
                        n = 1;
                    }
                    const int kl = s0 + n - 1;
                    nxl = __shfl_sync(0xffffffffu, pick(nx, kl % KPL), kl / KPL);
                }
                const int s1 = s0 + n;
                const bool last = lastwin && s1 == dend;
                const bool new_item = first && s0 == d;
                uint32_t rec_bytes = nxl - off0;
                if (nxl < off0 || rec_bytes > kStageRecBytes) {   // corrupt offsets
                    if (lane == 0) set_status(c.status, KVQ_ERR_DEVICE_CHECK);
                    rec_bytes = 0;
                }
                // the stage's copies go out first; the width sort below overlaps their flight
                const int stage = issued % kStages;
                const uint32_t phase = (uint32_t)(issued / kStages) & 1u;
                if (!mbar_wait(&sm.empty[stage], phase ^ 1u, c.status)) {
                    aborted = true;
                    break;
                }
                Stage<D> &sg = sm.st[stage];
                if (lane == 0) {
                    // the item's subgroup of queries: rows sh * G + g0 .. of q (query head
                    // hk * G + g of sequence s is row (s * H + hk) * G + g), contiguous
                    const int g0 = qinfo & 0xFF;
                    const int nq = min(kDecodeMaxQ, c.G - g0);
                    const uint32_t q_bytes = new_item ? (uint32_t)(2 * D * nq) : 0u;
                    mbar_expect_tx(&sm.full[stage], 16u * n + rec_bytes + q_bytes);
                    bulk_g2s(sg.side, c.side + sbase + ja + s0, 16u * n, &sm.full[stage]);
                    if (rec_bytes) {
                        if (!c.ptab) {
                            // contiguous: the stream starts at its first slot * 4 * D bytes
                            bulk_g2s(sg.rec, c.rec + sbase * (4 * D) + off0, rec_bytes, &sm.full[stage]);
                        } else {
                            // a paged stream: one copy per page the stage's bytes touch
                            const uint32_t *pt = c.ptab + (size_t)sh * c.max_lpages;
                            const uint32_t pm = (1u << c.page_shift) - 1u;
                            const uint32_t n0 = min(rec_bytes, (pm + 1u) - (off0 & pm));
                            bulk_g2s(sg.rec, c.rec + ((size_t)pt[off0 >> c.page_shift] << c.page_shift) + (off0 & pm),
                                     n0, &sm.full[stage]);
                            if (rec_bytes > n0) {
                                const uint32_t o1 = off0 + n0;
                                bulk_g2s(sg.rec + n0, c.rec + ((size_t)pt[o1 >> c.page_shift] << c.page_shift) + (o1 & pm),
                                         rec_bytes - n0, &sm.full[stage]);
                            }
                        }
                    }
                    if (q_bytes)
                        bulk_g2s(sg.q, q + ((int64_t)sh * c.G + g0) * D, q_bytes, &sm.full[stage]);
                }
                // counting sort by width, four classes packed as bytes of one word: per-lane
                // counts, one warp prefix sum; each class's run padded to whole chunks of KPS
                // keys. Byte c of `cst` is class c's first position, of `run` this lane's
                // next rank in class c (no byte overflows: at most 255 keys plus padding)
                uint32_t lc = 0, shc[KPL];
                bool inr[KPL];
#pragma unroll
                for (int r = 0; r < KPL; ++r) {
                    const int sl = KPL * lane + r;
                    inr[r] = sl >= s0 && sl < s1;
                    shc[r] = (m[r] & 3u) << 3;
                    if (inr[r]) lc += 1u << shc[r];
                }
                uint32_t incl = lc;
#pragma unroll
                for (int dd = 1; dd < 32; dd <<= 1) {
                    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, dd);
                    if (lane >= dd) incl += y;
                }
                const uint32_t tot = __shfl_sync(0xffffffffu, incl, 31);
                constexpr uint32_t kRound = 0x01010101u * (uint32_t)(KPS - 1);
                const uint32_t padded = (tot + kRound) & ~kRound;      // run lengths, whole chunks
                const uint32_t cst = (padded << 8) + (padded << 16) + (padded << 24);
                const int pstart = (int)((cst >> 24) + (padded >> 24));
                uint32_t run = cst + incl - lc;
#pragma unroll
                for (int r = 0; r < KPL; ++r) {
                    if (inr[r]) {
                        const int pos = (int)((run >> shc[r]) & 0xFFu);
                        run += 1u << shc[r];
                        // offset inside the stage; the clamp only bites on corrupt offsets and
                        // keeps every shared-memory read of the consumers inside the stage
                        const uint32_t ro = min((m[r] & ~15u) - off0, kStageRecBytes - ((uint32_t)(D / 2) << (shc[r] >> 3)));
                        sg.perm[pos] = kValid | ((uint32_t)(KPL * lane + r - s0) << 16) | ro;
                    }
                }
                // padding entries have no valid bit, so the consumers weight them 0; they must
                // still read finite data: any bytes read as b-bit codes are finite (record 0
                // of the stage will do), fp16 values are not, so the b = 16 run repeats its
                // first key
                const uint32_t pad_at = cst + tot, pad_n = padded - tot;
                __syncwarp();
#pragma unroll
                for (int cl = 0; cl < 3; ++cl)
                    if (lane < (int)((pad_n >> (8 * cl)) & 0xFFu)) sg.perm[((pad_at >> (8 * cl)) & 0xFFu) + lane] = 0u;
                if (lane < (int)(pad_n >> 24)) sg.perm[(pad_at >> 24) + lane] = sg.perm[cst >> 24] & ~kValid;
                if (lane == 0) {
                    sg.info[0] = it;
                    sg.info[1] = n;
                    sg.info[2] = (new_item ? kNewItem : 0) | (last ? kLastSub : 0);
                    sg.info[3] = pstart / KPS;
                    sg.info[4] = qinfo;
#pragma unroll
                    for (int cl = 0; cl < 4; ++cl) sg.cls_chunk[cl] = (int)((cst >> (8 * cl)) & 0xFFu) / KPS;
                    sg.cls_chunk[4] = pstart / KPS;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.full[stage]);   // the stage's key list is written
                ++issued;
                s0 = s1;
            }
        }
        if (!aborted) {
            // no more items: the next stage carries only the stop mark
            const int stage = issued % kStages;
            if (mbar_wait(&sm.empty[stage], ((uint32_t)(issued / kStages) & 1u) ^ 1u, c.status)) {
                if (lane == 0) {
                    sm.st[stage].info[2] = kStop;
                    mbar_arrive(&sm.full[stage]);
                }
            } else {
                aborted = true;
            }
        }
        if (aborted) {
            // no copy may still be writing this CTA's shared memory when it exits: wait
            // (bounded) for the last copy issued into each stage and each offset window
            sm.abort_flag = 1;
            for (int b = 0; b < kStages; ++b)
                if (issued > b) {
                    const int i_last = b + kStages * ((issued - 1 - b) / kStages);
                    mbar_wait(&sm.full[b], (uint32_t)(i_last / kStages) & 1u, c.status, 100000000ull);
                }
            for (int b = 0; b < kMetaSlots; ++b)
                if (filled > b) {
                    const int i_last = b + kMetaSlots * ((filled - 1 - b) / kMetaSlots);
                    mbar_wait(&sm.mfull[b], (uint32_t)(i_last / kMetaSlots) & 1u, c.status, 100000000ull);
                }
        }
        return;
    }

    // -------------------------------- consumers -------------------------------------
    // Every consumer warp deposits its state for every item, also after a timed-out wait: a
    // warp that gave up only skips the waits and the work. Nothing waits on the deposits.
    const int g = lane / LPK;            // key slot within a chunk
    const int li = lane % LPK;           // channel block: channels [32 li, 32 li + 32)
    const float qk_scale = kLog2e * rsqrtf((float)D);   // logits in log2 units
    int stage = 0, rot = 0;
    uint32_t phase = 0;
    bool dead = false;
    QRegs Q;
    float qsum_l = 0.f;
    int ring = 0;                         // this item's merge slot
    for (;; ring = (ring + 1) % kMergeRing) {
        // the item's first stage, or the producer's stop mark
        if (dead) break;
        if (*reinterpret_cast<volatile int32_t *>(&sm.abort_flag) || !mbar_wait(&sm.full[stage], phase, c.status)) {
            sm.abort_flag = 1;
            break;
        }
        if (sm.st[stage].info[2] & kStop) break;
        const int it = sm.st[stage].info[0];
        bool waited = true;                   // the first stage's wait is done
        rot = 0;                              // chunks dealt by the item's own stage count:
                                              // results do not depend on the CTA's earlier items
        KeyState ks;
        ks.m = kMInit;
        ks.l = 0.f;
        ks.pz = 0.f;
#pragma unroll
        for (int k = 0; k < 16; ++k) ks.o[k] = make_float2(0.f, 0.f);
        int nq = 1, rank = warp, nws = kConsumerWarps, qmask = 1;
        bool last = false;
        while (!last && !dead) {
            if (!waited && (*reinterpret_cast<volatile int32_t *>(&sm.abort_flag) ||
                            !mbar_wait(&sm.full[stage], phase, c.status))) {
                dead = true;
                sm.abort_flag = 1;
                break;
            }
            waited = false;
            Stage<D> &sg = sm.st[stage];
            const int flags = sg.info[2];
            last = (flags & kLastSub) != 0;
            if (flags & kNewItem) {
                qmask = sg.info[4] >> 8;
                nq = __popc(qmask);
                const int sidx = warp % nq;        // the sidx-th active query of the item
                rank = warp / nq;
                nws = (kConsumerWarps - sidx + nq - 1) / nq;
                int qi = 0;
                for (int b = 0, seen = 0; b < kDecodeMaxQ; ++b)
                    if ((qmask >> b) & 1) {
                        if (seen == sidx) qi = b;
                        ++seen;
                    }
                // this lane's 32 channels of query g0 + qi, scaled; sum(q) over all D
                const uint4 *src = reinterpret_cast<const uint4 *>(sg.q[qi] + 32 * li);
                float qs = 0.f;
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const uint4 a = src[u], b = src[2 + u];     // channels 8u.., 16 + 8u..
                    const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 fa = __half22float2(*reinterpret_cast<const __half2 *>(&wa[e]));
                        const float2 fb = __half22float2(*reinterpret_cast<const __half2 *>(&wb[e]));
                        qs += (fa.x + fa.y) + (fb.x + fb.y);
                        Q.q[8 * u + 2 * e] = make_float2(fa.x * kQScale, fb.x * kQScale);
                        Q.q[8 * u + 2 * e + 1] = make_float2(fa.y * kQScale, fb.y * kQScale);
                    }
                }
#pragma unroll
                for (int d = 1; d < LPK; d <<= 1) qs += __shfl_xor_sync(0xffffffffu, qs, d);
                qsum_l = qs * qk_scale;
            }
            const float cdot = qk_scale * kDotCodeUnscale;
            // chunks sorted by width: the warps of this query deal them round-robin
            // (rotated every stage) and walk one run per width class
            int ch = (rank + rot) % nws;
            ch = run_class<D, 0>(ks, Q, qsum_l, cdot, sg, ch, sg.cls_chunk[1], nws, g, li);
            ch = run_class<D, 1>(ks, Q, qsum_l, cdot, sg, ch, sg.cls_chunk[2], nws, g, li);
            ch = run_class<D, 2>(ks, Q, qsum_l, cdot, sg, ch, sg.cls_chunk[3], nws, g, li);
            run_class<D, 3>(ks, Q, qsum_l, qk_scale * kDotNativeUnscale, sg, ch, sg.cls_chunk[4], nws, g, li);
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.empty[stage]);
            rot = (rot + 1) % kConsumerWarps;
            if (++stage == kStages) {
                stage = 0;
                phase ^= 1u;
            }
        }

        // Merge the key groups of the warp, deposit the warp's state in the item's merge
        // slot, and go on: the warp that deposits last merges the item's warps into the
        // partials of each of its queries (no barrier across the consumer warps).
#pragma unroll
        for (int mask = LPK; mask < 32; mask <<= 1) merge_state(ks, mask);
        if (g == 0) {
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                sm.red_o[ring][warp][32 * li + k] = ks.o[k].x;
                sm.red_o[ring][warp][32 * li + 16 + k] = ks.o[k].y;
            }
            if (li == 0) {
                sm.red_m[ring][warp] = ks.m;
                sm.red_l[ring][warp] = ks.l;
                sm.red_pz[ring][warp] = ks.pz;
            }
        }
        __syncwarp();
        int prev = 0;
        if (lane == 0) {
            __threadfence_block();
            prev = atomicAdd(&sm.merge_cnt[ring], 1);
        }
        prev = __shfl_sync(0xffffffffu, prev, 0);
        if (prev == kConsumerWarps - 1) {
            __threadfence_block();
            if (!dead) {
                // query sidx of the item is served by warps sidx, sidx + nq, ...; its slot in
                // the partials is the sidx-th set bit of the mask
                for (int sidx = 0, qi = 0; sidx < nq; ++sidx, ++qi) {
                    while (!((qmask >> qi) & 1)) ++qi;
                    float M = kMInit;
                    for (int wv = sidx; wv < kConsumerWarps; wv += nq) M = fmaxf(M, sm.red_m[ring][wv]);
                    float L = 0.f, PZ = 0.f;
                    for (int wv = sidx; wv < kConsumerWarps; wv += nq) {
                        const float f = ex2(sm.red_m[ring][wv] - M);
                        L = fmaf(sm.red_l[ring][wv], f, L);
                        PZ = fmaf(sm.red_pz[ring][wv], f, PZ);
                    }
                    float *part = wk.partials + ((int64_t)it * wk.qslots + qi) * (D + 4);
                    for (int chn = lane; chn < D; chn += 32) {
                        float acc = 0.f;
                        for (int wv = sidx; wv < kConsumerWarps; wv += nq)
                            acc = fmaf(sm.red_o[ring][wv][chn], ex2(sm.red_m[ring][wv] - M), acc);
                        part[4 + chn] = fmaf(acc, kOUnscale, PZ);
                    }
                    if (lane == 0) {
                        part[0] = M;
                        part[1] = L;
                    }
                }
            }
            __syncwarp();
            if (lane == 0) atomicExch(&sm.merge_cnt[ring], 0);   // the slot is free again
        }
    }
}

// Calls with many (sequence, query head) outputs: one warp per output, kCombineWarps warps
// per CTA, D/32 channels per lane. The query's partials are those of its KV head's items whose subgroup holds it as an
// active query. The lanes share the per-item work (the maximum, then each item's weight
// 2^(m_i - M) and the sum of the l_i weights, 32 items a round); then every lane sums the
// weighted o_i of its channels over the round's items, in item order, with independent
// loads. No block barrier.
constexpr int kCombineWarps = 4;
constexpr int kCombineThreads = 32 * kCombineWarps;
constexpr int kCombineWarpMinPerSm = 4;      // outputs per SM from which the warp form is used

template <int D>
__global__ void __launch_bounds__(kCombineThreads)
decode_combine_warp_kernel(CacheView c, DecodeWork wk, float *__restrict__ out)
{
    constexpr int CPL = D / 32;                   // channels per lane
    static_assert(CPL == 2 || CPL == 4, "head_dim 64 or 128");
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int HQ = c.H * c.G;
    const int shq = blockIdx.x * kCombineWarps + (int)(threadIdx.x >> 5);
    if (shq >= c.B * HQ) return;                  // warp-uniform
    const int s = shq / HQ, hq = shq % HQ, hk = hq / c.G, gq = hq % c.G;
    const int unit = s * c.H + hk, BH = c.B * c.H;
    // the KV head's front, back and middle items (a run outside the list is ignored: the
    // planning kernel has reported it)
    int first[3], run[3];
#pragma unroll
    for (int r = 0; r < 3; ++r) {
        first[r] = wk.head_first[r * BH + unit];
        run[r] = wk.head_cnt[r * BH + unit];
        if (first[r] < 0 || run[r] < 0 || first[r] + (int64_t)run[r] > wk.max_items) run[r] = 0;
    }
    const int cnt = run[0] + run[1] + run[2];
    const int QS = wk.qslots;
    auto part_of = [&](int i) -> int64_t {      // this query's partial of the head's item i, or -1
        const int ix = (i < run[0]) ? first[0] + i
                     : (i < run[0] + run[1]) ? first[1] + (i - run[0]) : first[2] + (i - run[0] - run[1]);
        const int qinfo = wk.items[ix].qinfo;
        const int d = gq - (qinfo & 0xFF);
        if (d < 0 || d >= kDecodeMaxQ || !((qinfo >> (8 + d)) & 1)) return -1;
        return ((int64_t)ix * QS + d) * (D + 4);
    };
    // (m, l) of a partial; l = 0 marks a pair tail that the split-K kernel walked with its
    // head (a walked item has l >= 1): it takes no part
    auto ml_of = [&](int64_t p) { return *reinterpret_cast<const float2 *>(wk.partials + p); };
    auto o_of = [&](int64_t p, float (&v)[CPL]) {  // this lane's channels of o
        const float *src = wk.partials + p + 4 + CPL * lane;
        if constexpr (CPL == 4) {
            const float4 x = *reinterpret_cast<const float4 *>(src);
            v[0] = x.x;
            v[1] = x.y;
            v[2] = x.z;
            v[3] = x.w;
        } else {
            const float2 x = *reinterpret_cast<const float2 *>(src);
            v[0] = x.x;
            v[1] = x.y;
        }
    };
    float M = kMInit;
    for (int i = lane; i < cnt; i += 32) {
        const int64_t p = part_of(i);
        if (p >= 0) {
            const float2 ml = ml_of(p);
            if (ml.y > 0.f) M = fmaxf(M, ml.x);
        }
    }
#pragma unroll
    for (int dd = 16; dd >= 1; dd >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, dd));
    // (the summation order is fixed: results do not depend on thread timing)
    float L = 0.f, acc[CPL];
#pragma unroll
    for (int k = 0; k < CPL; ++k) acc[k] = 0.f;
    for (int i0 = 0; i0 < cnt; i0 += 32) {
        float f = 0.f;
        int64_t pi = -1;
        if (i0 + lane < cnt) {
            const int64_t p = part_of(i0 + lane);
            if (p >= 0) {
                const float2 ml = ml_of(p);
                if (ml.y > 0.f) {
                    f = ex2(ml.x - M);
                    L = fmaf(ml.y, f, L);
                    pi = p;
                }
            }
        }
        const int n = min(32, cnt - i0);
        int k = 0;
        for (; k + 8 <= n; k += 8) {               // 8 independent loads per round
            float v[8][CPL], fk[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int64_t pu = __shfl_sync(0xffffffffu, pi, k + u);
                fk[u] = __shfl_sync(0xffffffffu, f, k + u);
                if (pu >= 0) o_of(pu, v[u]);
                else {
#pragma unroll
                    for (int q = 0; q < CPL; ++q) v[u][q] = 0.f;
                }
            }
#pragma unroll
            for (int u = 0; u < 8; ++u)
#pragma unroll
                for (int q = 0; q < CPL; ++q) acc[q] = fmaf(v[u][q], fk[u], acc[q]);
        }
        for (; k < n; ++k) {
            const int64_t pu = __shfl_sync(0xffffffffu, pi, k);
            const float fu = __shfl_sync(0xffffffffu, f, k);
            if (pu >= 0) {
                float v[CPL];
                o_of(pu, v);
#pragma unroll
                for (int q = 0; q < CPL; ++q) acc[q] = fmaf(v[q], fu, acc[q]);
            }
        }
    }
#pragma unroll
    for (int dd = 16; dd >= 1; dd >>= 1) L += __shfl_xor_sync(0xffffffffu, L, dd);
    float *dst = out + (int64_t)shq * D + CPL * lane;
#pragma unroll
    for (int q = 0; q < CPL; ++q) dst[q] = (L > 0.f) ? acc[q] / L : 0.f;
}

// Calls with few outputs (long contexts over few heads, many items per output): one CTA of D
// threads per (sequence, query head). The query's partials are those of its
// KV head's items whose subgroup holds it as an active query. The threads first share the
// per-item work (the maximum, then each item's weight 2^(m_i - M) and the sum of l_i
// weights, kept in shared memory for a chunk of items), then thread = channel sums the
// weighted o_i of the chunk with independent loads.
constexpr int kCombineChunk = 256;

template <int D>
__global__ void __launch_bounds__(D)
decode_combine_kernel(CacheView c, DecodeWork wk, float *__restrict__ out)
{
    __shared__ float f_sh[kCombineChunk];
    __shared__ int32_t idx_sh[kCombineChunk];
    __shared__ float red[D / 32];
    pdl_wait();
    pdl_trigger();
    const int HQ = c.H * c.G;
    const int shq = blockIdx.x, ch = threadIdx.x, lane = ch & 31, wid = ch >> 5;
    const int s = shq / HQ, hq = shq % HQ, hk = hq / c.G, gq = hq % c.G;
    const int unit = s * c.H + hk, BH = c.B * c.H;
    // the KV head's front, back and middle items (a run outside the list is ignored: the
    // planning kernel has reported it)
    int first[3], run[3];
#pragma unroll
    for (int r = 0; r < 3; ++r) {
        first[r] = wk.head_first[r * BH + unit];
        run[r] = wk.head_cnt[r * BH + unit];
        if (first[r] < 0 || run[r] < 0 || first[r] + (int64_t)run[r] > wk.max_items) run[r] = 0;
    }
    const int cnt = run[0] + run[1] + run[2];
    const int QS = wk.qslots;
    auto part_of = [&](int i) -> int64_t {      // this query's partial of the head's item i, or -1
        const int ix = (i < run[0]) ? first[0] + i
                     : (i < run[0] + run[1]) ? first[1] + (i - run[0]) : first[2] + (i - run[0] - run[1]);
        const int qinfo = wk.items[ix].qinfo;
        const int d = gq - (qinfo & 0xFF);
        if (d < 0 || d >= kDecodeMaxQ || !((qinfo >> (8 + d)) & 1)) return -1;
        return ((int64_t)ix * QS + d) * (D + 4);
    };
    // (m, l) of a partial; l = 0 marks a pair tail that the split-K kernel walked with its
    // head (a walked item has l >= 1): it takes no part
    auto ml_of = [&](int64_t p) { return *reinterpret_cast<const float2 *>(wk.partials + p); };
    float M = kMInit;
    for (int i = ch; i < cnt; i += D) {
        const int64_t p = part_of(i);
        if (p >= 0) {
            const float2 ml = ml_of(p);
            if (ml.y > 0.f) M = fmaxf(M, ml.x);
        }
    }
#pragma unroll
    for (int dd = 16; dd >= 1; dd >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, dd));
    if (lane == 0) red[wid] = M;
    __syncthreads();
    M = red[0];
#pragma unroll
    for (int w2 = 1; w2 < D / 32; ++w2) M = fmaxf(M, red[w2]);
    __syncthreads();
    // (the summation order is fixed: results do not depend on thread timing)
    float L = 0.f, acc = 0.f;
    for (int i0 = 0; i0 < cnt; i0 += kCombineChunk) {
        const int n = min(cnt - i0, kCombineChunk);
        for (int k = ch; k < n; k += D) {
            int64_t p = part_of(i0 + k);
            float f = 0.f;
            if (p >= 0) {
                const float2 ml = ml_of(p);
                if (ml.y > 0.f) {
                    f = ex2(ml.x - M);
                    L = fmaf(ml.y, f, L);
                } else {
                    p = -1;
                }
            }
            f_sh[k] = f;
            idx_sh[k] = (p >= 0) ? (int32_t)(p / (D + 4)) : -1;
        }
        __syncthreads();
        // 16 independent loads per round: a long item list costs few L2 round trips
        int k = 0;
        for (; k + 16 <= n; k += 16) {
            float v[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int32_t ix = idx_sh[k + u];
                v[u] = (ix >= 0) ? wk.partials[(int64_t)ix * (D + 4) + 4 + ch] : 0.f;
            }
#pragma unroll
            for (int u = 0; u < 16; ++u) acc = fmaf(v[u], f_sh[k + u], acc);
        }
        for (; k + 4 <= n; k += 4) {
            float v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int32_t ix = idx_sh[k + u];
                v[u] = (ix >= 0) ? wk.partials[(int64_t)ix * (D + 4) + 4 + ch] : 0.f;
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) acc = fmaf(v[u], f_sh[k + u], acc);
        }
        for (; k < n; ++k) {
            const int32_t ix = idx_sh[k];
            if (ix >= 0) acc = fmaf(wk.partials[(int64_t)ix * (D + 4) + 4 + ch], f_sh[k], acc);
        }
        __syncthreads();
    }
    // L: every thread summed the l of its own items; the block sum is the denominator
#pragma unroll
    for (int dd = 16; dd >= 1; dd >>= 1) L += __shfl_xor_sync(0xffffffffu, L, dd);
    if (lane == 0) red[wid] = L;
    __syncthreads();
    L = 0.f;
#pragma unroll
    for (int w2 = 0; w2 < D / 32; ++w2) L += red[w2];
    out[(int64_t)shq * D + ch] = (L > 0.f) ? acc / L : 0.f;
}

template <int D>
cudaError_t launch_decode_t(const kvq_cache *cache, const DecodeWork &wk, uint32_t gen, const __half *q,
                            const uint8_t *modes, int w, float *out, cudaStream_t st, const AppendArgs *ap)
{
    const CacheView &c = cache->view;
    cudaError_t e;
    if (ap)
        e = launch_pdl(decode_plan_kernel<D, true>, dim3(c.B), dim3(kPlanThreads), 0, st, c, modes, w, wk, gen, *ap);
    else
        e = launch_pdl(decode_plan_kernel<D, false>, dim3(c.B), dim3(kPlanThreads), 0, st, c, modes, w, wk, gen,
                       AppendArgs{});
    if (e != cudaSuccess) return e;
    const size_t smem = sizeof(DecodeSmem<D>);
    e = ensure_smem_attr((const void *)decode_splitk_kernel<D>, smem);
    if (e != cudaSuccess) return e;
    const int grid = (int)std::min<int64_t>(wk.max_items, kCtasPerSm * (int64_t)num_sms());
    profile_before(st);
    e = launch_pdl(decode_splitk_kernel<D>, dim3(grid), dim3(kThreads), smem, st, c, q, wk);
    if (e != cudaSuccess) return e;
    profile_after(st);
    // a warp per output once there are enough outputs to fill the GPU with warps (measured:
    // decode_1p3b's 1024 outputs 0.9 us faster per step; decode_long's 128 outputs of about
    // 60 items each 4 us slower than with a CTA per output)
    const int n_out = c.B * c.H * c.G;
    if (n_out >= kCombineWarpMinPerSm * num_sms())
        e = launch_pdl(decode_combine_warp_kernel<D>, dim3((n_out + kCombineWarps - 1) / kCombineWarps),
                       dim3(kCombineThreads), 0, st, c, wk, out);
    else
        e = launch_pdl(decode_combine_kernel<D>, dim3(n_out), dim3(D), 0, st, c, wk, out);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

// wk.count points at kDecodeCountWords words: the pair of front count words, the item
// cursor, the pair of back count words, the pair of middle count words; the call uses the
// words of parity gen & 1. `stale` is set when a launch fails (a call whose planning kernel
// did not run leaves the next call's word unprepared); the words are then cleared (tag 0,
// never used) before the next call.
cudaError_t launch_any(const kvq_cache *cache, const DecodeWork &wk, uint32_t gen, const __half *q,
                       const uint8_t *modes, int w, float *out, cudaStream_t st, const AppendArgs *ap,
                       bool &stale)
{
    if (stale) {
        const cudaError_t e = cudaMemsetAsync(wk.count, 0, kDecodeCountWords * sizeof(unsigned long long), st);
        if (e != cudaSuccess) return e;
        stale = false;
    }
    DecodeWork cw = wk;
    cw.count = wk.count + (gen & 1u);
    cw.count_next = wk.count + ((gen + 1u) & 1u);
    cw.cursor = reinterpret_cast<uint32_t *>(wk.count + 2);
    cw.count_back = wk.count + 3 + (gen & 1u);
    cw.count_back_next = wk.count + 3 + ((gen + 1u) & 1u);
    cw.count_mid = wk.count + 5 + (gen & 1u);
    cw.count_mid_next = wk.count + 5 + ((gen + 1u) & 1u);
    cw.gen = gen;
    const cudaError_t e = (cache->D == 128) ? launch_decode_t<128>(cache, cw, gen, q, modes, w, out, st, ap)
                                            : launch_decode_t<64>(cache, cw, gen, q, modes, w, out, st, ap);
    if (e != cudaSuccess) stale = true;
    return e;
}

} // namespace

cudaError_t launch_decode(const kvq_cache *cache, const __half *q, const uint8_t *modes, int w,
                          float *out, cudaStream_t st)
{
    kvq_cache *mc = const_cast<kvq_cache *>(cache);   // the call's generation id only
    uint32_t gen = ++mc->decode_gen;
    if (gen == 0) gen = ++mc->decode_gen;             // 0 tags a count word never used
    return launch_any(cache, cache->work, gen, q, modes, w, out, st, nullptr, mc->work_stale);
}

cudaError_t launch_decode_step(kvq_cache *cache, const __half *q, const __half *k, const __half *v,
                               const uint8_t *bits, const int32_t *cu, int64_t n_tok,
                               const int32_t *positions, const uint8_t *modes, int w, float *out,
                               cudaStream_t st)
{
    AppendArgs ap{k, v, bits, cu, positions, n_tok, ++cache->write_gen};
    uint32_t gen = ++cache->decode_gen;
    if (gen == 0) gen = ++cache->decode_gen;
    return launch_any(cache, cache->work, gen, q, modes, w, out, st, &ap, cache->work_stale);
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
std::atomic<uint32_t> g_static_gen[256];   // per device ordinal: generation of the last call
bool g_static_stale[256] = {};             // per device ordinal: a launch failed (under g_scratch_mu)

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

} // namespace
} // namespace kvq

extern "C" int routed_attn_decode_noalloc(const void *q, const kvq_cache *cache, const uint8_t *modes,
                                          int w, float *out, kvq_stream_t stream)
{
    using namespace kvq;
    struct Range {                 // NVTX range around the call
        Range() { nvtxRangePushA("routed_attn_decode_noalloc"); }
        ~Range() { nvtxRangePop(); }
    } range;
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

    // scratch layout: count words and cursor | head_first | head_cnt | items | partials, each
    // 256-byte aligned, sized for the cache's worst case (every head full at capacity)
    const int BH = cache->B * cache->H;                     // (sequence, KV head) units
    const int64_t items = cache->work.max_items;
    const int qslots = cache->work.qslots;
    const size_t o_first = 256;
    const size_t o_cnt = o_first + align256(sizeof(int32_t) * 3 * (size_t)BH);
    const size_t o_items = o_cnt + align256(sizeof(int32_t) * 3 * (size_t)BH);
    const size_t o_part = o_items + align256(sizeof(DecodeItem) * (size_t)items);
    const size_t need = o_part + sizeof(float) * (size_t)items * qslots * (cache->D + 4);
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
    wk.count = reinterpret_cast<unsigned long long *>(base);
    wk.head_first = reinterpret_cast<int32_t *>(base + o_first);
    wk.head_cnt = reinterpret_cast<int32_t *>(base + o_cnt);
    wk.items = reinterpret_cast<DecodeItem *>(base + o_items);
    wk.partials = reinterpret_cast<float *>(base + o_part);
    wk.max_items = items;
    wk.mid_base = cache->work.mid_base;
    wk.qslots = qslots;
    // a generation id no earlier call on the shared array used (never 0, the tag of a word
    // never used: the array starts zeroed)
    uint32_t gen = ++g_static_gen[dev];
    if (gen == 0) gen = ++g_static_gen[dev];
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    {
        std::lock_guard<std::mutex> lock(g_scratch_mu);
        e = launch_any(cache, wk, gen, static_cast<const __half *>(q), modes, w, out, st, nullptr, g_static_stale[dev]);
    }
    if (e != cudaSuccess) return report_error(KVQ_ERR_CUDA, "routed_attn_decode_noalloc: kernel launch failed");
    return report_error(KVQ_OK, "");
}
