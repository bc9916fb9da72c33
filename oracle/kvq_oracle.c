/*
 * Plain CPU oracle for the routed mixed-precision KV write and routed attention of
 * "TriRoute: Unified Learned Routing for Joint Adaptive Attention, Experts, and
 * KV-Cache Allocation" (paper review page, section 3 "technical architecture").
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may link, load or call this
 * file: only the tests, the package's smoke check and the benchmark's CPU-baseline leg
 * use it. It shares no code, header, table or constant with the CUDA library.
 *
 * What it computes, and where each step comes from:
 *   - oracle_quantize:   Eq. 4, asymmetric min/max quantization of one vector
 *                        (s = (max - min) / (2^b - 1), z = min, code = round((x - z)/s)),
 *                        b = 16 meaning native (fp16) storage.
 *   - oracle_dequantize: Eq. 4, Q_b(x) = code * s + z, evaluated in fp64.
 *   - oracle_routed_attention_head: Eq. 2, Attn_t = sum_m 1[a_t = m] Attn_t^(m) with
 *                        skip -> 0, local -> Attn(q_t, K[t-w, t], V[t-w, t]),
 *                        full -> Attn(q_t, K[<=t], V[<=t]), over the dequantized cache,
 *                        softmax in fp64.
 *   - oracle_route_argmax: the inference-time router (section 3 item 5, Eq. 5, and the
 *                        "inference" paragraph of the training procedure): the hard argmax
 *                        of each row of controller logits, z^a over {skip, local, full} and
 *                        z^b over the widths {2, 4, 8, 16}.
 *
 * Readings taken where the pages leave a step open (each is also listed in the design notes):
 *   - the quantization group is one (token, head) vector of head_dim values;
 *   - the integer decision is made in fp32 with IEEE round-to-nearest-even subtraction,
 *     division and rint (the precision the kernels use), s = 0 gives code 0;
 *   - b = 16 keeps the raw fp16 bits, with side entry (s, z) = (1, 0);
 *   - local window is inclusive, keys max(0, t - w) .. t (w + 1 keys once t >= w);
 *   - the softmax scale is 1/sqrt(head_dim); the output is stored as fp32;
 *   - the router's argmax compares the fp32 logits as given; a tie goes to the first
 *     (lowest) index, and a NaN logit never wins (all-NaN rows give index 0).
 *
 * Build: gcc -O2 -std=c99 -ffp-contract=off -fno-fast-math -shared -fPIC
 * (no FMA contraction, so every fp32 operation rounds exactly once as written).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* IEEE-754 binary16 -> binary32, from the format's definition (exact). */
static float half_bits_to_float(uint16_t h)
{
    unsigned sign = (h >> 15) & 1u;
    unsigned e = (h >> 10) & 0x1Fu;
    unsigned m = h & 0x3FFu;
    float mag;
    if (e == 0) {
        mag = ldexpf((float)m, -24);                 /* subnormal: m * 2^-24 */
    } else if (e == 31) {
        mag = m ? NAN : INFINITY;
    } else {
        mag = ldexpf((float)(m + 1024u), (int)e - 25); /* (1024 + m) * 2^(e - 15 - 10) */
    }
    return sign ? -mag : mag;
}

double oracle_half_to_double(uint16_t h) { return (double)half_bits_to_float(h); }

/*
 * Eq. 4 on one vector of n fp16 values (raw bits).
 * b in {2, 4, 8}: codes[i] in [0, 2^b - 1], *s_out = (max - min) / (2^b - 1), *z_out = min.
 * b == 16: codes[i] = raw fp16 bits of x[i], (*s_out, *z_out) = (1, 0).
 * Returns 0, or -1 for an unsupported b or n <= 0.
 */
int oracle_quantize(const uint16_t *x, int n, int b, uint16_t *codes, float *s_out, float *z_out)
{
    if (n <= 0) return -1;
    if (b == 16) {
        for (int i = 0; i < n; ++i) codes[i] = x[i];
        *s_out = 1.0f;
        *z_out = 0.0f;
        return 0;
    }
    if (b != 2 && b != 4 && b != 8) return -1;

    /* min and max of the group (fp16 -> fp32 is exact) */
    float mn = half_bits_to_float(x[0]);
    float mx = mn;
    for (int i = 1; i < n; ++i) {
        float xi = half_bits_to_float(x[i]);
        if (xi < mn) mn = xi;
        if (xi > mx) mx = xi;
    }
    const unsigned top = (1u << b) - 1u;          /* 2^b - 1 */
    const float range = mx - mn;                  /* fp32, round to nearest even */
    /* "+ 0.0f" stores a zero as +0: min(x) and s are values, and -0 and +0 are one value
       (which of the two a min scan meets first depends on the scan order) */
    const float s = range / (float)top + 0.0f;    /* fp32 IEEE division */
    const float z = mn + 0.0f;
    for (int i = 0; i < n; ++i) {
        unsigned c = 0;
        if (s != 0.0f) {
            float xi = half_bits_to_float(x[i]);
            float r = (xi - z) / s;               /* fp32 sub, fp32 div */
            float rr = rintf(r);                  /* round half to even (default mode) */
            if (rr < 0.0f) rr = 0.0f;
            if (rr > (float)top) rr = (float)top;
            c = (unsigned)rr;
        }
        codes[i] = (uint16_t)c;
    }
    *s_out = s;
    *z_out = z;
    return 0;
}

/* Batched form: m vectors of n values each, bits[j] per vector. Returns 0 or -1. */
int oracle_quantize_many(const uint16_t *x, int m, int n, const uint8_t *bits,
                         uint16_t *codes, float *s_out, float *z_out)
{
    for (int j = 0; j < m; ++j) {
        int rc = oracle_quantize(x + (size_t)j * n, n, bits[j], codes + (size_t)j * n,
                                 s_out + j, z_out + j);
        if (rc) return rc;
    }
    return 0;
}

/* Eq. 4 reconstruction Q_b(x) = code * s + z in fp64; b == 16 reads the fp16 bits. */
void oracle_dequantize(const uint16_t *codes, int n, int b, float s, float z, double *out)
{
    for (int i = 0; i < n; ++i) {
        if (b == 16)
            out[i] = oracle_half_to_double(codes[i]);
        else
            out[i] = (double)codes[i] * (double)s + (double)z;
    }
}

enum { ORACLE_SKIP = 0, ORACLE_LOCAL = 1, ORACLE_FULL = 2 };

/*
 * Eq. 2 for one (sequence, head) over a cache of L tokens whose K/V were written with
 * Eq. 4 at widths bits[0..L).
 *   k, v:   fp16 bits [L][D] (the values before quantization)
 *   bits:   [L] in {2, 4, 8, 16}
 *   q:      fp16 bits [n_q][D]; pos[i] = 0-based position t of query i, t < L
 *   modes:  [n_q] 0 = skip, 1 = local-w, 2 = full
 *   out:    fp32 [n_q][D]
 * Returns 0; -1 on a bad argument (bad bits, bad mode, t outside [0, L), w < 0), -2 on
 * allocation failure.
 */
int oracle_routed_attention_head(int D, int L, const uint16_t *k, const uint16_t *v,
                                 const uint8_t *bits, int n_q, const uint16_t *q,
                                 const int32_t *pos, const uint8_t *modes, int w, float *out)
{
    if (D <= 0 || L < 0 || n_q < 0 || w < 0) return -1;

    /* The union of the key ranges the queries read: only those keys are dequantized. */
    int lo_all = L, hi_all = -1;
    for (int i = 0; i < n_q; ++i) {
        int t = pos[i];
        if (modes[i] > ORACLE_FULL) return -1;
        if (modes[i] == ORACLE_SKIP) continue;
        if (t < 0 || t >= L) return -1;
        int lo = (modes[i] == ORACLE_LOCAL) ? (t - w > 0 ? t - w : 0) : 0;
        if (lo < lo_all) lo_all = lo;
        if (t > hi_all) hi_all = t;
    }

    double *kd = NULL, *vd = NULL, *logit = NULL, *qd = NULL;
    uint16_t *codes = NULL;
    int n_keys = hi_all >= lo_all ? hi_all - lo_all + 1 : 0;
    int rc = 0;
    if (n_keys > 0) {
        kd = (double *)malloc(sizeof(double) * (size_t)n_keys * D);
        vd = (double *)malloc(sizeof(double) * (size_t)n_keys * D);
        logit = (double *)malloc(sizeof(double) * (size_t)n_keys);
        codes = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)D);
        if (!kd || !vd || !logit || !codes) { rc = -2; goto done; }
        for (int j = lo_all; j <= hi_all; ++j) {
            float s, z;
            int b = bits[j];
            if (oracle_quantize(k + (size_t)j * D, D, b, codes, &s, &z)) { rc = -1; goto done; }
            oracle_dequantize(codes, D, b, s, z, kd + (size_t)(j - lo_all) * D);
            if (oracle_quantize(v + (size_t)j * D, D, b, codes, &s, &z)) { rc = -1; goto done; }
            oracle_dequantize(codes, D, b, s, z, vd + (size_t)(j - lo_all) * D);
        }
    }
    qd = (double *)malloc(sizeof(double) * (size_t)D);
    if (!qd) { rc = -2; goto done; }

    const double scale = 1.0 / sqrt((double)D);
    for (int i = 0; i < n_q; ++i) {
        float *o = out + (size_t)i * D;
        if (modes[i] == ORACLE_SKIP) {            /* Attn^skip = 0 */
            for (int c = 0; c < D; ++c) o[c] = 0.0f;
            continue;
        }
        int t = pos[i];
        int lo = (modes[i] == ORACLE_LOCAL) ? (t - w > 0 ? t - w : 0) : 0;
        for (int c = 0; c < D; ++c) qd[c] = oracle_half_to_double(q[(size_t)i * D + c]);

        double mx = -INFINITY;
        for (int j = lo; j <= t; ++j) {
            const double *kj = kd + (size_t)(j - lo_all) * D;
            double acc = 0.0;
            for (int c = 0; c < D; ++c) acc += qd[c] * kj[c];
            logit[j - lo] = acc * scale;
            if (logit[j - lo] > mx) mx = logit[j - lo];
        }
        double denom = 0.0;
        for (int j = lo; j <= t; ++j) {
            logit[j - lo] = exp(logit[j - lo] - mx);
            denom += logit[j - lo];
        }
        for (int c = 0; c < D; ++c) {
            double acc = 0.0;
            for (int j = lo; j <= t; ++j) acc += logit[j - lo] * vd[(size_t)(j - lo_all) * D + c];
            o[c] = (float)(acc / denom);
        }
    }
done:
    free(kd);
    free(vd);
    free(logit);
    free(qd);
    free(codes);
    return rc;
}

/*
 * Hard argmax of n rows of k fp32 logits (row-major), first index on ties: the router at
 * inference picks the mode (k = 3: skip, local, full) and the width index (k = 4:
 * b = 2, 4, 8, 16) of each (token, head). NaN entries are passed over; a row of NaNs
 * gives index 0.
 */
void oracle_route_argmax(const float *z, int64_t n, int k, uint8_t *out)
{
    for (int64_t r = 0; r < n; ++r) {
        const float *row = z + r * k;
        int best = -1;
        for (int i = 0; i < k; ++i) {
            if (isnan(row[i])) continue;
            if (best < 0 || row[i] > row[best]) best = i;
        }
        out[r] = (uint8_t)(best < 0 ? 0 : best);
    }
}
