"""The quantize kernel forms the fp32 quotient u / s as q0 = RN(u * y), y = RN(1 / s),
r = fma(-s, q0, u), q = RN(q0 + r * y) (Markstein's correction, IBM J. Res. Dev. 34(1),
1990) and rounds it to an integer by adding 1.5 * 2^23. The codes must equal those of the
IEEE division followed by rint, bit for bit. This test checks that claim on the host in
plain C over the kernel's input domain: u = fl(x - z) is 0 or at least 2^-24 (x, z fp16),
0 <= u <= R, s = fl(R / (2^b - 1)) with R = fl(max - min) in [2^-24, 2^17).

Random pairs are drawn uniformly over the fp32 bit patterns of R and u, and half of them
are placed within a few ulps of a half-integer quotient (where a wrong rounding would
show). No GPU, no oracle: this pins the arithmetic identity the kernel relies on.
"""
import os
import subprocess

import pytest

BUILD = os.path.join(os.path.dirname(os.path.abspath(__file__)), "_build")

SRC = r"""
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

static uint64_t st = 0x9E3779B97F4A7C15ull;
static uint64_t rnd(void) { st ^= st << 13; st ^= st >> 7; st ^= st << 17; return st; }
static float fb(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t bf(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

int main(int argc, char **argv)
{
    const long n = atol(argv[1]);
    const float tops[3] = {3.f, 15.f, 255.f};
    long tested = 0, bad_q = 0, bad_code = 0;
    for (long i = 0; i < n; ++i) {
        const float top = tops[rnd() % 3];
        const float R = fb(0x33800000u + (uint32_t)(rnd() % (0x48000000u - 0x33800000u)));
        const float s = R / top;
        float u;
        if (rnd() & 1) {
            u = fb((uint32_t)(rnd() % (bf(R) + 1u)));
            if (u != 0.f && u < 0x1p-24f) continue;
        } else {                       /* near the half-integer k + 0.5 */
            const float k = (float)(rnd() % (uint32_t)top) + 0.5f;
            u = fb(bf(k * s) + (uint32_t)(rnd() % 9) - 4u);
            if (!(u >= 0x1p-24f && u <= R)) continue;
        }
        const float y = 1.0f / s;
        const float q0 = u * y;
        const float r = fmaf(-s, q0, u);
        const float q = fmaf(r, y, q0);
        const float ref = u / s;
        ++tested;
        if (bf(q) != bf(ref)) ++bad_q;
        const uint32_t code = bf(q + 12582912.0f) - 0x4B400000u;
        const float c = fminf(fmaxf(rintf(ref), 0.f), top);
        if (code != (uint32_t)c) ++bad_code;
    }
    printf("%ld %ld %ld\n", tested, bad_q, bad_code);
    return 0;
}
"""


def test_corrected_quotient_matches_ieee_division():
    os.makedirs(BUILD, exist_ok=True)
    c = os.path.join(BUILD, "exact_quotient.c")
    exe = os.path.join(BUILD, f"exact_quotient_{os.getpid()}")
    with open(c + f".{os.getpid()}", "w") as f:
        f.write(SRC)
    try:
        subprocess.run(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-x", "c", "-o", exe,
                        c + f".{os.getpid()}", "-lm"], check=True, capture_output=True)
    except (OSError, subprocess.CalledProcessError) as e:   # no C compiler: nothing to run
        pytest.skip(f"gcc unavailable: {e}")
    try:
        out = subprocess.run([exe, "20000000"], check=True, capture_output=True, text=True).stdout
    finally:
        for f in (exe, c + f".{os.getpid()}"):
            if os.path.exists(f):
                os.remove(f)
    tested, bad_q, bad_code = map(int, out.split())
    assert tested > 10_000_000
    assert bad_q == 0 and bad_code == 0, (tested, bad_q, bad_code)
