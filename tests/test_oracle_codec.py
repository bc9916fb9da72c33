"""Pins for the oracle's Eq. 4 codec (TriRoute paper review page, section 3, Eq. 4).

Each check ties the oracle to something other than itself: hand-worked examples
(tests/golden), numpy's own fp16 conversion, brute-force enumeration of every code,
closed-form properties (code of min/max, constant vectors, b = 16 round trip) and the
quantizer's error bound.
"""
import json
import os

import numpy as np
import pytest

import oracle


def _load(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


def test_half_conversion_matches_numpy_for_every_pattern():
    # every finite fp16 bit pattern converts exactly as numpy's independent conversion does
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([oracle.half_to_double(int(b)) for b in bits[::7]])
    r = ref[::7]
    finite = np.isfinite(r)
    assert np.array_equal(got[finite], r[finite])
    assert np.all(np.isinf(got[np.isinf(r)]))
    assert np.all(np.isnan(got[np.isnan(r)]))


def test_worked_examples(golden_dir):
    g = _load(golden_dir, "codec_worked_examples.json")
    for case in g["cases"]:
        if "x_bits" in case:
            x = np.array(case["x_bits"], dtype=np.uint16)
        else:
            x = np.array(case["x"], dtype=np.float16)
        codes, s, z = oracle.quantize(x, case["b"])
        assert codes.tolist() == case["codes"], case["name"]
        assert float(s) == pytest.approx(case["s"], rel=0, abs=0), case["name"]
        assert float(z) == case["z"], case["name"]
        deq = oracle.dequantize(codes, case["b"], s, z)
        assert deq.tolist() == case["deq"], case["name"]


def _rand_vectors(rng, m, n, scale=1.0):
    x = (rng.standard_normal((m, n)) * scale).astype(np.float16)
    return x


@pytest.mark.parametrize("b", [2, 4, 8])
def test_brute_force_nearest_code(b):
    # For tiny vectors, every stored code is the integer in [0, 2^b - 1] nearest to the fp32
    # quotient fl((x - z)/s), ties to the even code: checked by enumerating all 2^b codes.
    rng = np.random.default_rng(7 + b)
    top = (1 << b) - 1
    for _ in range(300):
        x = _rand_vectors(rng, 1, 8, scale=rng.uniform(0.01, 50.0))[0]
        codes, s, z = oracle.quantize(x, b)
        xf = x.astype(np.float32)
        for i in range(8):
            if s == 0:
                assert codes[i] == 0
                continue
            r = (xf[i] - np.float32(z)) / np.float32(s)      # the fp32 quotient
            cand = np.arange(top + 1, dtype=np.float64)
            d = np.abs(cand - np.float64(r))
            best = np.flatnonzero(d == d.min())
            want = best[0] if len(best) == 1 else best[best % 2 == 0][0]
            assert codes[i] == want


@pytest.mark.parametrize("b", [2, 4, 8])
def test_extremes_map_to_end_codes(b):
    rng = np.random.default_rng(100 + b)
    top = (1 << b) - 1
    x = _rand_vectors(rng, 400, 64, scale=3.0)
    codes, s, z = oracle.quantize_many(x, np.full(400, b, np.uint8))
    xf = x.astype(np.float32)
    for j in range(400):
        assert z[j] == xf[j].min()                       # z = min(x) exactly
        assert codes[j][np.argmin(xf[j])] == 0           # min -> code 0
        assert codes[j][np.argmax(xf[j])] == top         # max -> code 2^b - 1
        assert codes[j].max() <= top


@pytest.mark.parametrize("b", [2, 4, 8])
def test_error_bound(b):
    # |Q_b(x) - x| <= s/2, plus the fp32 rounding of s, of x - z and of the quotient
    rng = np.random.default_rng(200 + b)
    x = _rand_vectors(rng, 300, 128, scale=rng.uniform(0.1, 10))
    x[:, 5] *= 8  # an outlier channel widens the range
    for j in range(300):
        codes, s, z = oracle.quantize(x[j], b)
        deq = oracle.dequantize(codes, b, s, z)
        xf = x[j].astype(np.float64)
        rng_ = float(xf.max() - xf.min())
        slack = 4 * 2.0 ** -24 * max(abs(xf).max(), abs(float(z)), rng_)
        assert np.all(np.abs(deq - xf) <= float(s) / 2 + slack)
        # the minimum is reproduced exactly
        assert deq[np.argmin(xf)] == xf.min()
        # the maximum within two fp32 ulps of the largest magnitude involved
        assert abs(deq[np.argmax(xf)] - xf.max()) <= 2 * np.spacing(np.float32(max(abs(xf).max(), rng_)))


def test_constant_vector_exact():
    for b in (2, 4, 8):
        for val in (0.0, -3.25, 1000.0, 6e-5):
            x = np.full(64, val, dtype=np.float16)
            codes, s, z = oracle.quantize(x, b)
            assert s == 0 and np.all(codes == 0)
            assert np.all(oracle.dequantize(codes, b, s, z) == x.astype(np.float64))


def test_b16_round_trip_exact():
    rng = np.random.default_rng(3)
    bits = rng.integers(0, 65536, size=4096).astype(np.uint16)
    finite = np.isfinite(bits.view(np.float16))
    bits = bits[finite][:4000]
    codes, s, z = oracle.quantize(bits, 16)
    assert np.array_equal(codes, bits)
    assert s == 1.0 and z == 0.0
    deq = oracle.dequantize(codes, 16, s, z)
    assert np.array_equal(deq, bits.view(np.float16).astype(np.float64))


def test_more_bits_never_worse_on_average():
    # monotonicity the width axis is built on: mean |error| shrinks as b grows
    rng = np.random.default_rng(11)
    x = _rand_vectors(rng, 200, 128)
    errs = []
    for b in (2, 4, 8, 16):
        codes, s, z = oracle.quantize_many(x, np.full(200, b, np.uint8))
        e = 0.0
        for j in range(200):
            e += np.abs(oracle.dequantize(codes[j], b, s[j], z[j]) - x[j].astype(np.float64)).mean()
        errs.append(e)
    assert errs[0] > errs[1] > errs[2] > errs[3] == 0.0


def test_rejects_bad_width():
    with pytest.raises(ValueError):
        oracle.quantize(np.zeros(8, np.float16), 3)


def test_signed_zero_stored_as_plus_zero():
    # -0 and +0 are one value; whichever the min scan meets first, z and s are stored as +0
    for x in ([-0.0, 0.0, 0.0], [0.0, -0.0], [-0.0, -0.0], [-0.0, 1.0, 0.0]):
        codes, s, z = oracle.quantize(np.array(x, np.float16), 4)
        assert np.float32(z).view(np.uint32) == 0
        if max(x) == 0.0:
            assert np.float32(s).view(np.uint32) == 0 and np.all(codes == 0)
