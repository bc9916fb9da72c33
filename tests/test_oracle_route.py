"""Pins of the oracle's inference-time router (section 3 item 5, Eq. 5: attention head
z^a over {skip, local, full}, bit head z^b over the widths {2, 4, 8, 16}; at inference
the router takes the hard argmax). Reading: fp32 logits compared as given, the first
index wins a tie, NaN entries are passed over (a row of NaNs gives index 0)."""
import numpy as np
import pytest

import oracle


def test_worked_example():
    # by hand: row maxima at index 1, 2, 0 (tie 0/1 -> 0), 1 (NaN at 0 passed over), 0 (all NaN)
    za = np.array([[0.1, 2.0, -1.0],
                   [-3.0, -2.5, -2.0],
                   [4.0, 4.0, 1.0],
                   [np.nan, 0.5, 0.25],
                   [np.nan, np.nan, np.nan]], np.float32)
    zb = np.array([[1.0, 0.0, 0.0, 0.0],       # b = 2
                   [0.0, 1.0, 0.0, 0.0],       # b = 4
                   [-1.0, -1.0, 7.0, 7.0],     # tie 2/3 -> b = 8
                   [0.0, 0.0, 0.0, 1e-30],     # b = 16
                   [-np.inf, -np.inf, -np.inf, -np.inf]], np.float32)   # all equal -> b = 2
    modes, bits = oracle.route_argmax(za, zb)
    assert modes.tolist() == [1, 2, 0, 1, 0]
    assert bits.tolist() == [2, 4, 8, 16, 2]


def test_matches_library_argmax_without_nan():
    rng = np.random.default_rng(7)
    for k in (3, 4):
        z = rng.standard_normal((5000, k)).astype(np.float32)
        z[::7] = np.round(z[::7] * 2) / 2          # plenty of ties
        got = oracle.route_argmax(z if k == 3 else None, z if k == 4 else None)[0 if k == 3 else 1]
        want = np.argmax(z, axis=1)
        if k == 4:
            want = np.array([2, 4, 8, 16], np.uint8)[want]
        assert np.array_equal(got, want)


def test_invariances():
    rng = np.random.default_rng(8)
    z = rng.standard_normal((2000, 4)).astype(np.float32)
    _, b0 = oracle.route_argmax(None, z)
    # scaling by a positive power of two is exact in fp32, so every row keeps its order
    for f in (4.0, 0.5):
        _, b1 = oracle.route_argmax(None, (z * f).astype(np.float32))
        assert np.array_equal(b0, b1)
    # negating every logit turns the maximum into the minimum
    _, bn = oracle.route_argmax(None, -z)
    assert np.array_equal(np.array([2, 4, 8, 16], np.uint8)[np.argmin(z, axis=1)], bn)
    # permuting the entries of a row moves the winner with them
    perm = np.array([2, 0, 3, 1])
    _, bp = oracle.route_argmax(None, z[:, perm])
    widths = np.array([2, 4, 8, 16])
    idx0 = np.searchsorted(widths, b0)
    idxp = np.searchsorted(widths, bp)
    assert np.array_equal(perm[idxp], idx0)


def test_shape_errors():
    with pytest.raises(ValueError):
        oracle.route_argmax(np.zeros((4, 4), np.float32), None)
    with pytest.raises(ValueError):
        oracle.route_argmax(None, np.zeros((4, 3), np.float32))
