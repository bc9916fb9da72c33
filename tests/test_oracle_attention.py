"""Pins for the oracle's routed attention (TriRoute paper review page, section 3, Eq. 2).

Independent anchors: hand-worked closed forms (tests/golden), PyTorch's fp64
scaled_dot_product_attention as the textbook special case (all b = 16, all full -> causal
softmax attention), masked SDPA over the separately pinned codec's dequantized cache,
and invariants (skip -> 0, local with w >= t equals full, t = 0 returns deq(v_0),
permuting keys inside the window changes nothing).
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle


def _golden(golden_dir):
    with open(os.path.join(golden_dir, "attention_worked_examples.json")) as f:
        return json.load(f)


def test_two_key_closed_form(golden_dir):
    g = _golden(golden_dir)["two_key"]
    k = np.array(g["k"], np.float16)
    v = np.array(g["v"], np.float16)
    bits = np.full(2, 16, np.uint8)
    p1 = 1.0 / (1.0 + math.exp(-math.sqrt(2.0)))
    assert g["queries"][0]["out"][1] == pytest.approx(p1, abs=1e-15)
    for qq in g["queries"]:
        out = oracle.routed_attention_head(np.array([g["q"]], np.float16), [qq["t"]],
                                           [qq["mode"]], qq["w"], k, v, bits)
        np.testing.assert_allclose(out[0], qq["out"], rtol=0, atol=1e-7)


def test_window_endpoints(golden_dir):
    g = _golden(golden_dir)["window"]
    L, D = g["L"], g["D"]
    k = np.zeros((L, D), np.float16)
    v = np.stack([np.arange(L), np.ones(L)], axis=1).astype(np.float16)
    bits = np.full(L, 16, np.uint8)
    for qq in g["queries"]:
        out = oracle.routed_attention_head(np.ones((1, D), np.float16), [qq["t"]], [qq["mode"]],
                                           qq["w"], k, v, bits)
        np.testing.assert_allclose(out[0], qq["out"], rtol=0, atol=1e-6)


def _sdpa64(q, k, v, mask):
    """fp64 torch SDPA; q [n, D], k/v [L, D], boolean mask [n, L] (True = attend)."""
    Q = torch.from_numpy(q.astype(np.float64))[None, None]
    K = torch.from_numpy(k.astype(np.float64))[None, None]
    V = torch.from_numpy(v.astype(np.float64))[None, None]
    M = torch.from_numpy(mask)[None, None]
    return torch.nn.functional.scaled_dot_product_attention(Q, K, V, attn_mask=M)[0, 0].numpy()


@pytest.mark.parametrize("D", [8, 64, 128])
def test_native_full_equals_textbook_causal(D):
    rng = np.random.default_rng(D)
    L = 40
    q = rng.standard_normal((L, D)).astype(np.float16)
    k = rng.standard_normal((L, D)).astype(np.float16)
    v = rng.standard_normal((L, D)).astype(np.float16)
    out = oracle.routed_attention_head(q, np.arange(L), np.full(L, 2), 0, k, v, np.full(L, 16))
    Q = torch.from_numpy(q.astype(np.float64))[None, None]
    K = torch.from_numpy(k.astype(np.float64))[None, None]
    V = torch.from_numpy(v.astype(np.float64))[None, None]
    ref = torch.nn.functional.scaled_dot_product_attention(Q, K, V, is_causal=True)[0, 0].numpy()
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-6)


@pytest.mark.parametrize("w", [0, 3, 17, 100])
def test_quantized_cache_equals_masked_sdpa_over_dequantized(w):
    # the attention reads the Eq. 4 reconstruction; the codec is pinned separately
    rng = np.random.default_rng(50 + w)
    L, D = 48, 32
    k = (rng.standard_normal((L, D)) * 2).astype(np.float16)
    v = (rng.standard_normal((L, D)) * 2).astype(np.float16)
    q = rng.standard_normal((L, D)).astype(np.float16)
    bits = rng.choice([2, 4, 8, 16], size=L).astype(np.uint8)
    modes = rng.choice([0, 1, 2], size=L).astype(np.uint8)
    kd = np.zeros((L, D))
    vd = np.zeros((L, D))
    for j in range(L):
        c, s, z = oracle.quantize(k[j], bits[j])
        kd[j] = oracle.dequantize(c, bits[j], s, z)
        c, s, z = oracle.quantize(v[j], bits[j])
        vd[j] = oracle.dequantize(c, bits[j], s, z)
    mask = np.zeros((L, L), bool)
    for t in range(L):
        if modes[t] == 2:
            mask[t, : t + 1] = True
        elif modes[t] == 1:
            mask[t, max(0, t - w): t + 1] = True
        else:
            mask[t, t] = True  # placeholder row; skip rows are checked for zeros below
    ref = _sdpa64(q, kd, vd, mask)
    out = oracle.routed_attention_head(q, np.arange(L), modes, w, k, v, bits)
    for t in range(L):
        if modes[t] == 0:
            assert np.all(out[t] == 0.0)
        else:
            np.testing.assert_allclose(out[t], ref[t], rtol=0, atol=2e-6)


def test_local_with_large_window_equals_full():
    rng = np.random.default_rng(5)
    L, D = 33, 16
    k = rng.standard_normal((L, D)).astype(np.float16)
    v = rng.standard_normal((L, D)).astype(np.float16)
    q = rng.standard_normal((L, D)).astype(np.float16)
    bits = rng.choice([2, 4, 8, 16], size=L)
    t = np.arange(L)
    full = oracle.routed_attention_head(q, t, np.full(L, 2), 0, k, v, bits)
    for w in (L - 1, L, 1000):
        loc = oracle.routed_attention_head(q, t, np.full(L, 1), w, k, v, bits)
        assert np.array_equal(loc, full)
    # and a window smaller than t differs from full for late queries
    loc = oracle.routed_attention_head(q, t, np.full(L, 1), 4, k, v, bits)
    assert np.array_equal(loc[:5], full[:5])
    assert not np.allclose(loc[10:], full[10:])


def test_first_position_returns_its_own_value():
    rng = np.random.default_rng(9)
    D = 64
    for b in (2, 4, 8, 16):
        k = rng.standard_normal((4, D)).astype(np.float16)
        v = rng.standard_normal((4, D)).astype(np.float16)
        q = rng.standard_normal((1, D)).astype(np.float16)
        bits = np.full(4, b)
        for mode in (1, 2):
            out = oracle.routed_attention_head(q, [0], [mode], 7, k, v, bits)
            c, s, z = oracle.quantize(v[0], b)
            np.testing.assert_allclose(out[0], oracle.dequantize(c, b, s, z).astype(np.float32),
                                       rtol=0, atol=0)


def test_skip_is_exact_zero():
    rng = np.random.default_rng(1)
    L, D = 10, 8
    k = rng.standard_normal((L, D)).astype(np.float16)
    out = oracle.routed_attention_head(rng.standard_normal((L, D)).astype(np.float16),
                                       np.arange(L), np.zeros(L), 3, k, k, np.full(L, 4))
    assert np.all(out == 0.0)


def test_key_permutation_inside_window_is_invisible():
    # attention is a function of the key SET: permuting the keys 0..t-1 (with their
    # widths) of a full query leaves its output unchanged up to fp64 summation order
    rng = np.random.default_rng(12)
    L, D = 30, 16
    k = rng.standard_normal((L, D)).astype(np.float16)
    v = rng.standard_normal((L, D)).astype(np.float16)
    bits = rng.choice([2, 4, 8, 16], size=L)
    q = rng.standard_normal((1, D)).astype(np.float16)
    base = oracle.routed_attention_head(q, [L - 1], [2], 0, k, v, bits)
    perm = np.concatenate([rng.permutation(L - 1), [L - 1]])
    out = oracle.routed_attention_head(q, [L - 1], [2], 0, k[perm], v[perm], bits[perm])
    np.testing.assert_allclose(out, base, rtol=0, atol=1e-6)


def test_rejects_bad_arguments():
    k = np.zeros((4, 8), np.float16)
    with pytest.raises(ValueError):
        oracle.routed_attention_head(np.zeros((1, 8), np.float16), [4], [2], 0, k, k, np.full(4, 16))
    with pytest.raises(ValueError):
        oracle.routed_attention_head(np.zeros((1, 8), np.float16), [1], [3], 0, k, k, np.full(4, 16))
    with pytest.raises(ValueError):
        oracle.routed_attention_head(np.zeros((1, 8), np.float16), [1], [2], 0, k, k, np.full(4, 5))
