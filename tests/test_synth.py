"""The seeded generator: deterministic, right shapes, right category frequencies."""
import torch

from mixed_precision_kv_write_b200 import synth


def test_deterministic_and_per_sequence():
    wl = synth.scaled(synth.WORKLOADS["ragged_prefill"], seqlens=(40, 70, 33))
    k1, v1, b1 = synth.kv_tokens(wl, "cpu")
    k2, v2, b2 = synth.kv_tokens(wl, "cpu")
    assert torch.equal(k1, k2) and torch.equal(v1, v2) and torch.equal(b1, b2)
    ks, vs, bs = synth.kv_sequence(wl, 1, "cpu")
    assert torch.equal(ks, k1[40:110]) and torch.equal(bs, b1[40:110])
    assert k1.shape == (143, 16, 128) and k1.dtype == torch.float16
    assert b1.shape == (143, 16) and b1.dtype == torch.uint8


def test_category_frequencies():
    wl = synth.scaled(synth.WORKLOADS["prefill_160m"], seqlens=(4000,))
    _, _, bits = synth.kv_tokens(wl, "cpu")
    for val, p in zip(synth.BIT_VALUES, wl.bits_p):
        assert abs((bits == val).double().mean().item() - p) < 0.01
    _, modes = synth.prefill_queries(wl, "cpu")
    for val, p in enumerate(wl.modes_p):
        assert abs((modes == val).double().mean().item() - p) < 0.01


def test_outlier_channels():
    wl = synth.scaled(synth.WORKLOADS["prefill_160m"], seqlens=(3000,))
    k, _, _ = synth.kv_tokens(wl, "cpu")
    idx = synth.outlier_channels(12, 64, wl.seed, 5)
    assert idx.numel() == 8 and len(set(idx.tolist())) == 8
    std = k.float().reshape(3000, -1).std(0)
    assert torch.all(std[idx] > 6) and (std > 6).sum() == 8


def test_decode_queries_shape():
    wl = synth.WORKLOADS["decode_1p3b"]
    q, modes = synth.decode_queries(wl, "cpu")
    assert q.shape == (64, 16, 128) and modes.shape == (64, 16)
    assert set(modes.unique().tolist()) <= {0, 1, 2}
