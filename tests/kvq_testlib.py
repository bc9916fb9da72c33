"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI, run the
oracle on the same bytes, compare."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from mixed_precision_kv_write_b200 import kvq, synth

# Attention tolerance (floating point): max |gpu - oracle| <= 2e-3 and
# ||gpu - oracle||_2 / ||oracle||_2 <= 1e-3, per compared block of outputs.
ATOL = 2e-3
REL_L2 = 1e-3


def assert_close_attn(got: np.ndarray, ref: np.ndarray, what: str = ""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    err = np.abs(got - ref)
    mx = float(err.max()) if err.size else 0.0
    nref = float(np.linalg.norm(ref))
    rel = float(np.linalg.norm(got - ref)) / nref if nref > 0 else float(np.linalg.norm(got))
    assert mx <= ATOL and rel <= REL_L2, f"{what}: max abs err {mx:.3e}, rel L2 {rel:.3e}"
    return mx, rel


def build_cache(wl: synth.Workload, k, v, bits, capacity=None, device="cuda"):
    cap = list(wl.seqlens) if capacity is None else capacity
    cache = kvq.KVQCache(wl.batch, wl.heads, wl.head_dim, cap, device=device)
    cu = synth.cu_seqlens(wl.seqlens, device)
    kvq.kvq_write(k, v, bits, cu, cache)
    return cache


def check_records(cache, wl, k_cpu, v_cpu, bits_cpu, pairs, tok_ranges=None):
    """Codes, scales, zeros and widths of the stored records of (s, h) pairs are
    bit-exact with the oracle's Eq. 4 on the same fp16 inputs."""
    cu = synth.cu_seqlens(wl.seqlens).tolist()
    for (s, h) in pairs:
        L = wl.seqlens[s]
        j0, j1 = (0, L) if tok_ranges is None else tok_ranges
        j1 = min(j1, L)
        if j1 <= j0:
            continue
        kc, vc, sd, bt = cache.export(s, h, j0, j1 - j0)
        torch.cuda.synchronize()
        kc = kc.cpu().numpy().view(np.uint16)
        vc = vc.cpu().numpy().view(np.uint16)
        sd = sd.cpu().numpy()
        bt = bt.cpu().numpy()
        rows = slice(cu[s] + j0, cu[s] + j1)
        kk = k_cpu[rows, h].numpy().view(np.uint16)
        vv = v_cpu[rows, h].numpy().view(np.uint16)
        bb = bits_cpu[rows, h].numpy()
        assert np.array_equal(bt, bb), (s, h)
        ck, sk, zk = oracle.quantize_many(kk, bb)
        cv, sv, zv = oracle.quantize_many(vv, bb)
        assert np.array_equal(kc, ck), f"K codes differ at (s={s}, h={h})"
        assert np.array_equal(vc, cv), f"V codes differ at (s={s}, h={h})"
        for col, ref in ((0, sk), (1, zk), (2, sv), (3, zv)):
            assert np.array_equal(sd[:, col].view(np.uint32), ref.view(np.uint32)), \
                f"side column {col} differs at (s={s}, h={h})"


def check_records_seq(cache, s, heads, ks, vs, bs, what=""):
    """Bit-exact check of every stored record of sequence s for the listed heads, given the
    sequence's own fp16 K/V [L, H, D] and widths [L, H] on the CPU (all L tokens, including
    any written by later short appends)."""
    L = ks.shape[0]
    for h in heads:
        kc, vc, sd, bt = cache.export(s, h, 0, L)
        torch.cuda.synchronize()
        kc = kc.cpu().numpy().view(np.uint16)
        vc = vc.cpu().numpy().view(np.uint16)
        sd = sd.cpu().numpy()
        bb = bs[:, h].numpy()
        assert np.array_equal(bt.cpu().numpy(), bb), f"{what} widths differ at (s={s}, h={h})"
        ck, sk, zk = oracle.quantize_many(ks[:, h].contiguous().numpy().view(np.uint16), bb)
        cv, sv, zv = oracle.quantize_many(vs[:, h].contiguous().numpy().view(np.uint16), bb)
        assert np.array_equal(kc, ck), f"{what} K codes differ at (s={s}, h={h})"
        assert np.array_equal(vc, cv), f"{what} V codes differ at (s={s}, h={h})"
        for col, ref in ((0, sk), (1, zk), (2, sv), (3, zv)):
            assert np.array_equal(sd[:, col].view(np.uint32), ref.view(np.uint32)), \
                f"{what} side column {col} differs at (s={s}, h={h})"


def oracle_decode(wl, k_cpu, v_cpu, bits_cpu, q_cpu, modes_cpu, w, s, h, L=None):
    """Oracle output of the decode query of (s, h) at t = L - 1."""
    cu = synth.cu_seqlens(wl.seqlens).tolist()
    L = wl.seqlens[s] if L is None else L
    rows = slice(cu[s], cu[s] + L)
    return oracle.routed_attention_head(
        q_cpu[s, h][None].numpy(), [L - 1], [int(modes_cpu[s, h])], w,
        k_cpu[rows, h].contiguous().numpy(), v_cpu[rows, h].contiguous().numpy(),
        bits_cpu[rows, h].numpy())[0]


def oracle_prefill(wl, k_cpu, v_cpu, bits_cpu, q_cpu, modes_cpu, w, s, h, queries=None, pos0=0):
    """Oracle outputs of prefill queries (indices within sequence s) of head h."""
    cu = synth.cu_seqlens(wl.seqlens).tolist()
    L = wl.seqlens[s]
    qi = np.arange(L) if queries is None else np.asarray(queries)
    rows = slice(cu[s], cu[s] + L)
    return oracle.routed_attention_head(
        q_cpu[cu[s] + qi, h].contiguous().numpy(), pos0 + qi, modes_cpu[cu[s] + qi, h].numpy(), w,
        k_cpu[rows, h].contiguous().numpy(), v_cpu[rows, h].contiguous().numpy(),
        bits_cpu[rows, h].numpy())
