"""GPU parity of routed causal prefill attention (Eq. 2 over the Eq. 4 cache) against the
oracle: the whole tiny workload, ragged shapes with several query/key tiles and ragged
tails, chunked prefill (queries after an earlier write), edge cases, and the full prefill
workloads on sampled queries."""
import numpy as np
import pytest
import torch

from mixed_precision_kv_write_b200 import kvq, synth
from kvq_testlib import assert_close_attn, build_cache, check_records, oracle_prefill

pytestmark = pytest.mark.gpu
W = synth.WORKLOADS


def _prefill(wl, w=None, with_cache=False):
    k, v, bits = synth.kv_tokens(wl, "cuda")
    q, modes = synth.prefill_queries(wl, "cuda")
    cache = build_cache(wl, k, v, bits)
    out = kvq.routed_attn_prefill(q, cache, modes, wl.w if w is None else w,
                                  synth.cu_seqlens(wl.seqlens, "cuda"))
    cache.check()
    res = (out.cpu().numpy(), (k.cpu(), v.cpu(), bits.cpu(), q.cpu(), modes.cpu()))
    return res + (cache,) if with_cache else res


def _check_all(wl, out, cpu, w, heads=None, queries=None):
    kc, vc, bc, qc, mc = cpu
    cu = synth.cu_seqlens(wl.seqlens).tolist()
    for s in range(wl.batch):
        for h in (range(wl.heads) if heads is None else heads):
            qi = np.arange(wl.seqlens[s]) if queries is None else queries(s)
            ref = oracle_prefill(wl, kc, vc, bc, qc, mc, w, s, h, qi)
            got = out[cu[s] + qi, h]
            assert_close_attn(got, ref, f"{wl.name} s={s} h={h}")
            skip = mc[cu[s] + qi, h].numpy() == 0
            assert np.all(got[skip] == 0)


def test_prefill_tiny_workload_all_outputs():
    wl = W["tiny_prefill"]
    out, cpu = _prefill(wl)
    _check_all(wl, out, cpu, wl.w)


@pytest.mark.parametrize("name", ["prefill_160m", "ragged_prefill"])
@pytest.mark.parametrize("w", [0, 33, 256, 4000])
def test_prefill_ragged_small(name, w):
    wl = synth.scaled(W[name], seqlens=(1, 130, 257, 31), heads=2)
    out, cpu = _prefill(wl, w)
    _check_all(wl, out, cpu, w)


@pytest.mark.parametrize("bitval", [2, 16])
def test_prefill_single_width_all_full(bitval):
    wl = synth.scaled(W["ragged_prefill"], seqlens=(300,), heads=1)
    k, v, bits = synth.kv_tokens(wl, "cuda")
    bits.fill_(bitval)
    q, modes = synth.prefill_queries(wl, "cuda")
    modes.fill_(2)
    cache = build_cache(wl, k, v, bits)
    out = kvq.routed_attn_prefill(q, cache, modes, 0, synth.cu_seqlens(wl.seqlens, "cuda"))
    cache.check()
    _check_all(wl, out.cpu().numpy(), (k.cpu(), v.cpu(), bits.cpu(), q.cpu(), modes.cpu()), 0)


def test_chunked_prefill_positions():
    # write + prefill the first 150 tokens, then the next 170: queries of the second call
    # sit at positions 150.. and read the keys of both writes
    wl = synth.scaled(W["prefill_160m"], seqlens=(320,), heads=2)
    k, v, bits = synth.kv_tokens(wl, "cuda")
    q, modes = synth.prefill_queries(wl, "cuda")
    cache = kvq.KVQCache(1, 2, wl.head_dim, [320])
    outs = []
    for a, b in ((0, 150), (150, 320)):
        cu = synth.cu_seqlens([b - a], "cuda")
        kvq.kvq_write(k[a:b].contiguous(), v[a:b].contiguous(), bits[a:b].contiguous(), cu, cache)
        outs.append(kvq.routed_attn_prefill(q[a:b].contiguous(), cache, modes[a:b].contiguous(),
                                            wl.w, cu))
    cache.check()
    out = torch.cat(outs).cpu().numpy()
    _check_all(wl, out, (k.cpu(), v.cpu(), bits.cpu(), q.cpu(), modes.cpu()), wl.w)


def test_prefill_all_skip_is_zero():
    wl = synth.scaled(W["tiny_prefill"], seqlens=(70,))
    k, v, bits = synth.kv_tokens(wl, "cuda")
    q, modes = synth.prefill_queries(wl, "cuda")
    modes.zero_()
    cache = build_cache(wl, k, v, bits)
    out = kvq.routed_attn_prefill(q, cache, modes, 4, synth.cu_seqlens(wl.seqlens, "cuda"))
    cache.check()
    assert torch.all(out == 0)


@pytest.mark.parametrize("name,per_seq", [("prefill_160m", 24), ("ragged_prefill", 24)])
def test_prefill_full_size_sampled(name, per_seq):
    # The full workload in one write + one prefill call, as the benchmark runs it: the
    # stored records of every (sequence, head) are checked bit-exactly, and the attention
    # of every head on a sample of each sequence's queries (first, last and per_seq random).
    wl = W[name]
    out, cpu, cache = _prefill(wl, with_cache=True)
    kc, vc, bc = cpu[:3]
    check_records(cache, wl, kc, vc, bc, [(s, h) for s in range(wl.batch) for h in range(wl.heads)])
    rng = np.random.default_rng(3)
    qs = {}

    def queries(s):
        if s not in qs:
            L = wl.seqlens[s]
            qs[s] = np.unique(np.concatenate([[0, L - 1], rng.integers(0, L, per_seq)]))
        return qs[s]

    _check_all(wl, out, cpu, wl.w, queries=queries)
