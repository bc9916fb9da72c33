"""GPU parity of the fused decode step (kvq_decode_step: the step's tokens are written at
their widths, Eq. 4, then every query attends over the cache that holds them, Eq. 2, in
three launches), over several consecutive steps: the stored records stay bit-exact with
the oracle and every step's outputs match the oracle at t = len - 1. Also: roll-back to
explicit positions re-decodes a step exactly, and grouped-query caches."""
import numpy as np
import pytest
import torch

from mixed_precision_kv_write_b200 import kvq, synth
from kvq_testlib import assert_close_attn, check_records, oracle_decode

pytestmark = pytest.mark.gpu
W = synth.WORKLOADS


def _rows(cu, s, lo, hi):
    return list(range(cu[s] + lo, cu[s] + hi))


@pytest.mark.parametrize("D,group,w", [(128, 1, 40), (64, 1, 7), (128, 4, 300)])
def test_decode_steps_match_oracle(D, group, w):
    base = W["decode_1p3b"] if D == 128 else W["prefill_160m"]
    wl = synth.scaled(base, seqlens=(300, 77, 4, 700), heads=2)      # final lengths
    k, v, bits = synth.kv_tokens(wl, "cuda")
    cu = synth.cu_seqlens(wl.seqlens).tolist()
    n_steps = 4
    B, H, HQ = wl.batch, wl.heads, wl.heads * group
    cache = kvq.KVQCache(B, H, D, list(wl.seqlens), query_group=group)
    # prompt: all but the last n_steps tokens of each sequence
    pre = [L - n_steps for L in wl.seqlens]
    idx = torch.tensor(sum((_rows(cu, s, 0, pre[s]) for s in range(B)), []), device="cuda")
    kvq.kvq_write(k[idx].contiguous(), v[idx].contiguous(), bits[idx].contiguous(),
                  synth.cu_seqlens(pre, "cuda"), cache)
    kc, vc, bc = k.cpu(), v.cpu(), bits.cpu()
    g = torch.Generator(device="cuda").manual_seed(D + w + group)
    for step in range(n_steps):
        rows = torch.tensor([cu[s] + pre[s] + step for s in range(B)], device="cuda")
        q = torch.randn((B, HQ, D), generator=g, device="cuda").half()
        modes = torch.randint(0, 3, (B, HQ), generator=g, device="cuda").to(torch.uint8)
        out = kvq.decode_step(q, k[rows].contiguous(), v[rows].contiguous(), bits[rows].contiguous(),
                              synth.cu_seqlens([1] * B, "cuda"), cache, modes, w)
        cache.check()
        out = out.cpu().numpy()
        qc, mc = q.cpu(), modes.cpu()
        for s in range(B):
            L = pre[s] + step + 1
            for hq in range(HQ):
                hk = hq // group
                ref = oracle_decode(wl, kc, vc, bc, _q_as_kv_heads(qc, hq, H), mc[:, hq:hq + 1].repeat(1, H),
                                    w, s, hk, L=L)
                assert_close_attn(out[s, hq], ref, f"step {step} s={s} hq={hq} mode={int(mc[s, hq])}")
            assert np.all(out[s][mc[s].numpy() == 0] == 0)
    assert cache.lengths().tolist() == list(wl.seqlens)
    check_records(cache, wl, kc, vc, bc, [(s, h) for s in range(B) for h in range(H)])


def _q_as_kv_heads(qc, hq, H):
    """The query of query head hq placed at every KV head position (the oracle helper
    indexes q by KV head)."""
    return qc[:, hq:hq + 1].repeat(1, H, 1)


def test_decode_step_rollback_redecodes_exactly():
    wl = synth.scaled(W["decode_1p3b"], seqlens=(500, 60, 1300), heads=3)
    k, v, bits = synth.kv_tokens(wl, "cuda")
    B = wl.batch
    cu = synth.cu_seqlens(wl.seqlens).tolist()
    cache = kvq.KVQCache(B, 3, 128, list(wl.seqlens))
    pre = [L - 1 for L in wl.seqlens]
    idx = torch.tensor(sum((_rows(cu, s, 0, pre[s]) for s in range(B)), []), device="cuda")
    kvq.kvq_write(k[idx].contiguous(), v[idx].contiguous(), bits[idx].contiguous(),
                  synth.cu_seqlens(pre, "cuda"), cache)
    rows = torch.tensor([cu[s] + pre[s] for s in range(B)], device="cuda")
    q, modes = synth.decode_queries(wl, "cuda")
    one = synth.cu_seqlens([1] * B, "cuda")
    pos = torch.tensor(pre, dtype=torch.int32, device="cuda")
    first = kvq.decode_step(q, k[rows].contiguous(), v[rows].contiguous(), bits[rows].contiguous(), one,
                            cache, modes, 100)
    outs = []
    for _ in range(3):          # roll back to the same position and decode the step again
        outs.append(kvq.decode_step(q, k[rows].contiguous(), v[rows].contiguous(), bits[rows].contiguous(),
                                    one, cache, modes, 100, positions=pos))
    cache.check()
    for o in outs:
        assert torch.equal(o, first)
    assert cache.lengths().tolist() == list(wl.seqlens)
    # the same step through the separate calls gives the same result
    cache.truncate(pos)
    kvq.kvq_write(k[rows].contiguous(), v[rows].contiguous(), bits[rows].contiguous(), one, cache)
    sep = kvq.routed_attn_decode(q, cache, modes, 100)
    cache.check()
    assert torch.equal(sep, first)
    for s in range(B):
        for h in range(3):
            ref = oracle_decode(wl, k.cpu(), v.cpu(), bits.cpu(), q.cpu(), modes.cpu(), 100, s, h)
            assert_close_attn(first[s, h].cpu().numpy(), ref, f"s={s} h={h}")


def test_decode_entry_points_interleaved():
    # the three decode entry points alternate on one cache (the work-list counters of the
    # cache and of the allocation-free scratch flip between two words per call): every call
    # over the same cache state gives the same outputs
    wl = synth.scaled(W["decode_1p3b"], seqlens=(900, 33, 2100, 1), heads=2)
    k, v, bits = synth.kv_tokens(wl, "cuda")
    B = wl.batch
    cu = synth.cu_seqlens(wl.seqlens).tolist()
    cache = kvq.KVQCache(B, 2, 128, list(wl.seqlens))
    pre = [L - 1 for L in wl.seqlens]
    idx = torch.tensor(sum((_rows(cu, s, 0, pre[s]) for s in range(B)), []), device="cuda")
    kvq.kvq_write(k[idx].contiguous(), v[idx].contiguous(), bits[idx].contiguous(),
                  synth.cu_seqlens(pre, "cuda"), cache)
    rows = torch.tensor([cu[s] + pre[s] for s in range(B)], device="cuda")
    q, modes = synth.decode_queries(wl, "cuda")
    one = synth.cu_seqlens([1] * B, "cuda")
    pos = torch.tensor(pre, dtype=torch.int32, device="cuda")
    kr, vr, br = k[rows].contiguous(), v[rows].contiguous(), bits[rows].contiguous()
    first = kvq.decode_step(q, kr, vr, br, one, cache, modes, 64)
    outs = []
    for i in range(7):
        which = i % 3
        if which == 0:
            outs.append(kvq.routed_attn_decode(q, cache, modes, 64))
        elif which == 1:
            outs.append(kvq.routed_attn_decode_noalloc(q, cache, modes, 64).clone())
        else:
            outs.append(kvq.decode_step(q, kr, vr, br, one, cache, modes, 64, positions=pos))
        torch.cuda.synchronize()
        cache.check()
    for i, o in enumerate(outs):
        assert torch.equal(o, first), f"call {i}"
    for s in range(B):
        for h in range(2):
            ref = oracle_decode(wl, k.cpu(), v.cpu(), bits.cpu(), q.cpu(), modes.cpu(), 64, s, h)
            assert_close_attn(first[s, h].cpu().numpy(), ref, f"s={s} h={h}")
