"""GPU parity of grouped-query attention (the pages' models share each KV head among a group
of query heads, H_kv = H/4): a cache of H_kv KV heads created with query_group G serves
H_kv * G query heads; query head hq reads KV head hq // G under its own mode. The oracle is
the per-head Eq. 2 oracle applied to the query head's query and its KV head's cache."""
import numpy as np
import pytest
import torch

import oracle
from mixed_precision_kv_write_b200 import kvq, synth
from kvq_testlib import assert_close_attn

pytestmark = pytest.mark.gpu
W = synth.WORKLOADS
G = 4


def _ref(wl, kc, vc, bc, q_rows, pos, modes, w, s, hk):
    cu = synth.cu_seqlens(wl.seqlens).tolist()
    rows = slice(cu[s], cu[s] + wl.seqlens[s])
    return oracle.routed_attention_head(q_rows, pos, modes, w, kc[rows, hk].contiguous().numpy(),
                                        vc[rows, hk].contiguous().numpy(), bc[rows, hk].numpy())


@pytest.mark.parametrize("D,w", [(128, 33), (64, 0), (128, 5000)])
def test_gqa_decode(D, w):
    base = W["decode_1p3b"] if D == 128 else W["prefill_160m"]
    wl = synth.scaled(base, seqlens=(1, 300, 1500, 64), heads=2)       # 2 KV heads
    k, v, bits = synth.kv_tokens(wl, "cuda")
    cache = kvq.KVQCache(wl.batch, 2, D, list(wl.seqlens), query_group=G)
    kvq.kvq_write(k, v, bits, synth.cu_seqlens(wl.seqlens, "cuda"), cache)
    g = torch.Generator(device="cuda").manual_seed(D + w)
    q = torch.randn((wl.batch, 2 * G, D), generator=g, device="cuda").half()
    modes = torch.randint(0, 3, (wl.batch, 2 * G), generator=g, device="cuda").to(torch.uint8)
    modes[:, 1] = 1
    modes[:, 2] = 2
    out = kvq.routed_attn_decode(q, cache, modes, w)
    cache.check()
    kc, vc, bc, qc, mc = k.cpu(), v.cpu(), bits.cpu(), q.cpu(), modes.cpu()
    for s in range(wl.batch):
        for hq in range(2 * G):
            L = wl.seqlens[s]
            ref = _ref(wl, kc, vc, bc, qc[s, hq][None].numpy(), [L - 1], [int(mc[s, hq])], w, s, hq // G)[0]
            assert_close_attn(out[s, hq].cpu().numpy(), ref, f"s={s} hq={hq} mode={int(mc[s, hq])}")
    # the no-allocation entry point shares the kernels
    out2 = kvq.routed_attn_decode_noalloc(q, cache, modes, w)
    torch.cuda.synchronize()
    assert torch.equal(out, out2)


@pytest.mark.parametrize("D,w", [(128, 40), (64, 300)])
def test_gqa_prefill(D, w):
    base = W["ragged_prefill"] if D == 128 else W["prefill_160m"]
    wl = synth.scaled(base, seqlens=(130, 1, 257), heads=2)
    k, v, bits = synth.kv_tokens(wl, "cuda")
    cache = kvq.KVQCache(wl.batch, 2, D, list(wl.seqlens), query_group=G)
    cu = synth.cu_seqlens(wl.seqlens, "cuda")
    kvq.kvq_write(k, v, bits, cu, cache)
    wq = synth.scaled(wl, heads=2 * G)
    q, modes = synth.prefill_queries(wq, "cuda")
    out = kvq.routed_attn_prefill(q, cache, modes, w, cu)
    cache.check()
    kc, vc, bc, qc, mc = k.cpu(), v.cpu(), bits.cpu(), q.cpu(), modes.cpu()
    cul = synth.cu_seqlens(wl.seqlens).tolist()
    for s in range(wl.batch):
        L = wl.seqlens[s]
        for hq in range(2 * G):
            rows = slice(cul[s], cul[s] + L)
            ref = _ref(wl, kc, vc, bc, qc[rows, hq].contiguous().numpy(), np.arange(L),
                       mc[rows, hq].numpy(), w, s, hq // G)
            assert_close_attn(out[rows, hq].cpu().numpy(), ref, f"s={s} hq={hq}")


def test_gqa_group_one_matches_mha():
    wl = synth.scaled(W["decode_1p3b"], seqlens=(200, 77), heads=3)
    k, v, bits = synth.kv_tokens(wl, "cuda")
    cu = synth.cu_seqlens(wl.seqlens, "cuda")
    a = kvq.KVQCache(wl.batch, 3, 128, list(wl.seqlens))
    b = kvq.KVQCache(wl.batch, 3, 128, list(wl.seqlens), query_group=1)
    kvq.kvq_write(k, v, bits, cu, a)
    kvq.kvq_write(k, v, bits, cu, b)
    q, modes = synth.decode_queries(wl, "cuda")
    assert torch.equal(kvq.routed_attn_decode(q, a, modes, 64), kvq.routed_attn_decode(q, b, modes, 64))
