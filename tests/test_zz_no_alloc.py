"""The allocation-free decode entry point (routed_attn_decode_noalloc).

Some callers cannot allocate device memory at the point of a call (their allocations are
owned by a host framework's pool, or an allocation's implicit synchronization is not
allowed there). For them the library offers a decode variant whose scratch lives in its
own static device array. These checks call it through the C ABI and compare it with the
ordinary routed_attn_decode on the same inputs, on two calls in a row (the shared scratch
keeps the previous call's contents), and check that an oversized cache is rejected.
This file is named so that pytest collects it last.
"""
import numpy as np
import pytest
import torch

from mixed_precision_kv_write_b200 import kvq, synth
from kvq_testlib import assert_close_attn, build_cache

pytestmark = pytest.mark.gpu


def _case(seed):
    wl = synth.scaled(synth.WORKLOADS["decode_1p3b"], seqlens=(700, 64, 1, 1500, 513), heads=4)
    k, v, bits = synth.kv_tokens(wl, "cuda")
    cache = build_cache(wl, k, v, bits)
    g = torch.Generator(device="cuda").manual_seed(seed)
    q = torch.randn((wl.batch, 4, 128), generator=g, device="cuda").half()
    modes = torch.randint(0, 3, (wl.batch, 4), generator=g, device="cuda").to(torch.uint8)
    return cache, q, modes, wl.w


def test_noalloc_matches_decode_on_two_calls_in_a_row():
    cache, q, modes, w = _case(11)
    ref = kvq.routed_attn_decode(q, cache, modes, w).cpu().numpy()
    out = torch.empty_like(torch.from_numpy(ref)).cuda()
    for _ in range(2):
        out.fill_(float("nan"))
        kvq.routed_attn_decode_noalloc(q, cache, modes, w, out=out)
        cache.check()
        assert_close_attn(out.cpu().numpy(), ref, "noalloc vs decode")
    # a second cache and other queries right after: the shared scratch is fully rewritten
    cache2, q2, modes2, w2 = _case(12)
    ref2 = kvq.routed_attn_decode(q2, cache2, modes2, w2).cpu().numpy()
    got2 = kvq.routed_attn_decode_noalloc(q2, cache2, modes2, w2).cpu().numpy()
    assert_close_attn(got2, ref2, "noalloc vs decode, second cache")
    assert np.all(got2[modes2.cpu().numpy() == 0] == 0)


@pytest.mark.parametrize("D,group", [(64, 1), (128, 4), (64, 4)])
def test_noalloc_other_shapes_larger_then_smaller(D, group):
    # The scratch layout depends on the number of query heads (work-list head tables) and
    # on head_dim (partials stride). A call on a larger cache, then one on a smaller cache
    # of another shape, each matches routed_attn_decode on its own cache.
    base = synth.WORKLOADS["decode_1p3b"] if D == 128 else synth.WORKLOADS["prefill_160m"]
    results = []
    for seqlens, hk in (((1500, 700, 64, 2000, 9, 513), 4), ((300, 1), 2)):
        wl = synth.scaled(base, seqlens=seqlens, heads=hk)
        k, v, bits = synth.kv_tokens(wl, "cuda")
        cache = kvq.KVQCache(wl.batch, hk, D, list(wl.seqlens), query_group=group)
        kvq.kvq_write(k, v, bits, synth.cu_seqlens(wl.seqlens, "cuda"), cache)
        g = torch.Generator(device="cuda").manual_seed(D + group + hk)
        hq = hk * group
        q = torch.randn((wl.batch, hq, D), generator=g, device="cuda").half()
        modes = torch.randint(0, 3, (wl.batch, hq), generator=g, device="cuda").to(torch.uint8)
        ref = kvq.routed_attn_decode(q, cache, modes, 77).cpu().numpy()
        got = kvq.routed_attn_decode_noalloc(q, cache, modes, 77).cpu().numpy()
        cache.check()
        assert_close_attn(got, ref, f"noalloc D={D} G={group} heads={hk}")
        assert np.all(got[modes.cpu().numpy() == 0] == 0)
        results.append(got.shape)
    assert results[0] != results[1]


def test_noalloc_rejects_caches_beyond_the_static_scratch():
    # 64 x 1024 heads: its worst-case work list needs more than the 16 MiB of static scratch
    cache = kvq.KVQCache(64, 1024, 64, [1] * 64)
    q = torch.zeros((64, 1024, 64), dtype=torch.float16, device="cuda")
    modes = torch.zeros((64, 1024), dtype=torch.uint8, device="cuda")
    with pytest.raises(kvq.KVQError) as e:
        kvq.routed_attn_decode_noalloc(q, cache, modes, 4)
    assert e.value.code == kvq.KVQ_ERR_ARG and "static scratch" in str(e.value)
