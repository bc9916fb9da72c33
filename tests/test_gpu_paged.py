"""GPU parity of the paged mixed-precision cache (kvq_cache_create_paged): fixed-size pages
from a pool hold the variable-width records, each (sequence, KV head) stream is a page
table, and the pool hands pages out in a scrambled order so that pages of different
streams interleave. Stored records stay bit-exact with the oracle, attention matches the
oracle (and prefill matches the contiguous cache exactly), pool exhaustion is refused
with KVQ_ERR_CAPACITY, and a reset returns every page."""
import numpy as np
import pytest
import torch

from mixed_precision_kv_write_b200 import kvq, synth
from kvq_testlib import assert_close_attn, check_records, oracle_decode, oracle_prefill

pytestmark = pytest.mark.gpu
W = synth.WORKLOADS
PAGE = 4096


def _pages_needed(wl, bits, page=PAGE):
    cu = synth.cu_seqlens(wl.seqlens).tolist()
    b = bits.cpu().to(torch.int64)
    n = 0
    for s in range(wl.batch):
        per = (b[cu[s]:cu[s + 1]] * wl.head_dim // 4).sum(0)          # stream bytes per head
        n += int(((per + page - 1) // page).sum())
    return n


def _paged(wl, bits, extra=0, group=1, page=PAGE):
    return kvq.KVQCache(wl.batch, wl.heads, wl.head_dim, [max(1, L) for L in wl.seqlens], query_group=group,
                        page_bytes=page, pool_pages=_pages_needed(wl, bits, page) + extra)


@pytest.mark.parametrize("name", ["ragged_prefill", "prefill_160m"])
def test_paged_writes_bit_exact(name):
    # one long write, chunked writes and short (single-launch) appends, all through pages
    wl = synth.scaled(W[name], seqlens=(1024, 300, 17, 777, 0), heads=3)
    k, v, bits = synth.kv_tokens(wl, "cuda")
    cu = synth.cu_seqlens(wl.seqlens).tolist()
    cache = _paged(wl, bits, extra=8)
    pos = [0] * wl.batch
    rng = np.random.default_rng(5)
    while any(pos[s] < wl.seqlens[s] for s in range(wl.batch)):
        big = rng.random() < 0.3
        counts = [int(min(rng.integers(0, 400) if big else rng.integers(0, 3), wl.seqlens[s] - pos[s]))
                  for s in range(wl.batch)]
        rows = [cu[s] + pos[s] + i for s in range(wl.batch) for i in range(counts[s])]
        idx = torch.tensor(rows, dtype=torch.long, device="cuda")
        kvq.kvq_write(k[idx].contiguous(), v[idx].contiguous(), bits[idx].contiguous(),
                      synth.cu_seqlens(counts, "cuda"), cache)
        pos = [p + c for p, c in zip(pos, counts)]
    cache.check()
    assert cache.lengths().tolist() == list(wl.seqlens)
    check_records(cache, wl, k.cpu(), v.cpu(), bits.cpu(), [(s, h) for s in range(wl.batch) for h in range(3)])


@pytest.mark.parametrize("D", [128, 64])
def test_paged_prefill_equals_contiguous_and_decode_matches_oracle(D):
    base = W["ragged_prefill"] if D == 128 else W["prefill_160m"]
    wl = synth.scaled(base, seqlens=(900, 1, 2500, 333), heads=2)
    k, v, bits = synth.kv_tokens(wl, "cuda")
    q, modes = synth.prefill_queries(wl, "cuda")
    cu = synth.cu_seqlens(wl.seqlens, "cuda")
    flat = kvq.KVQCache(wl.batch, 2, D, list(wl.seqlens))
    paged = _paged(wl, bits)
    outs = []
    for c in (flat, paged):
        kvq.kvq_write(k, v, bits, cu, c)
        outs.append(kvq.routed_attn_prefill(q, c, modes, 200, cu))
        c.check()
    assert torch.equal(outs[0], outs[1])
    kc, vc, bc, qc, mc = k.cpu(), v.cpu(), bits.cpu(), q.cpu(), modes.cpu()
    got = outs[1].cpu().numpy()
    cul = synth.cu_seqlens(wl.seqlens).tolist()
    rng = np.random.default_rng(2)
    for s in range(wl.batch):
        L = wl.seqlens[s]
        qi = np.unique(np.concatenate([[0, L - 1], rng.integers(0, L, 20)]))
        for h in range(2):
            ref = oracle_prefill(wl, kc, vc, bc, qc, mc, 200, s, h, qi)
            assert_close_attn(got[cul[s] + qi, h], ref, f"paged prefill s={s} h={h}")
    # decode over the same paged cache (stages cut where records cross pages)
    g = torch.Generator(device="cuda").manual_seed(D)
    qd = torch.randn((wl.batch, 2, D), generator=g, device="cuda").half()
    md = torch.randint(0, 3, (wl.batch, 2), generator=g, device="cuda").to(torch.uint8)
    md[:, 0] = 2
    od = kvq.routed_attn_decode(qd, paged, md, 600).cpu().numpy()
    paged.check()
    for s in range(wl.batch):
        for h in range(2):
            ref = oracle_decode(wl, kc, vc, bc, qd.cpu(), md.cpu(), 600, s, h)
            assert_close_attn(od[s, h], ref, f"paged decode s={s} h={h} mode={int(md[s, h])}")


def test_paged_gqa_decode_steps():
    # grouped-query cache, fused decode steps with a roll-back, 8 KiB pages
    wl = synth.scaled(W["decode_1p3b"], seqlens=(1500, 64, 700), heads=2)
    k, v, bits = synth.kv_tokens(wl, "cuda")
    cu = synth.cu_seqlens(wl.seqlens).tolist()
    G, B = 4, wl.batch
    cache = _paged(wl, bits, group=G, page=8192)
    pre = [L - 2 for L in wl.seqlens]
    idx = torch.tensor([cu[s] + i for s in range(B) for i in range(pre[s])], device="cuda")
    kvq.kvq_write(k[idx].contiguous(), v[idx].contiguous(), bits[idx].contiguous(), synth.cu_seqlens(pre, "cuda"),
                  cache)
    kc, vc, bc = k.cpu(), v.cpu(), bits.cpu()
    g = torch.Generator(device="cuda").manual_seed(9)
    one = synth.cu_seqlens([1] * B, "cuda")
    for step in range(2):
        rows = torch.tensor([cu[s] + pre[s] + step for s in range(B)], device="cuda")
        q = torch.randn((B, 2 * G, 128), generator=g, device="cuda").half()
        modes = torch.randint(0, 3, (B, 2 * G), generator=g, device="cuda").to(torch.uint8)
        out = kvq.decode_step(q, k[rows].contiguous(), v[rows].contiguous(), bits[rows].contiguous(), one, cache,
                              modes, 100)
        if step == 1:      # decode the same step again after rolling back to its position
            pos = torch.tensor([pre[s] + 1 for s in range(B)], dtype=torch.int32, device="cuda")
            again = kvq.decode_step(q, k[rows].contiguous(), v[rows].contiguous(), bits[rows].contiguous(), one,
                                    cache, modes, 100, positions=pos)
            assert torch.equal(again, out)
        cache.check()
        out = out.cpu().numpy()
        for s in range(B):
            L = pre[s] + step + 1
            for hq in range(2 * G):
                qq = q.cpu()[:, hq:hq + 1].repeat(1, 2, 1)
                mm = modes.cpu()[:, hq:hq + 1].repeat(1, 2)
                ref = oracle_decode(wl, kc, vc, bc, qq, mm, 100, s, hq // G, L=L)
                assert_close_attn(out[s, hq], ref, f"paged gqa step {step} s={s} hq={hq}")
    check_records(cache, synth.scaled(wl, seqlens=[p + 2 for p in pre]), kc, vc, bc,
                  [(s, h) for s in range(B) for h in range(2)])


def test_paged_pool_exhaustion_and_reset():
    wl = synth.scaled(W["ragged_prefill"], seqlens=(2000, 2000), heads=2)
    k, v, bits = synth.kv_tokens(wl, "cuda")
    need = _pages_needed(wl, bits)
    cache = kvq.KVQCache(wl.batch, 2, 128, list(wl.seqlens), page_bytes=PAGE, pool_pages=need - 3)
    cu = synth.cu_seqlens(wl.seqlens, "cuda")
    kvq.kvq_write(k, v, bits, cu, cache)
    with pytest.raises(kvq.KVQError) as e:
        cache.check()
    assert e.value.code == kvq.KVQ_ERR_CAPACITY
    # at least one head was refused: it holds no tokens, the accepted ones are exact
    cache.reset()
    # after a reset every page is free again: the first sequence alone fits
    one = synth.scaled(wl, seqlens=(2000,))
    k1, v1, b1 = synth.kv_sequence(wl, 0, "cuda")
    kvq.kvq_write(k1, v1, b1, synth.cu_seqlens([2000, 0], "cuda"), cache)
    cache.check()
    assert cache.lengths().tolist() == [2000, 0]
    check_records(cache, one, k1.cpu(), v1.cpu(), b1.cpu(), [(0, 0), (0, 1)])


def test_paged_create_rejects_bad_pages():
    lib = kvq.load_library()
    with pytest.raises(kvq.KVQError):
        kvq.KVQCache(1, 1, 128, [10], page_bytes=3000, pool_pages=4)
    with pytest.raises(kvq.KVQError):
        kvq.KVQCache(1, 1, 128, [10], page_bytes=4096, pool_pages=0)
    assert lib is not None
