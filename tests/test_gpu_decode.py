"""GPU parity of routed decode attention (Eq. 2 over the Eq. 4 cache) against the oracle:
small ragged cases that span several work items and a ragged tail, edge cases, and the
full decode workloads in the launch configuration the benchmark times (the cache holds
L - 1 tokens, the step appends the query token, then decodes)."""
import numpy as np
import pytest
import torch

from mixed_precision_kv_write_b200 import kvq, synth
from kvq_testlib import assert_close_attn, build_cache, check_records_seq, oracle_decode

pytestmark = pytest.mark.gpu
W = synth.WORKLOADS


def _run_decode(wl, k, v, bits, q, modes, w):
    cache = build_cache(wl, k, v, bits)
    out = kvq.routed_attn_decode(q, cache, modes, w)
    cache.check()
    return out.cpu().numpy(), cache


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("w", [0, 5, 100, 600, 5000])
def test_decode_small_ragged(D, w):
    base = W["decode_1p3b"] if D == 128 else synth.scaled(W["prefill_160m"], heads=3)
    wl = synth.scaled(base, seqlens=(1, 37, 600, 1500, 64), heads=3)
    k, v, bits = synth.kv_tokens(wl, "cuda")
    g = torch.Generator(device="cuda").manual_seed(w + D)
    q = torch.randn((wl.batch, 3, D), generator=g, device="cuda").half()
    modes = torch.randint(0, 3, (wl.batch, 3), generator=g, device="cuda").to(torch.uint8)
    modes[:, 0] = 2
    modes[:, 1] = 1
    out, _ = _run_decode(wl, k, v, bits, q, modes, w)
    kc, vc, bc, qc, mc = k.cpu(), v.cpu(), bits.cpu(), q.cpu(), modes.cpu()
    for s in range(wl.batch):
        for h in range(3):
            ref = oracle_decode(wl, kc, vc, bc, qc, mc, w, s, h)
            assert_close_attn(out[s, h], ref, f"s={s} h={h} mode={int(mc[s, h])}")


@pytest.mark.parametrize("bitval", [2, 4, 8, 16])
def test_decode_single_width(bitval):
    wl = synth.scaled(W["decode_1p3b"], seqlens=(700, 129), heads=2)
    k, v, bits = synth.kv_tokens(wl, "cuda")
    bits.fill_(bitval)
    q = torch.randn((2, 2, 128), device="cuda").half()
    modes = torch.full((2, 2), 2, dtype=torch.uint8, device="cuda")
    out, _ = _run_decode(wl, k, v, bits, q, modes, 0)
    for s in range(2):
        for h in range(2):
            ref = oracle_decode(wl, k.cpu(), v.cpu(), bits.cpu(), q.cpu(), modes.cpu(), 0, s, h)
            assert_close_attn(out[s, h], ref, f"b={bitval} s={s} h={h}")


def test_decode_skip_and_empty_are_zero():
    wl = synth.scaled(W["decode_1p3b"], seqlens=(50, 1), heads=2)
    k, v, bits = synth.kv_tokens(wl, "cuda")
    cache = kvq.KVQCache(3, 2, 128, [50, 1, 10])           # third sequence stays empty
    kvq.kvq_write(k, v, bits, synth.cu_seqlens([50, 1, 0], "cuda"), cache)
    q = torch.randn((3, 2, 128), device="cuda").half()
    modes = torch.tensor([[0, 2], [0, 1], [2, 1]], dtype=torch.uint8, device="cuda")
    out = kvq.routed_attn_decode(q, cache, modes, 7).cpu().numpy()
    cache.check()
    assert np.all(out[0, 0] == 0) and np.all(out[1, 0] == 0) and np.all(out[2] == 0)
    # a length-1 sequence returns deq(v_0) in both local and full modes
    ref = oracle_decode(wl, k.cpu(), v.cpu(), bits.cpu(), q.cpu(), modes.cpu(), 7, 1, 1)
    assert_close_attn(out[1, 1], ref)


def test_decode_bad_mode_reports():
    wl = synth.scaled(W["decode_1p3b"], seqlens=(5,), heads=1)
    k, v, bits = synth.kv_tokens(wl, "cuda")
    cache = build_cache(wl, k, v, bits)
    q = torch.randn((1, 1, 128), device="cuda").half()
    modes = torch.full((1, 1), 7, dtype=torch.uint8, device="cuda")
    out = kvq.routed_attn_decode(q, cache, modes, 1)
    with pytest.raises(kvq.KVQError) as e:
        cache.check()
    assert e.value.code == kvq.KVQ_ERR_MODE
    assert torch.all(out == 0)


def _decode_step_like_bench(wl):
    """Cache of L - 1 tokens, then the step: append the query token, decode."""
    B, H, D = wl.batch, wl.heads, wl.head_dim
    L = wl.seqlens[0]
    cache = kvq.KVQCache(B, H, D, [L + 8] * B)
    cu_prev = synth.cu_seqlens([L - 1] * B, "cuda")
    for s in range(B):   # build per sequence, bounded memory
        ks, vs, bs = synth.kv_sequence(wl, s, "cuda")
        one = synth.cu_seqlens([L - 1 if i == s else 0 for i in range(B)], "cuda")
        kvq.kvq_write(ks[:-1].contiguous(), vs[:-1].contiguous(), bs[:-1].contiguous(), one, cache)
    del cu_prev
    # the step's new token of every sequence
    kn, vn, bn = [], [], []
    for s in range(B):
        ks, vs, bs = synth.kv_sequence(wl, s, "cuda")
        kn.append(ks[-1:]), vn.append(vs[-1:]), bn.append(bs[-1:])
    q, modes = synth.decode_queries(wl, "cuda")
    kvq.kvq_write(torch.cat(kn), torch.cat(vn), torch.cat(bn), synth.cu_seqlens([1] * B, "cuda"), cache)
    out = kvq.routed_attn_decode(q, cache, modes, wl.w)
    cache.check()
    return out.cpu().numpy(), q.cpu(), modes.cpu(), cache


@pytest.mark.parametrize("name,n_check,n_rec", [("decode_1p3b", 96, 64), ("decode_long", 48, 40)])
def test_decode_full_size_sampled(name, n_check, n_rec):
    # Full-size cache built as the benchmark builds it (long write of L - 1 tokens, then the
    # step token through the single-launch append). Attention is checked on n_check sampled
    # (sequence, head) queries; the stored records (codes, scales, zeros, widths of all L
    # tokens, the appended one included) bit-exactly on n_rec sampled (sequence, head) pairs.
    wl = W[name]
    out, qc, mc, cache = _decode_step_like_bench(wl)
    assert cache.lengths().tolist() == list(wl.seqlens)
    rng = np.random.default_rng(1)
    pairs = [(int(s), int(h)) for s, h in zip(rng.integers(0, wl.batch, n_check),
                                              rng.integers(0, wl.heads, n_check))]
    rec_pairs = {(s, int(rng.integers(wl.heads))) for s in range(wl.batch)}
    while len(rec_pairs) < n_rec:
        rec_pairs.add((int(rng.integers(wl.batch)), int(rng.integers(wl.heads))))
    by_seq = {}
    for s, h in pairs:
        by_seq.setdefault(s, [set(), set()])[0].add(h)
    for s, h in rec_pairs:
        by_seq.setdefault(s, [set(), set()])[1].add(h)
    for s, (hs, hr) in sorted(by_seq.items()):
        ks, vs, bs = synth.kv_sequence(wl, s, "cuda")
        ks, vs, bs = ks.cpu(), vs.cpu(), bs.cpu()
        one = synth.scaled(wl, seqlens=(wl.seqlens[s],))
        for h in sorted(hs):
            ref = oracle_decode(one, ks, vs, bs, qc[s:s + 1], mc[s:s + 1], wl.w, 0, h)
            assert_close_attn(out[s, h], ref, f"{name} s={s} h={h} mode={int(mc[s, h])}")
        check_records_seq(cache, s, sorted(hr), ks, vs, bs, name)
    # skip heads are exact zeros everywhere
    skip = (mc.numpy() == 0)
    assert np.all(out[skip] == 0)


def test_decode_bitwise_repeatable_with_many_items():
    # several times more work items than split-K CTAs (about 4,000, enough for front items
    # to be walked in pairs): which CTA takes which item, and where in the list a
    # sequence's items land, vary from call to call (items are reserved and claimed
    # dynamically), the outputs must not
    wl = synth.scaled(W["decode_1p3b"], seqlens=(4096,) * 64, heads=16)
    k, v, bits = synth.kv_tokens(wl, "cuda")
    cache = kvq.KVQCache(wl.batch, wl.heads, wl.head_dim, list(wl.seqlens))
    kvq.kvq_write(k, v, bits, synth.cu_seqlens(wl.seqlens, "cuda"), cache)
    del k, v
    g = torch.Generator(device="cuda").manual_seed(5)
    q = torch.randn((wl.batch, wl.heads, 128), generator=g, device="cuda").half()
    modes = torch.full((wl.batch, wl.heads), 2, dtype=torch.uint8, device="cuda")
    modes[::3, 1] = 1
    outs = [kvq.routed_attn_decode(q, cache, modes, 300) for _ in range(4)]
    outs.append(kvq.routed_attn_decode_noalloc(q, cache, modes, 300).clone())
    cache.check()
    for o in outs[1:]:
        assert torch.equal(o, outs[0])


@pytest.mark.parametrize("pattern", ["local", "full", "mixed"])
def test_decode_list_regions(pattern):
    # window pieces are listed at the back of the work list, the last piece of each other
    # range in the middle and its other pieces, two at a time, at the front: only-local
    # queries leave the front and middle empty, only-full ones the back; mixed heads and
    # queries fill all three (a head's items can sit in every region)
    wl = synth.scaled(W["decode_1p3b"], seqlens=(3000, 2500, 700, 1), heads=4)
    k, v, bits = synth.kv_tokens(wl, "cuda")
    g = torch.Generator(device="cuda").manual_seed(11)
    q = torch.randn((wl.batch, 4, 128), generator=g, device="cuda").half()
    fill = {"local": 1, "full": 2, "mixed": 2}[pattern]
    modes = torch.full((wl.batch, 4), fill, dtype=torch.uint8, device="cuda")
    if pattern == "mixed":
        modes[:, 1] = 1
        modes[1::2, 2] = 1
        modes[2, 3] = 0
    out, cache = _run_decode(wl, k, v, bits, q, modes, 300)
    again = kvq.routed_attn_decode_noalloc(q, cache, modes, 300).cpu().numpy()
    assert np.array_equal(again, out)
    kc, vc, bc, qc, mc = k.cpu(), v.cpu(), bits.cpu(), q.cpu(), modes.cpu()
    for s in range(wl.batch):
        for h in range(4):
            ref = oracle_decode(wl, kc, vc, bc, qc, mc, 300, s, h)
            assert_close_attn(out[s, h], ref, f"{pattern} s={s} h={h} mode={int(mc[s, h])}")


@pytest.mark.parametrize("D", [64, 128])
def test_decode_many_outputs(D):
    # at least 4 (sequence, query head) outputs per SM: the combine runs one warp per output
    # (fewer outputs take a CTA each, as in the small cases above)
    base = W["decode_1p3b"] if D == 128 else W["prefill_160m"]
    heads = 12
    wl = synth.scaled(base, seqlens=tuple(40 + 37 * i for i in range(64)), heads=heads)
    k, v, bits = synth.kv_tokens(wl, "cuda")
    g = torch.Generator(device="cuda").manual_seed(17 + D)
    q = torch.randn((wl.batch, heads, D), generator=g, device="cuda").half()
    modes = torch.randint(0, 3, (wl.batch, heads), generator=g, device="cuda").to(torch.uint8)
    out, _ = _run_decode(wl, k, v, bits, q, modes, 50)
    kc, vc, bc, qc, mc = k.cpu(), v.cpu(), bits.cpu(), q.cpu(), modes.cpu()
    for s in range(0, wl.batch, 7):
        for h in range(0, heads, 5):
            ref = oracle_decode(wl, kc, vc, bc, qc, mc, 50, s, h)
            assert_close_attn(out[s, h], ref, f"D={D} s={s} h={h} mode={int(mc[s, h])}")
