"""GPU parity of quantize-on-write (Eq. 4): stored codes, scales, zeros and widths are
bit-exact with the oracle, on every workload shape, plus the device-side error paths."""
import numpy as np
import pytest
import torch

from mixed_precision_kv_write_b200 import kvq, synth
from kvq_testlib import build_cache, check_records

pytestmark = pytest.mark.gpu
W = synth.WORKLOADS


@pytest.mark.parametrize("name,seqlens", [
    ("tiny_prefill", None),
    ("prefill_160m", (300, 1, 77, 2048)),
    ("ragged_prefill", (1024, 3000, 17, 129)),
    ("decode_1p3b", (513, 64, 1)),
])
def test_write_bit_exact(name, seqlens):
    wl = W[name] if seqlens is None else synth.scaled(W[name], seqlens=seqlens)
    k, v, bits = synth.kv_tokens(wl, "cuda")
    cache = build_cache(wl, k, v, bits)
    cache.check()
    kc, vc, bc = k.cpu(), v.cpu(), bits.cpu()
    pairs = [(s, h) for s in range(wl.batch) for h in range(wl.heads)]
    check_records(cache, wl, kc, vc, bc, pairs)
    assert cache.lengths().tolist() == list(wl.seqlens)


def test_write_full_size_sampled():
    # the full ragged-prefill workload (17771 tokens x 16 heads, head_dim 128), sampled heads
    wl = W["ragged_prefill"]
    k, v, bits = synth.kv_tokens(wl, "cuda")
    cache = build_cache(wl, k, v, bits)
    cache.check()
    rng = np.random.default_rng(0)
    pairs = [(s, int(rng.integers(wl.heads))) for s in range(wl.batch)]
    check_records(cache, wl, k.cpu(), v.cpu(), bits.cpu(), pairs)


def test_write_in_chunks_equals_one_write():
    # appending each sequence in pieces stores the same records as one write
    wl = synth.scaled(W["prefill_160m"], seqlens=(200, 130))
    k, v, bits = synth.kv_tokens(wl, "cuda")
    cache = kvq.KVQCache(wl.batch, wl.heads, wl.head_dim, list(wl.seqlens))
    cu_all = synth.cu_seqlens(wl.seqlens).tolist()
    for a, b in [(0, 1), (1, 70), (70, None)]:
        idx, lens = [], []
        for s in range(wl.batch):
            L = wl.seqlens[s]
            lo, hi = min(a, L), (L if b is None else min(b, L))
            idx += list(range(cu_all[s] + lo, cu_all[s] + hi))
            lens.append(hi - lo)
        idx_t = torch.tensor(idx, device="cuda", dtype=torch.long)
        kvq.kvq_write(k[idx_t].contiguous(), v[idx_t].contiguous(), bits[idx_t].contiguous(),
                      synth.cu_seqlens(lens, "cuda"), cache)
    cache.check()
    assert cache.lengths().tolist() == [200, 130]
    check_records(cache, wl, k.cpu(), v.cpu(), bits.cpu(),
                  [(s, h) for s in range(2) for h in range(wl.heads)])


def test_constant_and_extreme_vectors():
    wl = synth.Workload("edge", "prefill", (6,), 2, 128, 4, (0.25,) * 4, (1 / 3,) * 3, False, 7)
    k = torch.zeros((6, 2, 128), dtype=torch.float16)
    k[1] = 3.5                                        # constant: s = 0, codes 0
    k[2, :, ::2] = 65504.0                            # fp16 extremes
    k[2, :, 1::2] = -65504.0
    k[3] = torch.linspace(-1, 1, 128, dtype=torch.float16)
    k[4, :, 0] = -0.0                                 # signed zeros
    k[5] = torch.randn((2, 128)).half() * 1e-4        # subnormal-scale values
    v = k.flip(0).contiguous()
    bits = torch.tensor([[2, 4], [8, 2], [2, 8], [4, 16], [16, 2], [8, 4]], dtype=torch.uint8)
    cache = build_cache(wl, k.cuda(), v.cuda(), bits.cuda())
    cache.check()
    check_records(cache, wl, k, v, bits, [(0, 0), (0, 1)])


def test_bad_bits_rejected_on_device():
    wl = synth.scaled(W["tiny_prefill"], seqlens=(10,))
    k, v, bits = synth.kv_tokens(wl, "cuda")
    bits[3, 1] = 3
    cache = kvq.KVQCache(1, wl.heads, wl.head_dim, [10])
    kvq.kvq_write(k, v, bits, synth.cu_seqlens([10], "cuda"), cache)
    with pytest.raises(kvq.KVQError) as e:
        cache.check()
    assert e.value.code == kvq.KVQ_ERR_BITS
    cache.check()  # cleared
    # the sequence's write was rejected for every head
    assert cache.lengths().tolist() == [0]


def test_capacity_overflow_rejected_on_device():
    wl = synth.scaled(W["tiny_prefill"], seqlens=(10,))
    k, v, bits = synth.kv_tokens(wl, "cuda")
    cache = kvq.KVQCache(1, wl.heads, wl.head_dim, [8])
    kvq.kvq_write(k, v, bits, synth.cu_seqlens([10], "cuda"), cache)
    with pytest.raises(kvq.KVQError) as e:
        cache.check()
    assert e.value.code == kvq.KVQ_ERR_CAPACITY
    assert cache.lengths().tolist() == [0]


def test_truncate_then_rewrite():
    wl = synth.scaled(W["ragged_prefill"], seqlens=(100,), heads=3)
    k, v, bits = synth.kv_tokens(wl, "cuda")
    cache = build_cache(wl, k, v, bits)
    cache.truncate(torch.tensor([60], dtype=torch.int32, device="cuda"))
    assert cache.lengths().tolist() == [60]
    # rewrite positions 60..99 with the same tokens: the cache equals a one-shot write
    kvq.kvq_write(k[60:].contiguous(), v[60:].contiguous(), bits[60:].contiguous(),
                  synth.cu_seqlens([40], "cuda"), cache)
    cache.check()
    check_records(cache, wl, k.cpu(), v.cpu(), bits.cpu(), [(0, h) for h in range(3)])


def test_host_argument_errors():
    cache = kvq.KVQCache(1, 2, 64, [4])
    lib = kvq.load_library()
    assert lib.routed_attn_decode(None, cache.handle, None, 0, None, None) == kvq.KVQ_ERR_ARG
    q = torch.zeros((1, 2, 64), dtype=torch.float16, device="cuda")
    m = torch.zeros((1, 2), dtype=torch.uint8, device="cuda")
    with pytest.raises(kvq.KVQError):
        kvq.routed_attn_decode(q, cache, m, -1)


def _append_rows(k, v, bits, cu, pos, counts):
    """The call's tensors for appending counts[s] tokens after position pos[s] of each
    sequence (rows of the packed full-sequence tensors, in sequence order)."""
    rows = [cu[s] + pos[s] + i for s in range(len(counts)) for i in range(counts[s])]
    idx = torch.tensor(rows, dtype=torch.long, device=k.device)
    cus = torch.tensor([0] + np.cumsum(counts).tolist(), dtype=torch.int32, device=k.device)
    return k[idx].contiguous(), v[idx].contiguous(), bits[idx].contiguous(), cus


@pytest.mark.parametrize("name", ["decode_1p3b", "prefill_160m"])
def test_short_appends_bit_exact(name):
    # a long first write, then calls of at most 2 tokens per sequence (n_tok <= 2 * batch:
    # the single-launch append path), ragged and with empty sequences
    wl = synth.scaled(W[name], seqlens=(40, 7, 0, 33, 12))
    k, v, bits = synth.kv_tokens(wl, "cuda")
    cu = synth.cu_seqlens(wl.seqlens).tolist()
    cache = kvq.KVQCache(wl.batch, wl.heads, wl.head_dim, [max(1, L) for L in wl.seqlens])
    pos = [0] * wl.batch
    first = [min(5, L) for L in wl.seqlens]
    kvq.kvq_write(*_append_rows(k, v, bits, cu, pos, first), cache)
    pos = first[:]
    rng = np.random.default_rng(1)
    calls = 0
    while any(pos[s] < wl.seqlens[s] for s in range(wl.batch)):
        counts = [int(min(rng.integers(0, 3), wl.seqlens[s] - pos[s])) for s in range(wl.batch)]
        kvq.kvq_write(*_append_rows(k, v, bits, cu, pos, counts), cache)
        pos = [p + c for p, c in zip(pos, counts)]
        calls += 1
    assert calls > 10
    cache.check()
    assert cache.lengths().tolist() == list(wl.seqlens)
    pairs = [(s, h) for s in range(wl.batch) for h in range(wl.heads)]
    check_records(cache, wl, k.cpu(), v.cpu(), bits.cpu(), pairs)


def test_short_append_errors():
    # one token per sequence: a bad width in sequence 1 refuses its write for every head;
    # sequence 2 is full; the others are written
    wl = synth.scaled(W["decode_1p3b"], seqlens=(3, 3, 3, 3), heads=4)
    k, v, bits = synth.kv_tokens(wl, "cuda")
    cu = synth.cu_seqlens(wl.seqlens).tolist()
    cache = kvq.KVQCache(4, wl.heads, wl.head_dim, [3, 3, 2, 3])
    pos = [0, 0, 0, 0]
    for _ in range(2):
        kvq.kvq_write(*_append_rows(k, v, bits, cu, pos, [1, 1, 1, 1]), cache)
        pos = [p + 1 for p in pos]
    cache.check()
    kk, vv, bb, cus = _append_rows(k, v, bits, cu, pos, [1, 1, 1, 1])
    bb[1, 2] = 3
    kvq.kvq_write(kk, vv, bb, cus, cache)
    with pytest.raises(kvq.KVQError) as e:
        cache.check()
    assert e.value.code in (kvq.KVQ_ERR_BITS, kvq.KVQ_ERR_CAPACITY)
    assert cache.lengths().tolist() == [3, 2, 2, 3]
    check_records(cache, wl, k.cpu(), v.cpu(), bits.cpu(), [(s, h) for s in (0, 3) for h in range(4)])


def test_long_writes_in_several_calls_multi_chunk():
    # each call is long (more than 64 tokens per sequence on average), so the record offsets
    # are scanned in 1024-token chunks; the look-back of later calls must not read the flags
    # that earlier calls left behind
    wl = synth.scaled(W["ragged_prefill"], seqlens=(3000, 2600, 5), heads=3)
    k, v, bits = synth.kv_tokens(wl, "cuda")
    cache = kvq.KVQCache(wl.batch, wl.heads, wl.head_dim, list(wl.seqlens))
    cu = synth.cu_seqlens(wl.seqlens).tolist()
    pos = [0] * wl.batch
    for cut in (1100, 2300, None):
        counts = [(L if cut is None else min(cut, L)) - p for L, p in zip(wl.seqlens, pos)]
        assert sum(counts) > 64 * wl.batch
        kvq.kvq_write(*_append_rows(k, v, bits, cu, pos, counts), cache)
        pos = [p + c for p, c in zip(pos, counts)]
        cache.check()
    assert cache.lengths().tolist() == list(wl.seqlens)
    check_records(cache, wl, k.cpu(), v.cpu(), bits.cpu(),
                  [(s, h) for s in range(wl.batch) for h in range(wl.heads)])


def test_long_write_errors_in_later_chunks():
    # a long multi-chunk call where sequence 1 overflows its capacity and sequence 2 has a
    # bad width in its third chunk: both are refused for every head, sequence 0 is written
    wl = synth.scaled(W["ragged_prefill"], seqlens=(2500, 1500, 3100), heads=3)
    k, v, bits = synth.kv_tokens(wl, "cuda")
    bits_bad = bits.clone()
    cu = synth.cu_seqlens(wl.seqlens).tolist()
    bits_bad[cu[2] + 2600, 1] = 5
    cache = kvq.KVQCache(wl.batch, wl.heads, wl.head_dim, [2500, 1400, 3100])
    kvq.kvq_write(k, v, bits_bad, synth.cu_seqlens(wl.seqlens, "cuda"), cache)
    with pytest.raises(kvq.KVQError) as e:
        cache.check()
    assert e.value.code in (kvq.KVQ_ERR_BITS, kvq.KVQ_ERR_CAPACITY)
    cache.check()  # cleared
    assert cache.lengths().tolist() == [2500, 0, 0]
    check_records(cache, wl, k.cpu(), v.cpu(), bits.cpu(), [(0, h) for h in range(wl.heads)])
    # the refused sequences can be written afterwards (sequence 1 within its capacity)
    kk, vv, bb, cus = _append_rows(k, v, bits, cu, [0, 0, 0], [0, 1400, 3100])
    kvq.kvq_write(kk, vv, bb, cus, cache)
    cache.check()
    assert cache.lengths().tolist() == [2500, 1400, 3100]
    check_records(cache, wl, k.cpu(), v.cpu(), bits.cpu(), [(2, h) for h in range(wl.heads)])
    check_records(cache, wl, k.cpu(), v.cpu(), bits.cpu(), [(1, h) for h in range(wl.heads)],
                  tok_ranges=(0, 1400))


def test_long_write_beyond_direct_chunks():
    # a 20000-token sequence: 20 scan chunks of 1024 tokens, so the last three add the
    # running prefix published 17 chunks back to the 16 chunks they sum directly
    wl = synth.scaled(W["prefill_160m"], seqlens=(20000, 300), heads=2)
    k, v, bits = synth.kv_tokens(wl, "cuda")
    cache = build_cache(wl, k, v, bits)
    cache.check()
    assert cache.lengths().tolist() == list(wl.seqlens)
    check_records(cache, wl, k.cpu(), v.cpu(), bits.cpu(), [(s, h) for s in range(2) for h in range(2)])
