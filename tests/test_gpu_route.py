"""GPU parity of the router hard argmax (Eq. 5 heads, inference): modes and widths are
bit-exact with the oracle, including ties, NaN rows and ragged row counts."""
import numpy as np
import pytest
import torch

import oracle
from mixed_precision_kv_write_b200 import kvq, synth

pytestmark = pytest.mark.gpu
W = synth.WORKLOADS


def _check(za, zb):
    modes, bits = kvq.route_argmax(za, zb)
    torch.cuda.synchronize()
    rm, rb = oracle.route_argmax(None if za is None else za.cpu().numpy(),
                                 None if zb is None else zb.cpu().numpy())
    if za is not None:
        assert np.array_equal(modes.cpu().numpy(), rm)
    else:
        assert modes is None
    if zb is not None:
        assert np.array_equal(bits.cpu().numpy(), rb)
    else:
        assert bits is None


def test_route_full_size():
    # the ragged_prefill shape: 17771 tokens x 16 heads
    za, zb = synth.router_logits(W["ragged_prefill"], "cuda")
    _check(za, zb)


@pytest.mark.parametrize("rows", [1, 3, 4, 5, 1027])
def test_route_ragged_rows_and_specials(rows):
    g = torch.Generator(device="cuda").manual_seed(rows)
    za = torch.randn((rows, 3), generator=g, device="cuda")
    zb = torch.randn((rows, 4), generator=g, device="cuda")
    za[::3] = torch.round(za[::3])
    zb[::2] = torch.round(zb[::2])
    za[0, 0] = float("nan")
    zb[-1] = float("nan")
    if rows > 2:
        za[1] = float("-inf")
        zb[1, 2] = float("inf")
    _check(za, zb)
    _check(za, None)
    _check(None, zb)


def test_route_feeds_write_and_decode():
    # the router's outputs are valid kvq_write widths and decode modes
    wl = synth.scaled(W["decode_1p3b"], seqlens=(64, 33))
    za, zb = synth.router_logits(wl, "cuda")
    modes, bits = kvq.route_argmax(za, zb)
    k, v, _ = synth.kv_tokens(wl, "cuda")
    cache = kvq.KVQCache(wl.batch, wl.heads, wl.head_dim, list(wl.seqlens))
    kvq.kvq_write(k, v, bits, synth.cu_seqlens(wl.seqlens, "cuda"), cache)
    q, _ = synth.decode_queries(wl, "cuda")
    last = torch.tensor(np.cumsum(wl.seqlens) - 1, device="cuda")
    kvq.routed_attn_decode(q, cache, modes[last].contiguous(), wl.w)
    cache.check()
    assert cache.lengths().tolist() == list(wl.seqlens)
