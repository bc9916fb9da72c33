"""Failure paths of the library, driven on demand without faulting the GPU.

- An injected allocation failure in cache creation (as if cudaMalloc had failed at the
  n-th buffer) returns KVQ_ERR_NOMEM, leaves the handle NULL and frees everything the
  call had allocated; the next creation works.
- A bounded device wait that runs out (a barrier nothing completes, with a 1 ms limit)
  records KVQ_ERR_DEVICE_CHECK in the cache's status word; the kernel returns, and the
  context stays usable for ordinary calls afterwards.
"""
import ctypes

import numpy as np
import pytest
import torch

from mixed_precision_kv_write_b200 import kvq, synth
from kvq_testlib import assert_close_attn, build_cache, oracle_decode

pytestmark = pytest.mark.gpu


def _create(lib, batch, heads, head_dim, cap):
    h = ctypes.c_void_p()
    arr = (ctypes.c_int64 * batch)(*([cap] * batch))
    rc = lib.kvq_cache_create(ctypes.byref(h), batch, heads, head_dim, ctypes.cast(arr, ctypes.c_void_p), None)
    return rc, h


@pytest.mark.parametrize("nth", [1, 4, 9, 20])
def test_injected_allocation_failure_frees_everything(nth):
    lib = kvq.load_library()
    torch.cuda.synchronize()
    rc, h = _create(lib, 4, 8, 128, 50000)            # ~0.8 GB of records: a leak would show
    assert rc == kvq.KVQ_OK
    lib.kvq_cache_destroy(h)
    free0, _ = torch.cuda.mem_get_info()
    assert lib.kvq_test_fail_alloc(nth) == kvq.KVQ_OK
    rc, h = _create(lib, 4, 8, 128, 50000)
    assert rc == kvq.KVQ_ERR_NOMEM
    assert h.value is None
    assert b"cudaMalloc failed" in lib.kvq_last_error()
    free1, _ = torch.cuda.mem_get_info()
    assert abs(free1 - free0) <= (16 << 20), (free0, free1)
    # the injection was consumed: the next create succeeds and releases its memory
    rc, h = _create(lib, 4, 8, 128, 50000)
    assert rc == kvq.KVQ_OK and h.value
    assert lib.kvq_cache_destroy(h) == kvq.KVQ_OK
    free2, _ = torch.cuda.mem_get_info()
    assert abs(free2 - free0) <= (16 << 20)


def test_bounded_wait_runs_out_and_reports():
    wl = synth.scaled(synth.WORKLOADS["decode_1p3b"], seqlens=(300, 41), heads=2)
    k, v, bits = synth.kv_tokens(wl, "cuda")
    cache = build_cache(wl, k, v, bits)
    cache.check()
    lib = kvq.load_library()
    assert lib.kvq_test_bounded_wait(cache.handle, 1_000_000, None) == kvq.KVQ_OK
    with pytest.raises(kvq.KVQError) as e:
        cache.check()
    assert e.value.code == kvq.KVQ_ERR_DEVICE_CHECK
    cache.check()                                      # the status word was cleared
    # the context is still usable: an ordinary decode after the timed-out wait is correct
    q = torch.randn((2, 2, 128), device="cuda").half()
    modes = torch.tensor([[2, 1], [1, 2]], dtype=torch.uint8, device="cuda")
    out = kvq.routed_attn_decode(q, cache, modes, 50).cpu().numpy()
    cache.check()
    for s in range(2):
        for h in range(2):
            ref = oracle_decode(wl, k.cpu(), v.cpu(), bits.cpu(), q.cpu(), modes.cpu(), 50, s, h)
            assert_close_attn(out[s, h], ref, f"after timeout s={s} h={h}")
    assert np.isfinite(out).all()
