"""The C-ABI library builds, loads without a GPU, exports every symbol include/kvq.h
declares, and rejects bad host-side arguments before touching the device."""
import ctypes
import os
import re

import pytest

from mixed_precision_kv_write_b200 import build, kvq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return kvq.load_library()


def _declared():
    src = open(os.path.join(ROOT, "include", "kvq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?\w+\s*\**\s*(\w+)\s*\(", src, flags=re.M)
    return sorted(set(n for n in names if n not in ("if", "return")))


def test_every_declared_symbol_is_exported(lib):
    declared = _declared()
    assert "kvq_write" in declared and "routed_attn_decode" in declared
    for name in declared:
        assert hasattr(lib, name), name
    assert sorted(kvq.EXPORTS) == declared


def test_create_rejects_bad_arguments_on_host(lib):
    h = ctypes.c_void_p()
    cap = (ctypes.c_int64 * 2)(16, 16)
    capp = ctypes.cast(cap, ctypes.c_void_p)
    assert lib.kvq_cache_create(ctypes.byref(h), 2, 4, 96, capp, None) == kvq.KVQ_ERR_ARG
    assert b"head_dim" in lib.kvq_last_error()
    assert lib.kvq_cache_create(ctypes.byref(h), 0, 4, 64, capp, None) == kvq.KVQ_ERR_ARG
    assert lib.kvq_cache_create(ctypes.byref(h), 2, 4, 64, None, None) == kvq.KVQ_ERR_ARG
    bad = (ctypes.c_int64 * 2)(16, 0)
    assert lib.kvq_cache_create(ctypes.byref(h), 2, 4, 64, ctypes.cast(bad, ctypes.c_void_p),
                                None) == kvq.KVQ_ERR_ARG
    assert h.value is None


def test_calls_reject_null_cache(lib):
    assert lib.kvq_write(None, None, None, None, 0, None, None) == kvq.KVQ_ERR_ARG
    assert lib.routed_attn_decode(None, None, None, 0, None, None) == kvq.KVQ_ERR_ARG
    assert lib.routed_attn_prefill(None, None, None, 0, None, 0, None, None) == kvq.KVQ_ERR_ARG
    assert lib.kvq_cache_export(None, 0, 0, 0, 1, None, None, None, None, None) == kvq.KVQ_ERR_ARG
    assert lib.kvq_cache_destroy(None) == kvq.KVQ_OK
    assert lib.kvq_last_error() == b""


def test_test_hooks_check_arguments_on_host(lib):
    assert lib.kvq_test_fail_alloc(-1) == kvq.KVQ_ERR_ARG
    assert lib.kvq_test_fail_alloc(0) == kvq.KVQ_OK
    assert lib.kvq_test_bounded_wait(None, 1000000, None) == kvq.KVQ_ERR_ARG


def test_paged_create_checks_pages_on_host(lib):
    h = ctypes.c_void_p()
    cap = (ctypes.c_int64 * 2)(16, 16)
    capp = ctypes.cast(cap, ctypes.c_void_p)
    assert lib.kvq_cache_create_paged(ctypes.byref(h), 2, 4, 1, 128, capp, 3000, 8, None) == kvq.KVQ_ERR_ARG
    assert b"page_bytes" in lib.kvq_last_error()
    assert lib.kvq_cache_create_paged(ctypes.byref(h), 2, 4, 1, 128, capp, 8192, 0, None) == kvq.KVQ_ERR_ARG
    assert lib.kvq_cache_create_paged(ctypes.byref(h), 2, 4, 1, 128, capp, 1 << 22, 8, None) == kvq.KVQ_ERR_ARG
    assert h.value is None
