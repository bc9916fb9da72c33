"""Thin ctypes binding of libkvq.so (C ABI in include/kvq.h).

Argument marshalling only: every step of the write and attention paths runs in the CUDA
library. Tensors must be CUDA tensors on the cache's device; the current torch stream is
passed to every call unless `stream` is given. There is no CPU fallback: if the library is
missing or a tensor is on the CPU, the call raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libkvq.so")

KVQ_OK, KVQ_ERR_ARG, KVQ_ERR_BITS, KVQ_ERR_MODE, KVQ_ERR_CAPACITY, KVQ_ERR_CUDA, \
    KVQ_ERR_DEVICE_CHECK, KVQ_ERR_NOMEM = range(8)
MODE_SKIP, MODE_LOCAL, MODE_FULL = 0, 1, 2

# every symbol include/kvq.h declares
EXPORTS = ("kvq_cache_create", "kvq_cache_create_gqa", "kvq_cache_create_paged", "kvq_cache_destroy", "kvq_cache_reset", "kvq_cache_truncate",
           "kvq_cache_lengths", "kvq_write", "routed_attn_prefill", "routed_attn_decode",
           "routed_attn_decode_noalloc", "kvq_decode_step", "kvq_cache_export", "kvq_check", "kvq_set_profile_events",
           "kvq_route_argmax", "kvq_test_fail_alloc", "kvq_test_bounded_wait", "kvq_last_error")

_lib = None


class KVQError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"kvq status {code}: {msg}")
        self.code = code


def load_library(path: str = LIB_PATH):
    """Load libkvq.so (raises if it was not built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with "
                           "`python -m mixed_precision_kv_write_b200.build`")
    lib = ctypes.CDLL(path)
    vp, i32, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
    sig = {
        "kvq_cache_create": ([ctypes.POINTER(vp), i32, i32, i32, vp, vp], i32),
        "kvq_cache_create_gqa": ([ctypes.POINTER(vp), i32, i32, i32, i32, vp, vp], i32),
        "kvq_cache_create_paged": ([ctypes.POINTER(vp), i32, i32, i32, i32, vp, i64, i64, vp], i32),
        "kvq_cache_destroy": ([vp], i32),
        "kvq_cache_reset": ([vp, vp], i32),
        "kvq_cache_truncate": ([vp, vp, vp], i32),
        "kvq_cache_lengths": ([vp, vp, vp], i32),
        "kvq_write": ([vp, vp, vp, vp, i64, vp, vp], i32),
        "routed_attn_prefill": ([vp, vp, vp, i32, vp, i64, vp, vp], i32),
        "routed_attn_decode": ([vp, vp, vp, i32, vp, vp], i32),
        "routed_attn_decode_noalloc": ([vp, vp, vp, i32, vp, vp], i32),
        "kvq_decode_step": ([vp, vp, vp, vp, vp, i64, vp, vp, i32, vp, vp, vp], i32),
        "kvq_cache_export": ([vp, i32, i32, i64, i64, vp, vp, vp, vp, vp], i32),
        "kvq_check": ([vp, vp], i32),
        "kvq_set_profile_events": ([vp, vp], i32),
        "kvq_route_argmax": ([vp, vp, i64, vp, vp, vp], i32),
        "kvq_test_fail_alloc": ([i32], i32),
        "kvq_test_bounded_wait": ([vp, i64, vp], i32),
        "kvq_last_error": ([], ctypes.c_char_p),
    }
    for name, (args, res) in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = res
    _lib = lib
    return lib


def _raise(code: int):
    if code != KVQ_OK:
        raise KVQError(code, load_library().kvq_last_error().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream, device):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def _check(t, name, dtype, device, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda" or t.device.index != device.index:
        raise ValueError(f"{name} must be on {device} (got {t.device})")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype} (got {t.dtype})")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)} (got {tuple(t.shape)})")


class KVQCache:
    """Owning handle of a routed mixed-precision KV cache (kvq_cache_create/destroy)."""

    def __init__(self, batch: int, heads: int, head_dim: int, capacity, device=None, stream=None,
                 query_group: int = 1, page_bytes: int = 0, pool_pages: int = 0):
        lib = load_library()
        dev = torch.device("cuda") if device is None else torch.device(device)
        if dev.type != "cuda":
            raise ValueError(f"the cache lives on a CUDA device (got {dev})")
        self.device = dev if dev.index is not None else \
            torch.device("cuda", torch.cuda.current_device())
        cap = [int(capacity)] * batch if isinstance(capacity, int) else [int(x) for x in capacity]
        if len(cap) != batch:
            raise ValueError("capacity must be an int or have one entry per sequence")
        self.batch, self.heads, self.head_dim, self.capacity = batch, heads, head_dim, cap
        self.query_group = int(query_group)
        self.query_heads = heads * self.query_group      # heads of q / modes / out
        arr = (ctypes.c_int64 * batch)(*cap)
        h = ctypes.c_void_p()
        self.page_bytes, self.pool_pages = int(page_bytes), int(pool_pages)
        with torch.cuda.device(self.device):
            _raise(lib.kvq_cache_create_paged(ctypes.byref(h), batch, heads, self.query_group, head_dim,
                                              ctypes.cast(arr, ctypes.c_void_p), self.page_bytes,
                                              self.pool_pages, _stream(stream, self.device)))
        self._h = h

    @property
    def handle(self):
        return self._h

    def close(self):
        if getattr(self, "_h", None) is not None and self._h.value:
            with torch.cuda.device(self.device):
                load_library().kvq_cache_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def reset(self, stream=None):
        _raise(load_library().kvq_cache_reset(self._h, _stream(stream, self.device)))

    def truncate(self, lengths: torch.Tensor, stream=None):
        _check(lengths, "lengths", torch.int32, self.device, (self.batch,))
        _raise(load_library().kvq_cache_truncate(self._h, _ptr(lengths), _stream(stream, self.device)))

    def lengths(self, stream=None) -> torch.Tensor:
        out = torch.empty(self.batch, dtype=torch.int32, device=self.device)
        _raise(load_library().kvq_cache_lengths(self._h, _ptr(out), _stream(stream, self.device)))
        return out

    def check(self, stream=None):
        """Synchronize and raise KVQError if a device-side check failed."""
        _raise(load_library().kvq_check(self._h, _stream(stream, self.device)))

    def export(self, seq: int, head: int, first: int, count: int, stream=None):
        """(k_codes uint16 [count, D], v_codes, side fp32 [count, 4], bits uint8 [count])."""
        D = self.head_dim
        kc = torch.empty((count, D), dtype=torch.int16, device=self.device)
        vc = torch.empty((count, D), dtype=torch.int16, device=self.device)
        sd = torch.empty((count, 4), dtype=torch.float32, device=self.device)
        bt = torch.empty((count,), dtype=torch.uint8, device=self.device)
        _raise(load_library().kvq_cache_export(self._h, seq, head, first, count, _ptr(kc), _ptr(vc),
                                               _ptr(sd), _ptr(bt), _stream(stream, self.device)))
        return kc, vc, sd, bt


def kvq_set_profile_events(before=None, after=None):
    """Record torch.cuda.Event pairs around the main kernel of the following calls."""
    for e in (before, after):
        if e is not None and e.cuda_event == 0:
            e.record()          # torch creates the CUDA event on first record
    b = None if before is None else ctypes.c_void_p(before.cuda_event)
    a = None if after is None else ctypes.c_void_p(after.cuda_event)
    _raise(load_library().kvq_set_profile_events(b, a))


def kvq_write(k, v, bits, cu_seqlens, cache: KVQCache, stream=None):
    """Quantize-on-write of k, v [n_tok, H, D] fp16 at widths bits [n_tok, H] (Eq. 4)."""
    dev = cache.device
    n = k.shape[0]
    _check(k, "k", torch.float16, dev, (n, cache.heads, cache.head_dim))
    _check(v, "v", torch.float16, dev, (n, cache.heads, cache.head_dim))
    _check(bits, "bits", torch.uint8, dev, (n, cache.heads))
    _check(cu_seqlens, "cu_seqlens", torch.int32, dev, (cache.batch + 1,))
    _raise(load_library().kvq_write(_ptr(k), _ptr(v), _ptr(bits), _ptr(cu_seqlens), n, cache.handle,
                                    _stream(stream, dev)))


def routed_attn_prefill(q, cache: KVQCache, modes, w: int, cu_seqlens, out=None, stream=None):
    """Routed causal attention (Eq. 2) of q [n_tok, H, D] over the cache; returns fp32 out."""
    dev = cache.device
    n = q.shape[0]
    _check(q, "q", torch.float16, dev, (n, cache.query_heads, cache.head_dim))
    _check(modes, "modes", torch.uint8, dev, (n, cache.query_heads))
    _check(cu_seqlens, "cu_seqlens", torch.int32, dev, (cache.batch + 1,))
    if out is None:
        out = torch.empty((n, cache.query_heads, cache.head_dim), dtype=torch.float32, device=dev)
    _check(out, "out", torch.float32, dev, (n, cache.query_heads, cache.head_dim))
    _raise(load_library().routed_attn_prefill(_ptr(q), cache.handle, _ptr(modes), int(w),
                                              _ptr(cu_seqlens), n, _ptr(out), _stream(stream, dev)))
    return out


def routed_attn_decode(q, cache: KVQCache, modes, w: int, out=None, stream=None):
    """Routed decode attention (Eq. 2), q [B, H, D] at t = len - 1; returns fp32 out."""
    dev = cache.device
    shape = (cache.batch, cache.query_heads, cache.head_dim)
    _check(q, "q", torch.float16, dev, shape)
    _check(modes, "modes", torch.uint8, dev, shape[:2])
    if out is None:
        out = torch.empty(shape, dtype=torch.float32, device=dev)
    _check(out, "out", torch.float32, dev, shape)
    _raise(load_library().routed_attn_decode(_ptr(q), cache.handle, _ptr(modes), int(w), _ptr(out),
                                             _stream(stream, dev)))
    return out


def decode_step(q, k, v, bits, cu_seqlens, cache: KVQCache, modes, w: int, positions=None, out=None,
                stream=None):
    """One decode step (kvq_decode_step): append k, v [n_tok, H, D] at widths bits (Eq. 4),
    optionally after rolling each sequence back to `positions` [B] (int32), then routed
    decode attention (Eq. 2) of q [B, HQ, D]; returns fp32 out [B, HQ, D]."""
    dev = cache.device
    n = k.shape[0]
    shape = (cache.batch, cache.query_heads, cache.head_dim)
    _check(q, "q", torch.float16, dev, shape)
    _check(modes, "modes", torch.uint8, dev, shape[:2])
    _check(k, "k", torch.float16, dev, (n, cache.heads, cache.head_dim))
    _check(v, "v", torch.float16, dev, (n, cache.heads, cache.head_dim))
    _check(bits, "bits", torch.uint8, dev, (n, cache.heads))
    _check(cu_seqlens, "cu_seqlens", torch.int32, dev, (cache.batch + 1,))
    if positions is not None:
        _check(positions, "positions", torch.int32, dev, (cache.batch,))
    if out is None:
        out = torch.empty(shape, dtype=torch.float32, device=dev)
    _check(out, "out", torch.float32, dev, shape)
    _raise(load_library().kvq_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(bits), _ptr(cu_seqlens), n,
                                          _ptr(positions), _ptr(modes), int(w), cache.handle, _ptr(out),
                                          _stream(stream, dev)))
    return out


def routed_attn_decode_noalloc(q, cache: KVQCache, modes, w: int, out=None, stream=None):
    """routed_attn_decode without any device allocation in the call: its scratch is the
    library's static device array (see include/kvq.h). Pass a preallocated `out` to keep
    the whole call allocation-free; the first call on a device should precede any stream
    capture, and calls that overlap on the GPU race on the shared scratch."""
    dev = cache.device
    shape = (cache.batch, cache.query_heads, cache.head_dim)
    _check(q, "q", torch.float16, dev, shape)
    _check(modes, "modes", torch.uint8, dev, shape[:2])
    if out is None:
        out = torch.empty(shape, dtype=torch.float32, device=dev)
    _check(out, "out", torch.float32, dev, shape)
    _raise(load_library().routed_attn_decode_noalloc(_ptr(q), cache.handle, _ptr(modes), int(w),
                                                     _ptr(out), _stream(stream, dev)))
    return out


def route_argmax(z_attn=None, z_bits=None, stream=None):
    """Router hard argmax (Eq. 5 heads): modes uint8 [...] from z_attn fp32 [..., 3] and
    bits uint8 [...] in {2, 4, 8, 16} from z_bits fp32 [..., 4]; either may be None."""
    ref = z_attn if z_attn is not None else z_bits
    if ref is None:
        raise ValueError("route_argmax: pass z_attn, z_bits or both")
    dev = ref.device
    if dev.type != "cuda":
        raise ValueError(f"route_argmax: logits must be on a CUDA device (got {dev})")
    outs, n = [], None
    for z, k in ((z_attn, 3), (z_bits, 4)):
        if z is None:
            outs.append(None)
            continue
        if z.dtype != torch.float32 or not z.is_contiguous() or z.shape[-1] != k or z.device != dev:
            raise ValueError(f"route_argmax: expected contiguous fp32 [..., {k}] on {dev}")
        rows = z.numel() // k
        if n is not None and rows != n:
            raise ValueError("route_argmax: z_attn and z_bits have different row counts")
        n = rows
        outs.append(torch.empty(z.shape[:-1], dtype=torch.uint8, device=dev))
    _raise(load_library().kvq_route_argmax(_ptr(z_attn) if z_attn is not None else None,
                                           _ptr(z_bits) if z_bits is not None else None, n,
                                           _ptr(outs[0]) if outs[0] is not None else None,
                                           _ptr(outs[1]) if outs[1] is not None else None,
                                           _stream(stream, dev)))
    return outs[0], outs[1]
