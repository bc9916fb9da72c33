"""CPU oracle for the routed mixed-precision KV write (Eq. 4) and routed attention (Eq. 2)
of the TriRoute paper review page, section 3.

TEST INFRASTRUCTURE. Only the tests, ``__graft_entry__.smoke()`` and the benchmark's
CPU-baseline / reference leg may import this package. The product path (the CUDA library
and its Python binding) never imports it; the two share no code.

The arithmetic lives in ``kvq_oracle.c`` (plain C99, no FMA contraction); this module
compiles it with gcc on first use and marshals numpy arrays through ctypes.

Parity pins for every function here are in ``tests/test_oracle_*.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kvq_oracle.c")
_LIB = os.path.join(_HERE, "libkvq_oracle.so")
_lock = threading.Lock()
_lib = None

SKIP, LOCAL, FULL = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math, no FMA contraction). Returns the .so path."""
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c99", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
           "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            p = ctypes.c_void_p
            lib.oracle_quantize.argtypes = [p, ctypes.c_int, ctypes.c_int, p, p, p]
            lib.oracle_quantize.restype = ctypes.c_int
            lib.oracle_quantize_many.argtypes = [p, ctypes.c_int, ctypes.c_int, p, p, p, p]
            lib.oracle_quantize_many.restype = ctypes.c_int
            lib.oracle_dequantize.argtypes = [p, ctypes.c_int, ctypes.c_int, ctypes.c_float,
                                              ctypes.c_float, p]
            lib.oracle_dequantize.restype = None
            lib.oracle_routed_attention_head.argtypes = [
                ctypes.c_int, ctypes.c_int, p, p, p, ctypes.c_int, p, p, p, ctypes.c_int, p]
            lib.oracle_routed_attention_head.restype = ctypes.c_int
            lib.oracle_half_to_double.argtypes = [ctypes.c_uint16]
            lib.oracle_half_to_double.restype = ctypes.c_double
            lib.oracle_route_argmax.argtypes = [p, ctypes.c_int64, ctypes.c_int, p]
            lib.oracle_route_argmax.restype = None
            _lib = lib
    return _lib


def _bits16(x) -> np.ndarray:
    """fp16 array (or its raw uint16 bits) -> contiguous uint16 bit array."""
    a = np.asarray(x)
    if a.dtype == np.float16:
        a = a.view(np.uint16)
    if a.dtype != np.uint16:
        raise TypeError(f"expected float16 or uint16 bits, got {a.dtype}")
    return np.ascontiguousarray(a)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def quantize(x, b: int):
    """Eq. 4 on one vector: returns (codes uint16[n], s float32, z float32).

    b in {2, 4, 8}: asymmetric min/max codes; b == 16: raw fp16 bits with (s, z) = (1, 0).
    """
    xb = _bits16(x).reshape(-1)
    codes = np.empty(xb.shape[0], dtype=np.uint16)
    s = np.zeros(1, dtype=np.float32)
    z = np.zeros(1, dtype=np.float32)
    rc = _load().oracle_quantize(_ptr(xb), xb.shape[0], int(b), _ptr(codes), _ptr(s), _ptr(z))
    if rc:
        raise ValueError(f"oracle_quantize rejected b={b}, n={xb.shape[0]}")
    return codes, s[0], z[0]


def quantize_many(x, bits):
    """Eq. 4 on m vectors x[m, n] with widths bits[m]: (codes uint16[m, n], s[m], z[m])."""
    xb = _bits16(x)
    m, n = xb.shape
    bb = np.ascontiguousarray(np.asarray(bits, dtype=np.uint8).reshape(m))
    codes = np.empty((m, n), dtype=np.uint16)
    s = np.empty(m, dtype=np.float32)
    z = np.empty(m, dtype=np.float32)
    rc = _load().oracle_quantize_many(_ptr(xb), m, n, _ptr(bb), _ptr(codes), _ptr(s), _ptr(z))
    if rc:
        raise ValueError("oracle_quantize_many: unsupported bit-width")
    return codes, s, z


def dequantize(codes, b: int, s, z) -> np.ndarray:
    """Eq. 4 reconstruction code*s + z in fp64 (b == 16: the fp16 value)."""
    c = np.ascontiguousarray(np.asarray(codes, dtype=np.uint16).reshape(-1))
    out = np.empty(c.shape[0], dtype=np.float64)
    _load().oracle_dequantize(_ptr(c), c.shape[0], int(b), float(s), float(z), _ptr(out))
    return out


def routed_attention_head(q, pos, modes, w: int, k, v, bits) -> np.ndarray:
    """Eq. 2 for one (sequence, head) over the Eq. 4 cache built from k, v at widths bits.

    q: fp16 [n_q, D]; pos: int [n_q] (0-based t < L); modes: [n_q] (0 skip, 1 local, 2 full);
    k, v: fp16 [L, D]; bits: [L]. Returns fp32 [n_q, D].
    """
    qb = _bits16(q)
    kb = _bits16(k)
    vb = _bits16(v)
    n_q, D = qb.shape
    L = kb.shape[0]
    if kb.shape != (L, D) or vb.shape != (L, D):
        raise ValueError("k, v must be [L, D] with the query's D")
    bb = np.ascontiguousarray(np.asarray(bits, dtype=np.uint8).reshape(L))
    pp = np.ascontiguousarray(np.asarray(pos, dtype=np.int32).reshape(n_q))
    mm = np.ascontiguousarray(np.asarray(modes, dtype=np.uint8).reshape(n_q))
    out = np.empty((n_q, D), dtype=np.float32)
    rc = _load().oracle_routed_attention_head(D, L, _ptr(kb), _ptr(vb), _ptr(bb), n_q, _ptr(qb),
                                              _ptr(pp), _ptr(mm), int(w), _ptr(out))
    if rc:
        raise ValueError(f"oracle_routed_attention_head failed with {rc}")
    return out


def half_to_double(h: int) -> float:
    return _load().oracle_half_to_double(int(h))


WIDTHS = (2, 4, 8, 16)


def route_argmax(z_attn=None, z_bits=None):
    """Inference-time router (Eq. 5 heads, hard argmax): modes uint8 [...] from z_attn
    [..., 3] (0 skip, 1 local, 2 full) and widths uint8 [...] in {2, 4, 8, 16} from
    z_bits [..., 4]. Either input may be None."""
    def amax(z, k):
        z = np.ascontiguousarray(np.asarray(z, dtype=np.float32))
        if z.shape[-1] != k:
            raise ValueError(f"last dimension must be {k}")
        out = np.empty(z.shape[:-1], dtype=np.uint8)
        _load().oracle_route_argmax(_ptr(z), int(out.size), k, _ptr(out))
        return out
    modes = None if z_attn is None else amax(z_attn, 3)
    bits = None if z_bits is None else np.asarray(WIDTHS, dtype=np.uint8)[amax(z_bits, 4)]
    return modes, bits
