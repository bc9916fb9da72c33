"""Routed mixed-precision KV cache for NVIDIA B200 (sm_100a).

Quantize-on-write of K/V at a per-(token, head) width b in {2, 4, 8, 16} (TriRoute
paper review page, Eq. 4) and causal attention over that cache with per-(token, head)
modes skip / local-w / full (Eq. 2). The compute runs in the CUDA library
``libkvq.so`` (C ABI in ``include/kvq.h``); ``kvq`` is its thin ctypes binding.
"""
__all__ = ["kvq", "synth"]
