"""B200-native QVG 2-bit KV-cache codec.

The compute path is the CUDA library ``libqvg.so`` (hand-written sm_100a
kernels behind a C ABI declared in ``include/qvg.h``).  ``bit_kv_cache_qvg_b200.qvg``
is its thin ctypes binding; importing this package does not load the library,
so the input generator (``synth``) can be used on machines without it.
"""
__all__ = ["qvg", "synth"]
