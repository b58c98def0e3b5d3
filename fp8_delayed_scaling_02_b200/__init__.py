"""B200-native FP8 per-tensor delayed-scaling linear: quantize_fp8 + mm_fp8.

The compute path is a C-ABI shared library (``libfp8ds.so``, built from
``csrc/`` for sm_100a).  ``fp8_delayed_scaling_02_b200.ops`` is the thin
Python binding; it loads the library on first use and raises if it is
missing -- there is no CPU fallback.
"""

__all__ = ["ops", "synthetic"]
