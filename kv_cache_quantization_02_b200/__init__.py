"""kvq: B200-native fused KV-cache rotate-and-quantize.

The compute lives in ``libkvq.so`` (hand-written CUDA for sm_100a behind a
C ABI, declared in ``include/kvq.h``).  ``kv_cache_quantization_02_b200.kvq``
is the thin ctypes binding with the same names; ``workloads`` draws seeded
synthetic inputs.  Importing this package loads nothing; the binding loads the
library on import and raises if it is missing.
"""

__all__ = ["kvq", "workloads"]
