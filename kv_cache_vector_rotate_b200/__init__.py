"""TurboQuant KV-cache codec for NVIDIA B200 (sm_100a).

The compute lives in libtq.so (CUDA kernels behind the C ABI of
include/tq.h); ``kv_cache_vector_rotate_b200.tq`` is its Python binding and
``kv_cache_vector_rotate_b200.synth`` draws seeded synthetic inputs.
"""

from . import tq  # noqa: F401  (the binding loads libtq.so on first use)

__all__ = ["tq"]
