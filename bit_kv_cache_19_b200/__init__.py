"""B200-native RoPE-aware packed KV-cache quantization (Block-GTQ on TQ-MSE).

The work happens in ``libkvq.so`` (CUDA, sm_100a) behind the C ABI of
``include/kvq.h``; ``kvq`` is its ctypes binding and ``runtime`` holds the
device-memory plumbing (caches, plans, pointer arrays) built on PyTorch.
Build the library with ``python -m bit_kv_cache_19_b200.build``.
"""
from . import kvq  # noqa: F401

__all__ = ["kvq"]
