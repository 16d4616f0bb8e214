"""KVA (late-layer KV approximation) prefill path, native to NVIDIA B200 (sm_100a).

The compute lives in ``libkva.so`` (hand-written CUDA kernels behind the C ABI
declared in ``include/kva.h`` and ``include/kva_ops.h``); this package is its thin
ctypes binding.  Importing it fails loudly when the library has not been built:
there is no CPU or library fallback.
"""
from .kva import *  # noqa: F401,F403
from .kva import LIB_PATH, EXPORTED, KvaError, Weights, KvCache, make_dims  # noqa: F401
