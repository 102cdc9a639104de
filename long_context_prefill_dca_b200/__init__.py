"""B200 (sm_100a) library for long-context prefill attention of one GQA layer: Dual Chunk
Attention with YaRN scaling and vertical-slash sparse attention under chunked prefill.

The product is the C ABI in include/q1m.h (libq1m.so, built by ``build.py``); ``q1m`` is
its Python binding and ``layer`` a small convenience wrapper over it.
"""
from . import q1m  # noqa: F401
