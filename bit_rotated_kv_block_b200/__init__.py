"""Rotated token-wise INT4 paged KV cache for B200 (sm_100a).

The compute lives in ``libkvq.so`` (hand-written CUDA behind a C ABI declared
in ``include/kvq.h``); ``kvq`` is the thin ctypes binding over it and
``workloads`` draws the seeded synthetic inputs. Importing the package does
not load the CUDA library; ``kvq.lib()`` does, and fails loudly if it is
missing.
"""
