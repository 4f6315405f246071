"""Paged decode attention for B200 (sm_100a).

The compute path lives in ``libpa.so`` (CUDA kernels behind a C ABI, built
from ``csrc/``).  ``paged_kv_cache_458_b200.pa`` is the thin ctypes binding;
``paged_kv_cache_458_b200.gen`` builds seeded synthetic inputs.
"""
