"""HySparse hybrid-block attention hot path for B200 (sm_100a).

The compute lives in ``libhysparse.so`` (hand-written CUDA kernels behind a C
ABI declared in ``include/hysparse.h``).  ``attention_tcgen05_tma_b200.hysparse``
is the thin ctypes binding; ``attention_tcgen05_tma_b200.inputs`` draws the
seeded synthetic workloads.  Importing this package does not load the library.
"""
__all__ = ["hysparse", "inputs"]
