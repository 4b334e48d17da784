"""B200-native rotation + INT4 W4A4 hot path.

The compute lives in ``libpq.so`` (hand-written CUDA for sm_100a behind a C ABI, see
``include/pq.h``); :mod:`rotation_int4_w4a4_b200.pq` is the thin ctypes binding with the
same entry-point names.  :mod:`rotation_int4_w4a4_b200.inputs` holds the seeded synthetic
input generators.  Importing this package does not load the library; importing ``pq`` does,
and raises if the library has not been built.
"""
__all__ = ["pq", "inputs"]
