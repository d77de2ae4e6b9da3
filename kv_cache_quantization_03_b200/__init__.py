"""KVarN-style variance-normalised KV-cache quantisation for B200 (sm_100a).

Modules:
  kvq        ctypes binding of the C ABI in include/kvq.h (libkvq.so; raises
             ImportError when the library is not built)
  cache      torch-allocated cache arrays and a view for the C ABI
  workloads  seeded synthetic inputs (no method arithmetic)
  build      nvcc build of libkvq.so

The package imports nothing heavy at import time, so the seeded workloads can
be used where the library is not built.
"""
__all__ = ["kvq", "cache", "workloads", "build"]
