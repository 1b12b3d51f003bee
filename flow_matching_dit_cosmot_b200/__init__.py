"""B200-native Cosmos 3 Mixture-of-Transformers layer hot path.

The compute lives in libcosmot.so (hand-written sm_100a CUDA, C ABI declared
in include/cosmot.h); this package holds its build script (`build`), a ctypes
binding (`_lib`) and torch marshalling helpers (`api`).  Importing `api` loads
the shared library and raises ImportError if it has not been built; there is
no fallback implementation.
"""
