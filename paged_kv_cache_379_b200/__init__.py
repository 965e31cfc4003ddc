"""Paged-KV decode attention for NVIDIA B200 (sm_100a).

The product is the C-ABI shared library ``libpagedkv.so`` (include/pagedkv.h):
hand-written CUDA kernels for slot mapping, cache write, copy-on-write block
copies and single-query paged decode attention (one-pass, split + log-sum-exp
reduce), plus a native host block pool.  This package is the thin Python
binding (argument marshalling only) and the seeded input generators.
"""

from . import workload  # noqa: F401  (numpy-only; importable without the library)
from ._lib import LIB_PATH, PagedKVError, load  # noqa: F401


def __getattr__(name):
    # lazy: the binding modules need torch / the built library
    if name in ("ops", "pool", "step"):
        import importlib
        return importlib.import_module(f".{name}", __name__)
    raise AttributeError(name)
