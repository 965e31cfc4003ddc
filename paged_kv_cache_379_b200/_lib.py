"""ctypes loader for libpagedkv.so and the raw C signatures.

The shared library is built in-tree (``python -m paged_kv_cache_379_b200.build``
or ``__graft_entry__.build()``).  There is no fallback: if the library is
missing or fails to load, every call raises.
"""

from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libpagedkv.so")

_P = ctypes.c_void_p
_I = ctypes.c_int
_SZ = ctypes.c_size_t
_F = ctypes.c_float

# name -> (restype, argtypes), mirroring include/pagedkv.h
SIGNATURES = {
    "pa_status_string": (ctypes.c_char_p, [_I]),
    "pa_last_cuda_error": (_I, []),
    "pa_version": (_I, []),
    "pa_slot_mapping": (_I, [_P, _P, _I, _I, _P, _P, _P, _I, _I, _P]),
    "pa_reshape_and_cache": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P]),
    "pa_reshape_and_cache_fp8": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _F, _P]),
    "pa_decode_fp8": (_I, [_P, _P, _P, _P, _P, _P, _F, _F, _F, _I, _I, _I, _I, _I, _I, _I, _I, _P, _SZ, _P]),
    "pa_decode_fp8_split": (_I, [_P, _P, _P, _P, _P, _P, _F, _F, _F, _I, _I, _I, _I, _I, _I, _I, _I, _I, _P, _SZ,
                                 _P]),
    "pa_prefill": (_I, [_P, _P, _P, _P, _P, _P, _P, _F, _I, _I, _I, _I, _I, _I, _I, _I, _P]),
    "pa_append_decode_kv": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P]),
    "pa_append_decode_kv_cow": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P]),
    "pa_append_decode_kv_fp8": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _F, _P]),
    "pa_copy_blocks": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _P]),
    "pa_swap_blocks": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P]),
    "pa_decode": (_I, [_P, _P, _P, _P, _P, _P, _F, _I, _I, _I, _I, _I, _I, _I, _I, _P, _SZ, _P]),
    "pa_decode_workspace_size": (_SZ, [_I, _I, _I, _I, _I, _I]),
    "pa_decode_plan": (_I, [_I, _I, _I, _I, _I, _SZ]),
    "pa_decode_one_pass": (_I, [_P, _P, _P, _P, _P, _P, _F, _I, _I, _I, _I, _I, _I, _I, _I, _P]),
    "pa_decode_split": (_I, [_P, _P, _P, _P, _P, _P, _F, _I, _I, _I, _I, _I, _I, _I, _I, _I, _P, _SZ, _P]),
    "pa_decode_split_noalloc": (_I, [_P, _P, _P, _P, _P, _P, _F, _I, _I, _I, _I, _I, _I, _I, _I, _I, _P]),
    "pa_decode_partitions": (_I, [_P, _P, _P, _P, _P, _F, _I, _I, _I, _I, _I, _I, _I, _I, _I, _P, _SZ, _P]),
    "pa_lse_reduce": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _P]),
    "pa_validate_tables": (_I, [_P, _P, _I, _I, _I, _I, _I, _P, _P]),
    "pa_device_status": (_I, []),
    "pa_selftest_bounded_wait": (_I, [_P]),
    "pa_pool_create": (_P, [_I, _I, _P]),
    "pa_pool_destroy": (None, [_P]),
    "pa_pool_num_free": (_I, [_P]),
    "pa_pool_num_blocks": (_I, [_P]),
    "pa_pool_refcount": (_I, [_P, _I]),
    "pa_pool_allocate": (_I, [_P, _I, _P]),
    "pa_pool_free": (_I, [_P, _I]),
    "pa_pool_fork": (_I, [_P, _P, _I]),
    "pa_pool_cow": (_I, [_P, _I, _P, _P]),
    "pa_pool_import": (_I, [_P, _P, _I, _I, _P]),
    "pa_pool_prepare_decode": (_I, [_P, _I, _P, _I, _P, _P, _P, _P, _P]),
    "pa_cow_sources": (_I, [_P, _I, _I, _P, _I, _P]),
    "pa_prefix_groups": (_I, [_P, _I, _I, _P, _I, _I, _P, _P, _P]),
    "pa_decode_shared": (_I, [_P, _P, _P, _P, _P, _P, _F, _I, _I, _I, _I, _I, _I, _I, _I, _I, _P, _P, _I, _P, _SZ,
                              _P]),
    "pa_pool_free_table": (_I, [_P, _P, _I]),
    "pa_block_hash": (ctypes.c_uint64, [ctypes.c_uint64, _P, _I]),
    "pa_pool_allocate_prompt_cached": (_I, [_P, _P, _I, _P, _I, _P, _P]),
    "pa_pool_num_cached_blocks": (_I, [_P]),
    "pa_pool_swap_plan": (_I, [_P, _P, _P, _I, _P, _P]),
}

_lib = None


class PagedKVError(RuntimeError):
    """A C-ABI call returned a negative status."""

    def __init__(self, name: str, status: int, detail: str = ""):
        self.status = status
        super().__init__(f"{name} failed: {status_string(status)} ({status}){detail}")


def load():
    """Load libpagedkv.so (never builds it implicitly; never falls back)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m paged_kv_cache_379_b200.build` "
                "(needs nvcc); there is no CPU fallback")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def status_string(status: int) -> str:
    return load().pa_status_string(int(status)).decode()


def check(name: str, status: int) -> None:
    if status != 0:
        detail = ""
        if status == -5:
            detail = f"; cudaError_t {load().pa_last_cuda_error()}"
        raise PagedKVError(name, status, detail)
