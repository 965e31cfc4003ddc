"""Host block pool: a Python handle over the native pa_pool_* C ABI.

The pool lives in host memory (C++ in csrc/block_pool.cpp) and only produces
integers: block ids, block tables, slot mappings and copy-on-write pairs.  See
include/pagedkv.h for the rules it follows (free list popped from its end,
reference counts, fork, copy-on-write, a new block only when the last is full).
"""

from __future__ import annotations

import ctypes

import numpy as np

from ._lib import PagedKVError, check, load


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


class BlockPool:
    def __init__(self, num_blocks: int, block_size: int, free_order=None):
        lib = load()
        self._keep = None
        if free_order is not None:
            fo = np.ascontiguousarray(free_order, dtype=np.int32)
            if fo.shape != (num_blocks,):
                raise ValueError("free_order must have num_blocks entries")
            h = lib.pa_pool_create(int(num_blocks), int(block_size), _ptr(fo))
        else:
            h = lib.pa_pool_create(int(num_blocks), int(block_size), None)
        if not h:
            raise ValueError("pa_pool_create failed (bad sizes or free_order not a permutation)")
        self._h = ctypes.c_void_p(h)
        self.num_blocks = int(num_blocks)
        self.block_size = int(block_size)

    def close(self) -> None:
        if getattr(self, "_h", None):
            load().pa_pool_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    # ---- BlockAllocator -------------------------------------------------------
    def get_num_free_blocks(self) -> int:
        return int(load().pa_pool_num_free(self._h))

    def refcount(self, block: int) -> int:
        rc = int(load().pa_pool_refcount(self._h, int(block)))
        if rc < 0:
            raise PagedKVError("pa_pool_refcount", rc)
        return rc

    def refcounts(self) -> list[int]:
        return [self.refcount(b) for b in range(self.num_blocks)]

    def allocate(self, n: int) -> list[int]:
        out = np.empty(max(n, 1), dtype=np.int32)
        check("pa_pool_allocate", load().pa_pool_allocate(self._h, int(n), _ptr(out)))
        return out[:n].tolist()

    def free(self, block: int) -> None:
        check("pa_pool_free", load().pa_pool_free(self._h, int(block)))

    def fork(self, table) -> list[int]:
        ids = np.ascontiguousarray(table, dtype=np.int32)
        check("pa_pool_fork", load().pa_pool_fork(self._h, _ptr(ids), int(ids.size)))
        return ids.tolist()

    def allocate_or_get_cow(self, block: int):
        out = np.zeros(1, dtype=np.int32)
        copied = np.zeros(1, dtype=np.int32)
        check("pa_pool_cow", load().pa_pool_cow(self._h, int(block), _ptr(out), _ptr(copied)))
        new_id = int(out[0])
        return new_id, ((int(block), new_id) if copied[0] else None)

    def import_tables(self, block_tables: np.ndarray, num_table_blocks: np.ndarray) -> None:
        bt = np.ascontiguousarray(block_tables, dtype=np.int32)
        nb = np.ascontiguousarray(num_table_blocks, dtype=np.int32)
        check("pa_pool_import", load().pa_pool_import(self._h, _ptr(bt), bt.shape[0], bt.shape[1], _ptr(nb)))

    def prepare_decode(self, block_tables: np.ndarray, num_table_blocks: np.ndarray, context_lens):
        """One decode step's host work; updates block_tables / num_table_blocks in place.

        Returns (slot_mapping int64 [B], src_dst_pairs int64 [P, 2]).
        """
        if block_tables.dtype != np.int32 or not block_tables.flags.c_contiguous:
            raise TypeError("block_tables must be a C-contiguous int32 array (updated in place)")
        if num_table_blocks.dtype != np.int32 or not num_table_blocks.flags.c_contiguous:
            raise TypeError("num_table_blocks must be a C-contiguous int32 array (updated in place)")
        ctx = np.ascontiguousarray(context_lens, dtype=np.int32)
        B = ctx.shape[0]
        slots = np.empty(max(B, 1), dtype=np.int64)
        pairs = np.empty((max(B, 1), 2), dtype=np.int64)
        n = ctypes.c_int(0)
        check("pa_pool_prepare_decode", load().pa_pool_prepare_decode(
            self._h, B, _ptr(block_tables), block_tables.shape[1], _ptr(num_table_blocks), _ptr(ctx),
            _ptr(slots), _ptr(pairs), ctypes.byref(n)))
        return slots[:B], pairs[:n.value].copy()

    def free_table(self, table) -> None:
        ids = np.ascontiguousarray(table, dtype=np.int32)
        check("pa_pool_free_table", load().pa_pool_free_table(self._h, _ptr(ids), int(ids.size)))

    # ---- prefix caching ----------------------------------------------------------
    def allocate_prompt_cached(self, token_ids, max_blocks: int | None = None):
        """Table for a prompt, reusing registered full blocks of an equal prefix.

        Returns (table, num_cached_tokens)."""
        toks = np.ascontiguousarray(token_ids, dtype=np.int32)
        n_all = -(-toks.size // self.block_size)
        cap = n_all if max_blocks is None else int(max_blocks)
        table = np.empty(max(cap, 1), dtype=np.int32)
        nb = ctypes.c_int(0)
        cached = ctypes.c_int(0)
        check("pa_pool_allocate_prompt_cached", load().pa_pool_allocate_prompt_cached(
            self._h, _ptr(toks), int(toks.size), _ptr(table), cap, ctypes.byref(nb), ctypes.byref(cached)))
        return table[:nb.value].tolist(), cached.value

    def num_cached_blocks(self) -> int:
        return int(load().pa_pool_num_cached_blocks(self._h))


def swap_plan(src: BlockPool, dst: BlockPool, table):
    """pa_pool_swap_plan: move a table's blocks from `src` to `dst`.

    Returns (new_table, src_dst_pairs int64 [P, 2])."""
    t = np.ascontiguousarray(table, dtype=np.int32).copy()
    pairs = np.empty((max(t.size, 1), 2), dtype=np.int64)
    n = ctypes.c_int(0)
    check("pa_pool_swap_plan", load().pa_pool_swap_plan(src._h, dst._h, _ptr(t), int(t.size), _ptr(pairs),
                                                        ctypes.byref(n)))
    return t.tolist(), pairs[:n.value].copy()


def block_hash(parent_hash: int, token_ids) -> int:
    """pa_block_hash: chained FNV-1a-64 of a block's tokens."""
    toks = np.ascontiguousarray(token_ids, dtype=np.int32)
    return int(load().pa_block_hash(ctypes.c_uint64(parent_hash), _ptr(toks), int(toks.size)))
