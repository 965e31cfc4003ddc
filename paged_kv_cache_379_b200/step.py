"""One decode step of the paged-KV hot path on a device-resident batch.

A step is:  slot mapping (a1)  ->  copy-on-write block copies (a3, if any)
            ->  cache write of the new tokens (a2)  ->  decode attention (a4, or
            the partition kernel a5 + log-sum-exp reduce a6); a1-a3 run as one
            launch (a1 + a2, or a1 + a2 + a3 given per-sequence copy sources).
Every stage is one call of the C ABI; this module only moves arrays to the
device and sequences the calls on one stream.  The host-side block-pool work
of a step (a7: growth and copy-on-write decisions) is `host_step`.
"""

from __future__ import annotations

import numpy as np
import torch

from . import ops
from .pool import BlockPool
from .workload import Workload


def bf16_to_device(bits: np.ndarray, device) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.to(device).view(torch.bfloat16)


def bf16_to_host_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().view(torch.int16).cpu().numpy().view(np.uint16)


def host_step(wl: Workload, fork_all: bool = False, pool_factory=BlockPool):
    """The block pool's work for one decode step of `wl` (host only).

    The pool adopts the workload's tables; with fork_all every sequence first
    gains a second owner of all its blocks (a retained parent snapshot, as in
    parallel sampling), so a write into an existing block copies it.  Each
    sequence then appends its token at position seq_len - 1.
    Returns (pool, tables, blocks_per_seq, slots, pairs).
    """
    tables = np.ascontiguousarray(wl.block_tables, dtype=np.int32).copy()
    nblk = np.ascontiguousarray(wl.blocks_per_seq, dtype=np.int32).copy()
    # Initial free stack: owned blocks first (import removes them), then the
    # workload's unowned blocks reversed, so they are handed out in drawn order.
    unowned = np.asarray(wl.free_blocks, dtype=np.int32)
    is_free = np.zeros(wl.num_blocks, dtype=bool)
    is_free[unowned] = True
    owned = np.flatnonzero(~is_free).astype(np.int32)
    full_order = np.concatenate([owned, unowned[::-1]])
    pool = pool_factory(wl.num_blocks, wl.block_size, free_order=full_order)
    pool.import_tables(tables, nblk)
    if fork_all:
        for s in range(wl.num_seqs):
            pool.fork(tables[s, :nblk[s]])
    slots, pairs = pool.prepare_decode(tables, nblk, wl.seq_lens.astype(np.int64) - 1)
    return pool, tables, nblk, slots, pairs


class DecodeBatch:
    """Device copies of a workload plus the buffers a step writes."""

    def __init__(self, wl: Workload, device="cuda", tables: np.ndarray | None = None,
                 pairs: np.ndarray | None = None, workspace: bool = True, cow_src: np.ndarray | None = None):
        self.wl = wl
        self.device = torch.device(device)
        self.key_cache = bf16_to_device(wl.key_cache, self.device)
        self.value_cache = bf16_to_device(wl.value_cache, self.device)
        tb = wl.block_tables if tables is None else tables
        self.block_tables = torch.from_numpy(np.ascontiguousarray(tb, dtype=np.int32)).to(self.device)
        self.seq_lens = torch.from_numpy(wl.seq_lens.astype(np.int32)).to(self.device)
        self.query = bf16_to_device(wl.query, self.device)
        self.new_key = bf16_to_device(wl.new_key, self.device)
        self.new_value = bf16_to_device(wl.new_value, self.device)
        self.slots = torch.empty(wl.num_seqs, dtype=torch.int64, device=self.device)
        self.out = torch.empty_like(self.query)
        self.pairs = None
        if pairs is not None and len(pairs):
            self.pairs = torch.from_numpy(np.ascontiguousarray(pairs, dtype=np.int64)).to(self.device)
        # per-sequence copy sources: the step's copies run fused with its cache write
        self.cow_src = None
        if cow_src is not None:
            self.cow_src = torch.from_numpy(np.ascontiguousarray(cow_src, dtype=np.int32)).to(self.device)
        self.max_seq_len = wl.max_seq_len
        self.workspace = None
        if workspace:
            self.workspace = ops.new_workspace(wl.num_seqs, wl.num_heads, wl.num_kv_heads, wl.head_dim, self.max_seq_len,
                                               device=self.device)

    def run_step(self, stream=None, decode_fn=None):
        """Copy-on-write copies (if any), then the newest token's slot and cache
        write in one launch, then the decode.  With per-sequence copy sources
        the copies and the cache write are one launch."""
        wl = self.wl
        if self.cow_src is not None:
            ops.append_decode_kv_cow(self.new_key, self.new_value, self.key_cache, self.value_cache,
                                     self.block_tables, self.seq_lens, self.cow_src, slot_mapping=self.slots,
                                     stream=stream)
        else:
            if self.pairs is not None:
                ops.copy_blocks(self.key_cache, self.value_cache, self.pairs, stream=stream)
            ops.append_decode_kv(self.new_key, self.new_value, self.key_cache, self.value_cache, self.block_tables,
                                 self.seq_lens, slot_mapping=self.slots, stream=stream)
        if decode_fn is None:
            ops.decode(self.query, self.key_cache, self.value_cache, self.block_tables, self.seq_lens,
                       wl.scale, self.max_seq_len, out=self.out, workspace=self.workspace, stream=stream)
        else:
            decode_fn(self)
        return self.out
