"""Python binding of the C ABI: the same names, argument marshalling only.

Each function checks dtypes / devices / contiguity of the torch tensors it is
given, passes their device pointers and the current CUDA stream to the
library, and raises :class:`PagedKVError` on a negative status.  Every step of
the computation runs in the library's CUDA kernels; nothing here computes.

Tensor conventions (see include/pagedkv.h):
  key_cache, value_cache : bf16 [num_blocks, block_size, num_kv_heads, head_dim]
  query, out             : bf16 [num_seqs, num_heads, head_dim]
  block_tables           : int32 [num_seqs, max_blocks_per_seq]
  seq_lens               : int32 [num_seqs]
  slot_mapping           : int64 [num_tokens]
  src_dst_pairs          : int64 [num_pairs, 2]
  FP8 caches             : uint8 E4M3 codes [num_blocks, block_size, num_kv_heads, head_dim]
                           with one fp32 scale per cache (k_scale, v_scale)
"""

from __future__ import annotations

import ctypes

import numpy as np
import torch

from ._lib import PagedKVError, check, load  # noqa: F401

# First bytes of every decode workspace: the dynamic scheduler's counters.
WORKSPACE_HEADER_BYTES = 256

__all__ = [
    "slot_mapping", "reshape_and_cache", "copy_blocks", "decode", "decode_one_pass",
    "decode_split", "decode_partitions", "lse_reduce", "decode_workspace_size", "decode_plan",
    "validate_tables", "device_status", "PagedKVError", "new_workspace", "workspace_views",
    "decode_split_noalloc", "swap_blocks", "reshape_and_cache_fp8", "decode_fp8", "decode_fp8_split",
    "prefill", "append_decode_kv", "append_decode_kv_fp8", "selftest_bounded_wait", "append_decode_kv_cow",
    "cow_sources", "prefix_groups", "decode_shared",
]


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dev(t: torch.Tensor | None, dtype, name: str, ndim: int | None = None):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {tuple(t.shape)}")
    return t.data_ptr()


def _cache_dims(key_cache, value_cache, dtype=torch.bfloat16):
    _dev(key_cache, dtype, "key_cache", 4)
    _dev(value_cache, dtype, "value_cache", 4)
    if key_cache.shape != value_cache.shape:
        raise ValueError("key_cache and value_cache shapes differ")
    nb, bs, hkv, d = key_cache.shape
    return nb, bs, hkv, d


def slot_mapping(block_tables, block_size: int, *, seq_lens=None, positions=None, seq_ids=None,
                 out=None, stream=None):
    """Device address translation; decode form (positions=None) uses pos = seq_len - 1."""
    lib = load()
    bt = _dev(block_tables, torch.int32, "block_tables", 2)
    n = positions.shape[0] if positions is not None else (
        seq_ids.shape[0] if seq_ids is not None else seq_lens.shape[0])
    if out is None:
        out = torch.empty(n, dtype=torch.int64, device=block_tables.device)
    check("pa_slot_mapping", lib.pa_slot_mapping(
        _dev(out, torch.int64, "out", 1), bt, block_tables.shape[0], block_tables.shape[1],
        _dev(seq_ids, torch.int32, "seq_ids", 1),
        _dev(positions, torch.int64, "positions", 1), _dev(seq_lens, torch.int32, "seq_lens", 1),
        n, int(block_size), _stream(stream)))
    return out


def reshape_and_cache(key, value, key_cache, value_cache, slot_mapping, stream=None) -> None:
    lib = load()
    nb, bs, hkv, d = _cache_dims(key_cache, value_cache)
    k = _dev(key, torch.bfloat16, "key", 3)
    v = _dev(value, torch.bfloat16, "value", 3)
    if tuple(key.shape[1:]) != (hkv, d) or key.shape != value.shape:
        raise ValueError("key/value must be [num_tokens, num_kv_heads, head_dim] matching the cache")
    sm = _dev(slot_mapping, torch.int64, "slot_mapping", 1)
    if slot_mapping.shape[0] != key.shape[0]:
        raise ValueError("slot_mapping length != num_tokens")
    check("pa_reshape_and_cache", lib.pa_reshape_and_cache(
        k, v, key_cache.data_ptr(), value_cache.data_ptr(), sm, key.shape[0], hkv, d, bs, nb,
        _stream(stream)))


def reshape_and_cache_fp8(key, value, key_cache, value_cache, slot_mapping, k_scale: float, v_scale: float,
                          stream=None) -> None:
    """pa_reshape_and_cache_fp8: bf16 rows quantised to E4M3 codes in uint8 caches."""
    lib = load()
    nb, bs, hkv, d = _cache_dims(key_cache, value_cache, torch.uint8)
    k = _dev(key, torch.bfloat16, "key", 3)
    v = _dev(value, torch.bfloat16, "value", 3)
    if tuple(key.shape[1:]) != (hkv, d) or key.shape != value.shape:
        raise ValueError("key/value must be [num_tokens, num_kv_heads, head_dim] matching the cache")
    sm = _dev(slot_mapping, torch.int64, "slot_mapping", 1)
    if slot_mapping.shape[0] != key.shape[0]:
        raise ValueError("slot_mapping length != num_tokens")
    check("pa_reshape_and_cache_fp8", lib.pa_reshape_and_cache_fp8(
        k, v, key_cache.data_ptr(), value_cache.data_ptr(), sm, key.shape[0], hkv, d, bs, nb, float(k_scale),
        float(v_scale), _stream(stream)))


def _append_args(key, value, key_cache, value_cache, block_tables, seq_lens, slot_mapping, cache_dtype):
    nb, bs, hkv, d = _cache_dims(key_cache, value_cache, cache_dtype)
    k = _dev(key, torch.bfloat16, "key", 3)
    v = _dev(value, torch.bfloat16, "value", 3)
    B = seq_lens.shape[0]
    if tuple(key.shape) != (B, hkv, d) or key.shape != value.shape:
        raise ValueError("key/value must be [num_seqs, num_kv_heads, head_dim] matching the cache")
    bt = _dev(block_tables, torch.int32, "block_tables", 2)
    if block_tables.shape[0] != B:
        raise ValueError("block_tables rows != num_seqs")
    sm = _dev(slot_mapping, torch.int64, "slot_mapping", 1)
    return (k, v, key_cache.data_ptr(), value_cache.data_ptr(), bt, _dev(seq_lens, torch.int32, "seq_lens", 1), sm,
            B, block_tables.shape[1], hkv, d, bs, nb)


def append_decode_kv(key, value, key_cache, value_cache, block_tables, seq_lens, slot_mapping=None,
                     stream=None) -> None:
    """pa_append_decode_kv: slot of each sequence's newest position + cache write, one launch."""
    a = _append_args(key, value, key_cache, value_cache, block_tables, seq_lens, slot_mapping, torch.bfloat16)
    check("pa_append_decode_kv", load().pa_append_decode_kv(*a, _stream(stream)))


def append_decode_kv_cow(key, value, key_cache, value_cache, block_tables, seq_lens, cow_src, slot_mapping=None,
                         stream=None) -> None:
    """pa_append_decode_kv_cow: the step's copy-on-write copies and cache write,
    one launch; cow_src int32 [num_seqs] (device): the block each sequence's
    write block is a copy of, or -1 (see cow_sources)."""
    a = _append_args(key, value, key_cache, value_cache, block_tables, seq_lens, slot_mapping, torch.bfloat16)
    cs = _dev(cow_src, torch.int32, "cow_src", 1)
    if cow_src is not None and cow_src.shape[0] != seq_lens.shape[0]:
        raise ValueError("cow_src length != num_seqs")
    check("pa_append_decode_kv_cow", load().pa_append_decode_kv_cow(*a[:6], cs, *a[6:], _stream(stream)))


def cow_sources(slot_mapping, block_size: int, src_dst_pairs) -> np.ndarray:
    """pa_cow_sources (host): per-sequence copy source of the block each slot
    lies in, from the pool's (src, dst) pairs; -1 where none."""
    slots = np.ascontiguousarray(slot_mapping, dtype=np.int64)
    pairs = np.ascontiguousarray(src_dst_pairs, dtype=np.int64).reshape(-1, 2)
    out = np.empty(slots.shape[0], dtype=np.int32)
    check("pa_cow_sources", load().pa_cow_sources(
        slots.ctypes.data_as(ctypes.c_void_p), int(slots.shape[0]), int(block_size),
        pairs.ctypes.data_as(ctypes.c_void_p), int(pairs.shape[0]), out.ctypes.data_as(ctypes.c_void_p)))
    return out


def prefix_groups(block_tables, seq_lens, block_size: int, partition_size: int):
    """pa_prefix_groups (host): runs of consecutive sequences sharing leading
    partitions.  Returns (group_start int32 [G+1], group_parts int32 [G])."""
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    B = int(sl.shape[0])
    start = np.empty(B + 1, dtype=np.int32)
    parts = np.empty(max(B, 1), dtype=np.int32)
    n = ctypes.c_int(0)
    check("pa_prefix_groups", load().pa_prefix_groups(
        bt.ctypes.data_as(ctypes.c_void_p), B, int(bt.shape[1]) if bt.ndim == 2 else 1,
        sl.ctypes.data_as(ctypes.c_void_p), int(block_size), int(partition_size),
        start.ctypes.data_as(ctypes.c_void_p), parts.ctypes.data_as(ctypes.c_void_p), ctypes.byref(n)))
    return start[:n.value + 1].copy(), parts[:n.value].copy()


def append_decode_kv_fp8(key, value, key_cache, value_cache, block_tables, seq_lens, k_scale: float,
                         v_scale: float, slot_mapping=None, stream=None) -> None:
    """pa_append_decode_kv_fp8: as append_decode_kv into E4M3 code caches."""
    a = _append_args(key, value, key_cache, value_cache, block_tables, seq_lens, slot_mapping, torch.uint8)
    check("pa_append_decode_kv_fp8", load().pa_append_decode_kv_fp8(*a, float(k_scale), float(v_scale),
                                                                    _stream(stream)))


def copy_blocks(key_cache, value_cache, src_dst_pairs, stream=None) -> None:
    lib = load()
    nb, bs, hkv, d = _cache_dims(key_cache, value_cache)
    pr = _dev(src_dst_pairs, torch.int64, "src_dst_pairs", 2)
    if src_dst_pairs.shape[1] != 2:
        raise ValueError("src_dst_pairs must be [num_pairs, 2]")
    check("pa_copy_blocks", lib.pa_copy_blocks(
        key_cache.data_ptr(), value_cache.data_ptr(), pr, src_dst_pairs.shape[0], hkv, d, bs, nb,
        _stream(stream)))


def swap_blocks(dst_key_cache, dst_value_cache, src_key_cache, src_value_cache, src_dst_pairs, stream=None) -> None:
    """pa_swap_blocks: block copies between a device cache and a pinned host cache (either way).

    Host-side tensors must be pinned (``tensor.pin_memory()``); ``src_dst_pairs``
    is an int64 [P, 2] tensor in device or pinned host memory."""
    lib = load()
    for name, t in (("dst_key_cache", dst_key_cache), ("dst_value_cache", dst_value_cache),
                    ("src_key_cache", src_key_cache), ("src_value_cache", src_value_cache)):
        if t.dtype != torch.bfloat16 or not t.is_contiguous() or t.dim() != 4:
            raise ValueError(f"{name} must be a contiguous bf16 [num_blocks, block_size, heads, head_dim] tensor")
        if not t.is_cuda and not t.is_pinned():
            raise ValueError(f"{name} must be a CUDA tensor or pinned host memory")
    if src_key_cache.shape[1:] != dst_key_cache.shape[1:] or src_key_cache.shape != src_value_cache.shape or \
            dst_key_cache.shape != dst_value_cache.shape:
        raise ValueError("cache shapes do not match")
    if src_dst_pairs.dtype != torch.int64 or src_dst_pairs.dim() != 2 or src_dst_pairs.shape[1] != 2 or \
            not src_dst_pairs.is_contiguous():
        raise ValueError("src_dst_pairs must be a contiguous int64 [P, 2] tensor")
    _, bs, hkv, d = src_key_cache.shape
    check("pa_swap_blocks", lib.pa_swap_blocks(
        dst_key_cache.data_ptr(), dst_value_cache.data_ptr(), src_key_cache.data_ptr(), src_value_cache.data_ptr(),
        src_dst_pairs.data_ptr(), src_dst_pairs.shape[0], hkv, d, bs, src_key_cache.shape[0],
        dst_key_cache.shape[0], _stream(stream)))


def _decode_common(query, key_cache, value_cache, block_tables, seq_lens, cache_dtype=torch.bfloat16):
    nb, bs, hkv, d = _cache_dims(key_cache, value_cache, cache_dtype)
    q = _dev(query, torch.bfloat16, "query", 3)
    B, hq, dq = query.shape
    if dq != d:
        raise ValueError("query head_dim != cache head_dim")
    bt = _dev(block_tables, torch.int32, "block_tables", 2)
    sl = _dev(seq_lens, torch.int32, "seq_lens", 1)
    if block_tables.shape[0] != B or seq_lens.shape[0] != B:
        raise ValueError("block_tables / seq_lens batch size != query batch size")
    return q, bt, sl, B, hq, hkv, d, bs, nb, block_tables.shape[1]


def decode_workspace_size(num_seqs: int, num_heads: int, num_kv_heads: int, head_dim: int, max_seq_len: int,
                          partition_size: int = 0) -> int:
    """Bytes of decode workspace; partition_size 0 = what pa_decode would choose."""
    return int(load().pa_decode_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim, max_seq_len,
                                               partition_size))


def decode_plan(num_seqs: int, num_heads: int, num_kv_heads: int, head_dim: int, max_seq_len: int,
                workspace_bytes: int) -> int:
    """0 if pa_decode runs one pass for these sizes, else the split partition size."""
    return int(load().pa_decode_plan(num_seqs, num_heads, num_kv_heads, head_dim, max_seq_len,
                                     int(workspace_bytes)))


def _out(out, query):
    if out is None:
        out = torch.empty_like(query)
    return _dev(out, torch.bfloat16, "out", 3), out


def _ws(workspace):
    if workspace is None:
        return None, 0
    if not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    return workspace.data_ptr(), workspace.numel() * workspace.element_size()


def decode(query, key_cache, value_cache, block_tables, seq_lens, scale: float, max_seq_len: int,
           *, out=None, workspace=None, stream=None):
    """pa_decode: one pass or split, chosen by the library."""
    lib = load()
    q, bt, sl, B, hq, hkv, d, bs, nb, mb = _decode_common(query, key_cache, value_cache, block_tables, seq_lens)
    o, out = _out(out, query)
    wp, wb = _ws(workspace)
    check("pa_decode", lib.pa_decode(o, q, key_cache.data_ptr(), value_cache.data_ptr(), bt, sl, float(scale),
                                     bs, hkv, B, hq, d, mb, nb, int(max_seq_len), wp, wb, _stream(stream)))
    return out


def decode_fp8(query, key_cache, value_cache, block_tables, seq_lens, scale: float, k_scale: float,
               v_scale: float, max_seq_len: int, *, out=None, workspace=None, stream=None):
    """pa_decode_fp8: pa_decode over uint8 E4M3 caches with per-tensor scales."""
    lib = load()
    q, bt, sl, B, hq, hkv, d, bs, nb, mb = _decode_common(query, key_cache, value_cache, block_tables, seq_lens,
                                                          torch.uint8)
    o, out = _out(out, query)
    wp, wb = _ws(workspace)
    check("pa_decode_fp8", lib.pa_decode_fp8(
        o, q, key_cache.data_ptr(), value_cache.data_ptr(), bt, sl, float(scale), float(k_scale), float(v_scale),
        bs, hkv, B, hq, d, mb, nb, int(max_seq_len), wp, wb, _stream(stream)))
    return out


def decode_fp8_split(query, key_cache, value_cache, block_tables, seq_lens, scale: float, k_scale: float,
                     v_scale: float, max_seq_len: int, partition_size: int, workspace=None, *, out=None,
                     stream=None):
    """pa_decode_fp8_split: partition_size 0 = one pass, else the split form."""
    lib = load()
    q, bt, sl, B, hq, hkv, d, bs, nb, mb = _decode_common(query, key_cache, value_cache, block_tables, seq_lens,
                                                          torch.uint8)
    o, out = _out(out, query)
    wp, wb = _ws(workspace)
    check("pa_decode_fp8_split", lib.pa_decode_fp8_split(
        o, q, key_cache.data_ptr(), value_cache.data_ptr(), bt, sl, float(scale), float(k_scale), float(v_scale),
        bs, hkv, B, hq, d, mb, nb, int(max_seq_len), int(partition_size), wp, wb, _stream(stream)))
    return out


def prefill(query, key_cache, value_cache, block_tables, seq_lens, q_start, scale: float, *, out=None,
            stream=None):
    """pa_prefill: causal multi-query attention of each sequence's chunk (query rows
    q_start[s] .. q_start[s+1]-1, the last positions of the sequence) over its paged cache."""
    if not (float(scale) > 0.0 and float(scale) < float("inf")):
        raise ValueError("scale must be positive and finite")
    lib = load()
    nb, bs, hkv, d = _cache_dims(key_cache, value_cache)
    q = _dev(query, torch.bfloat16, "query", 3)
    T, hq, dq = query.shape
    if dq != d:
        raise ValueError("query head_dim != cache head_dim")
    bt = _dev(block_tables, torch.int32, "block_tables", 2)
    sl = _dev(seq_lens, torch.int32, "seq_lens", 1)
    qs = _dev(q_start, torch.int32, "q_start", 1)
    B = seq_lens.shape[0]
    if block_tables.shape[0] != B or q_start.shape[0] != B + 1:
        raise ValueError("block_tables rows / q_start length do not match seq_lens")
    o, out = _out(out, query)
    check("pa_prefill", lib.pa_prefill(o, q, key_cache.data_ptr(), value_cache.data_ptr(), bt, sl, qs,
                                       float(scale), bs, hkv, B, hq, d, block_tables.shape[1], nb, T,
                                       _stream(stream)))
    return out


def decode_one_pass(query, key_cache, value_cache, block_tables, seq_lens, scale: float, max_seq_len: int,
                    *, out=None, stream=None):
    lib = load()
    q, bt, sl, B, hq, hkv, d, bs, nb, mb = _decode_common(query, key_cache, value_cache, block_tables, seq_lens)
    o, out = _out(out, query)
    check("pa_decode_one_pass", lib.pa_decode_one_pass(
        o, q, key_cache.data_ptr(), value_cache.data_ptr(), bt, sl, float(scale), bs, hkv, B, hq, d, mb, nb,
        int(max_seq_len), _stream(stream)))
    return out


def decode_split(query, key_cache, value_cache, block_tables, seq_lens, scale: float, max_seq_len: int,
                 partition_size: int, workspace, *, out=None, stream=None):
    lib = load()
    q, bt, sl, B, hq, hkv, d, bs, nb, mb = _decode_common(query, key_cache, value_cache, block_tables, seq_lens)
    o, out = _out(out, query)
    wp, wb = _ws(workspace)
    check("pa_decode_split", lib.pa_decode_split(
        o, q, key_cache.data_ptr(), value_cache.data_ptr(), bt, sl, float(scale), bs, hkv, B, hq, d, mb, nb,
        int(max_seq_len), int(partition_size), wp, wb, _stream(stream)))
    return out


def decode_shared(query, key_cache, value_cache, block_tables, seq_lens, scale: float, max_seq_len: int,
                  partition_size: int, group_start, group_parts, workspace, *, out=None, stream=None):
    """pa_decode_shared: the split decode with shared-prefix groups (int32 device
    tensors group_start [G+1], group_parts [G]; see prefix_groups)."""
    lib = load()
    q, bt, sl, B, hq, hkv, d, bs, nb, mb = _decode_common(query, key_cache, value_cache, block_tables, seq_lens)
    o, out = _out(out, query)
    wp, wb = _ws(workspace)
    gs = _dev(group_start, torch.int32, "group_start", 1)
    gp = _dev(group_parts, torch.int32, "group_parts", 1)
    ng = int(group_parts.shape[0])
    if group_start.shape[0] != ng + 1:
        raise ValueError("group_start must have num_groups + 1 entries")
    check("pa_decode_shared", lib.pa_decode_shared(
        o, q, key_cache.data_ptr(), value_cache.data_ptr(), bt, sl, float(scale), bs, hkv, B, hq, d, mb, nb,
        int(max_seq_len), int(partition_size), gs, gp, ng, wp, wb, _stream(stream)))
    return out


# Bytes of the fixed scratch array inside the library (PA_NOALLOC_SCRATCH_BYTES).
NOALLOC_SCRATCH_BYTES = 16 << 20


def decode_split_noalloc(query, key_cache, value_cache, block_tables, seq_lens, scale: float, max_seq_len: int,
                         partition_size: int, *, out=None, stream=None):
    """pa_decode_split_noalloc: the split form with the library's own fixed scratch.

    For callers that cannot provide a workspace (see include/pagedkv.h).  Raises
    PagedKVError(PA_ERR_SCRATCH_TOO_SMALL) if the problem needs more than
    NOALLOC_SCRATCH_BYTES of split workspace.  Calls must not overlap on the GPU.
    """
    lib = load()
    q, bt, sl, B, hq, hkv, d, bs, nb, mb = _decode_common(query, key_cache, value_cache, block_tables, seq_lens)
    o, out = _out(out, query)
    check("pa_decode_split_noalloc", lib.pa_decode_split_noalloc(
        o, q, key_cache.data_ptr(), value_cache.data_ptr(), bt, sl, float(scale), bs, hkv, B, hq, d, mb, nb,
        int(max_seq_len), int(partition_size), _stream(stream)))
    return out


def decode_partitions(query, key_cache, value_cache, block_tables, seq_lens, scale: float, max_seq_len: int,
                      partition_size: int, workspace, stream=None):
    """pa_decode_partitions; returns views (o, m, l) into the workspace."""
    lib = load()
    q, bt, sl, B, hq, hkv, d, bs, nb, mb = _decode_common(query, key_cache, value_cache, block_tables, seq_lens)
    wp, wb = _ws(workspace)
    check("pa_decode_partitions", lib.pa_decode_partitions(
        q, key_cache.data_ptr(), value_cache.data_ptr(), bt, sl, float(scale), bs, hkv, B, hq, d, mb, nb,
        int(max_seq_len), int(partition_size), wp, wb, _stream(stream)))
    return workspace_views(workspace, B, hq, d, max_seq_len, partition_size)


def workspace_views(workspace, num_seqs, num_heads, head_dim, max_seq_len, partition_size):
    """(o, m, l) float32 views of a split-form workspace (layout of include/pagedkv.h)."""
    parts = max(1, -(-int(max_seq_len) // int(partition_size)))
    rows = num_seqs * num_heads * parts
    a256 = lambda x: (x + 255) // 256 * 256  # noqa: E731
    raw = workspace.view(torch.uint8)[WORKSPACE_HEADER_BYTES:]
    ob = rows * head_dim * 4
    o = raw[:ob].view(torch.float32).view(num_seqs, num_heads, parts, head_dim)
    m = raw[a256(ob):a256(ob) + rows * 4].view(torch.float32).view(num_seqs, num_heads, parts)
    lo = a256(ob) + a256(rows * 4)
    l = raw[lo:lo + rows * 4].view(torch.float32).view(num_seqs, num_heads, parts)
    return o, m, l


def new_workspace(num_seqs: int, num_heads: int, num_kv_heads: int, head_dim: int, max_seq_len: int,
                  partition_size: int = 0, device="cuda"):
    """A zero-filled decode workspace (the scheduler counters must start at zero)."""
    nbytes = decode_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim, max_seq_len, partition_size)
    return torch.zeros(max(nbytes, WORKSPACE_HEADER_BYTES), dtype=torch.uint8, device=device)


def lse_reduce(out, workspace, seq_lens, max_seq_len: int, partition_size: int, stream=None):
    lib = load()
    o = _dev(out, torch.bfloat16, "out", 3)
    B, hq, d = out.shape
    wp, _ = _ws(workspace)
    check("pa_lse_reduce", lib.pa_lse_reduce(o, wp, _dev(seq_lens, torch.int32, "seq_lens", 1), B, hq, d,
                                             int(max_seq_len), int(partition_size), _stream(stream)))
    return out


def validate_tables(block_tables, seq_lens, block_size: int, num_blocks: int, max_seq_len: int,
                    stream=None) -> int:
    """Number of sequences breaking a decode precondition (synchronises)."""
    lib = load()
    bad = torch.zeros(1, dtype=torch.int32, device=block_tables.device)
    check("pa_validate_tables", lib.pa_validate_tables(
        _dev(block_tables, torch.int32, "block_tables", 2), _dev(seq_lens, torch.int32, "seq_lens", 1),
        block_tables.shape[0], block_tables.shape[1], int(block_size), int(num_blocks), int(max_seq_len),
        bad.data_ptr(), _stream(stream)))
    return int(bad.item())


def selftest_bounded_wait(stream=None) -> None:
    """Launch one device wait that nothing satisfies; it gives up after about a
    second and leaves PA_ERR_DEVICE_TIMEOUT for device_status() to report."""
    check("pa_selftest_bounded_wait", load().pa_selftest_bounded_wait(_stream(stream)))


def device_status() -> int:
    """0, or a negative status: PA_ERR_DEVICE_TIMEOUT (-9) if a bounded device wait
    gave up, PA_ERR_VALUE_RANGE (-12) if the prefill read a value entry beyond the
    fp16 range of its P.V operand.  Reading clears it."""
    return int(load().pa_device_status())
