"""The oracle: a plain, slow, fp64 CPU restatement of the paged-KV decode path.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this package.  The product package
(``paged_kv_cache_379_b200``) never imports it, and it never imports the
product: the two share no code.  The C part (``oracle.c``) is compiled with gcc
into ``liboracle.so`` beside it by :func:`build`.

Functions, each restating a passage of the pages (see ``oracle.c`` and
``pool.py`` for the citations):

* :func:`slot_mapping`      -- address translation pos -> physical slot
* :func:`reshape_and_cache` -- write new K/V rows at their slots
* :func:`copy_blocks`       -- copy-on-write block copies
* :func:`swap_blocks`       -- whole-block copies between a GPU and a host cache
* :func:`paged_decode`      -- softmax(scale * q K^T) V, K/V gathered through the table
* :func:`paged_decode_partials`, :func:`lse_merge` -- the split form and its merge
* :func:`reshape_and_cache_fp8`, :func:`paged_decode_fp8` -- the same over an E4M3 cache
* :class:`pool.OraclePool`  -- free list, reference counts, fork, copy-on-write
"""

from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c with gcc (fp64, -O2, OpenMP) into liboracle.so."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        I = ctypes.c_int
        lib.oracle_slot_mapping.argtypes = [P, I, P, P, I, I, P]
        lib.oracle_slot_mapping.restype = I
        lib.oracle_reshape_and_cache.argtypes = [P, P, P, P, P, I, I, I, I]
        lib.oracle_reshape_and_cache.restype = None
        lib.oracle_copy_blocks.argtypes = [P, P, P, I, I, I, I]
        lib.oracle_copy_blocks.restype = None
        lib.oracle_swap_blocks.argtypes = [P, P, P, P, P, I, I, I, I]
        lib.oracle_swap_blocks.restype = None
        lib.oracle_paged_decode.argtypes = [P, P, P, P, P, P, ctypes.c_double, I, I, I, I, I, I, I]
        lib.oracle_paged_decode.restype = None
        lib.oracle_paged_decode_partials.argtypes = [P, P, P, P, P, P, P, P, ctypes.c_double,
                                                     I, I, I, I, I, I, I, I]
        lib.oracle_paged_decode_partials.restype = None
        lib.oracle_lse_merge.argtypes = [P, P, P, P, I, I, I]
        lib.oracle_lse_merge.restype = None
        lib.oracle_e4m3_to_f64.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_to_f64.restype = ctypes.c_double
        lib.oracle_f64_to_e4m3.argtypes = [ctypes.c_double]
        lib.oracle_f64_to_e4m3.restype = ctypes.c_uint8
        lib.oracle_reshape_and_cache_fp8.argtypes = [P, P, P, P, P, I, I, I, I, ctypes.c_float, ctypes.c_float]
        lib.oracle_reshape_and_cache_fp8.restype = None
        lib.oracle_paged_decode_fp8.argtypes = [P, P, P, P, P, P, ctypes.c_double, ctypes.c_double,
                                                ctypes.c_double, I, I, I, I, I, I, I]
        lib.oracle_paged_decode_fp8.restype = None
        lib.oracle_paged_prefill.argtypes = [P, P, P, P, P, P, P, ctypes.c_double, I, I, I, I, I, I, I]
        lib.oracle_paged_prefill.restype = None
        lib.oracle_num_threads.argtypes = []
        lib.oracle_num_threads.restype = I
        _lib = lib
    return _lib


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a, a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def bf16_bits_to_f64(bits) -> np.ndarray:
    """Exact widening of raw bf16 patterns (uint16) to float64."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def slot_mapping(block_tables, seq_ids, positions, block_size: int) -> np.ndarray:
    lib = _load()
    bt, btp = _c(block_tables, np.int32)
    sid, sidp = _c(seq_ids, np.int32)
    pos, posp = _c(positions, np.int64)
    out = np.empty(pos.shape[0], dtype=np.int64)
    rc = lib.oracle_slot_mapping(btp, bt.shape[1], sidp, posp, pos.shape[0], block_size,
                                 out.ctypes.data_as(ctypes.c_void_p))
    if rc != 0:
        raise ValueError("position outside its block table")
    return out


def reshape_and_cache(key, value, key_cache, value_cache, slots, block_size: int) -> None:
    """In place on key_cache / value_cache (uint16 arrays [nb, bs, Hkv, D])."""
    lib = _load()
    k, kp = _c(key, np.uint16)
    v, vp = _c(value, np.uint16)
    s, sp = _c(slots, np.int64)
    assert key_cache.dtype == np.uint16 and key_cache.flags.c_contiguous
    assert value_cache.dtype == np.uint16 and value_cache.flags.c_contiguous
    T, H, D = k.shape
    lib.oracle_reshape_and_cache(kp, vp, key_cache.ctypes.data_as(ctypes.c_void_p),
                                 value_cache.ctypes.data_as(ctypes.c_void_p), sp, T, H, D, block_size)


def copy_blocks(key_cache, value_cache, pairs) -> None:
    lib = _load()
    pr, prp = _c(np.asarray(pairs, dtype=np.int64).reshape(-1, 2), np.int64)
    nb, bs, H, D = key_cache.shape
    assert key_cache.dtype == np.uint16 and key_cache.flags.c_contiguous
    lib.oracle_copy_blocks(key_cache.ctypes.data_as(ctypes.c_void_p),
                           value_cache.ctypes.data_as(ctypes.c_void_p), prp, pr.shape[0], H, D, bs)


def swap_blocks(dst_key_cache, dst_value_cache, src_key_cache, src_value_cache, pairs) -> None:
    """In place on dst_*: whole-block copies from the src caches."""
    lib = _load()
    pr, prp = _c(np.asarray(pairs, dtype=np.int64).reshape(-1, 2), np.int64)
    sk, skp = _c(src_key_cache, np.uint16)
    sv, svp = _c(src_value_cache, np.uint16)
    for a in (dst_key_cache, dst_value_cache):
        assert a.dtype == np.uint16 and a.flags.c_contiguous
    nb, bs, H, D = sk.shape
    lib.oracle_swap_blocks(dst_key_cache.ctypes.data_as(ctypes.c_void_p),
                           dst_value_cache.ctypes.data_as(ctypes.c_void_p), skp, svp, prp, pr.shape[0], H, D, bs)


def _check_tables(block_tables, seq_lens, block_size: int, num_blocks: int) -> None:
    """The decode's precondition, checked before the C loop reads a block:
    every table entry a sequence uses lies in [0, num_blocks)."""
    bt = np.asarray(block_tables)
    for s, L in enumerate(np.asarray(seq_lens)):
        n = -(-int(L) // block_size) if L > 0 else 0
        if n > bt.shape[1]:
            raise ValueError(f"sequence {s}: {n} blocks needed, table width {bt.shape[1]}")
        used = bt[s, :n]
        if n and (used.min() < 0 or used.max() >= num_blocks):
            raise ValueError(f"sequence {s}: a table entry outside [0, {num_blocks})")


def paged_decode(query, key_cache, value_cache, block_tables, seq_lens, scale: float,
                 threads: int = 1) -> np.ndarray:
    """fp64 [B, Hq, D] output.  query: uint16 bf16 bits [B, Hq, D]."""
    lib = _load()
    q, qp = _c(query, np.uint16)
    kc, kcp = _c(key_cache, np.uint16)
    vc, vcp = _c(value_cache, np.uint16)
    bt, btp = _c(block_tables, np.int32)
    sl, slp = _c(seq_lens, np.int32)
    B, Hq, D = q.shape
    nb, bs, Hkv, D2 = kc.shape
    assert D2 == D and Hq % Hkv == 0 and bt.shape[0] == B and sl.shape[0] == B
    _check_tables(bt, sl, bs, nb)
    out = np.empty((B, Hq, D), dtype=np.float64)
    lib.oracle_paged_decode(out.ctypes.data_as(ctypes.c_void_p), qp, kcp, vcp, btp, slp,
                            float(scale), bs, Hkv, B, Hq, D, bt.shape[1], int(threads))
    return out


def paged_prefill(query, key_cache, value_cache, block_tables, seq_lens, q_lens, scale: float,
                  threads: int = 1) -> np.ndarray:
    """fp64 [T, Hq, D] causal prefill of each sequence's last q_lens[s] positions.

    query: uint16 bf16 bits [T, Hq, D], T = sum(q_lens), rows of sequence s
    consecutive and in position order."""
    lib = _load()
    q, qp = _c(query, np.uint16)
    kc, kcp = _c(key_cache, np.uint16)
    vc, vcp = _c(value_cache, np.uint16)
    bt, btp = _c(block_tables, np.int32)
    sl, slp = _c(seq_lens, np.int32)
    ql = np.asarray(q_lens, dtype=np.int64)
    B = sl.shape[0]
    assert ql.shape == (B,) and (ql >= 0).all() and (ql <= sl).all()
    start = np.zeros(B + 1, dtype=np.int32)
    start[1:] = np.cumsum(ql)
    st, stp = _c(start, np.int32)
    T, Hq, D = q.shape
    nb, bs, Hkv, D2 = kc.shape
    assert T == int(start[-1]) and D2 == D and Hq % Hkv == 0 and bt.shape[0] == B
    out = np.empty((T, Hq, D), dtype=np.float64)
    lib.oracle_paged_prefill(out.ctypes.data_as(ctypes.c_void_p), qp, kcp, vcp, btp, slp, stp, float(scale),
                             bs, Hkv, B, Hq, D, bt.shape[1], int(threads))
    return out


def paged_decode_partials(query, key_cache, value_cache, block_tables, seq_lens, scale: float,
                          partition_size: int, max_parts: int):
    """(m, l, o): m, l [B, Hq, P]; o [B, Hq, P, D] in fp64, natural-log units."""
    lib = _load()
    q, qp = _c(query, np.uint16)
    kc, kcp = _c(key_cache, np.uint16)
    vc, vcp = _c(value_cache, np.uint16)
    bt, btp = _c(block_tables, np.int32)
    sl, slp = _c(seq_lens, np.int32)
    B, Hq, D = q.shape
    nb, bs, Hkv, _ = kc.shape
    m = np.empty((B, Hq, max_parts), dtype=np.float64)
    l = np.empty((B, Hq, max_parts), dtype=np.float64)
    o = np.empty((B, Hq, max_parts, D), dtype=np.float64)
    lib.oracle_paged_decode_partials(m.ctypes.data_as(ctypes.c_void_p), l.ctypes.data_as(ctypes.c_void_p),
                                     o.ctypes.data_as(ctypes.c_void_p), qp, kcp, vcp, btp, slp,
                                     float(scale), bs, Hkv, B, Hq, D, bt.shape[1],
                                     int(partition_size), int(max_parts))
    return m, l, o


def e4m3_to_f64(code: int) -> float:
    return float(_load().oracle_e4m3_to_f64(int(code) & 0xFF))


def f64_to_e4m3(x: float) -> int:
    return int(_load().oracle_f64_to_e4m3(float(x)))


def reshape_and_cache_fp8(key, value, key_cache, value_cache, slots, block_size: int, k_scale: float,
                          v_scale: float) -> None:
    """In place on uint8 E4M3 caches [nb, bs, Hkv, D]; the inverse scales are formed in fp32."""
    lib = _load()
    k, kp = _c(key, np.uint16)
    v, vp = _c(value, np.uint16)
    s, sp = _c(slots, np.int64)
    for a in (key_cache, value_cache):
        assert a.dtype == np.uint8 and a.flags.c_contiguous
    T, H, D = k.shape
    k_inv = float(np.float32(1.0) / np.float32(k_scale))
    v_inv = float(np.float32(1.0) / np.float32(v_scale))
    lib.oracle_reshape_and_cache_fp8(kp, vp, key_cache.ctypes.data_as(ctypes.c_void_p),
                                     value_cache.ctypes.data_as(ctypes.c_void_p), sp, T, H, D, block_size,
                                     k_inv, v_inv)


def paged_decode_fp8(query, key_cache, value_cache, block_tables, seq_lens, scale: float, k_scale: float,
                     v_scale: float, threads: int = 1) -> np.ndarray:
    """fp64 [B, Hq, D] decode over uint8 E4M3 caches (value = e4m3(code) * scale)."""
    lib = _load()
    q, qp = _c(query, np.uint16)
    kc, kcp = _c(key_cache, np.uint8)
    vc, vcp = _c(value_cache, np.uint8)
    bt, btp = _c(block_tables, np.int32)
    sl, slp = _c(seq_lens, np.int32)
    B, Hq, D = q.shape
    nb, bs, Hkv, _ = kc.shape
    out = np.empty((B, Hq, D), dtype=np.float64)
    lib.oracle_paged_decode_fp8(out.ctypes.data_as(ctypes.c_void_p), qp, kcp, vcp, btp, slp, float(scale),
                                float(np.float32(k_scale)), float(np.float32(v_scale)), bs, Hkv, B, Hq, D,
                                bt.shape[1], int(threads))
    return out


def lse_merge(m, l, o) -> np.ndarray:
    lib = _load()
    m, mp = _c(m, np.float64)
    l, lp = _c(l, np.float64)
    o, op = _c(o, np.float64)
    D = o.shape[-1]
    P = m.shape[-1]
    rows = m.size // P
    out = np.empty(m.shape[:-1] + (D,), dtype=np.float64)
    lib.oracle_lse_merge(out.ctypes.data_as(ctypes.c_void_p), mp, lp, op, rows, P, D)
    return out


def allclose_report(gpu, ref, atol: float = 2e-3, rtol: float = 1e-2):
    """Elementwise |gpu - ref| <= atol + rtol*|ref| (the tolerance reading used in the tests).

    Returns (ok, max_abs_err, max_rel_err, worst_index).
    """
    g = np.asarray(gpu, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    err = np.abs(g - r)
    bound = atol + rtol * np.abs(r)
    ok = bool(np.all(err <= bound)) and not np.any(np.isnan(g))
    rel = err / np.maximum(np.abs(r), 1e-30)
    worst = int(np.argmax(err - bound)) if err.size else -1
    return ok, float(err.max(initial=0.0)), float(rel.max(initial=0.0)), worst
