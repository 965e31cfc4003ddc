"""Helpers shared by the GPU parity tests: poisoning, the oracle's version of a
whole decode step, and the tolerance check."""

from __future__ import annotations

import os

import numpy as np

import oracle
from paged_kv_cache_379_b200 import workload as wl

# Attention tolerance: an element passes if |gpu - ref| <= ATOL + RTOL * |ref|
# (max-abs 2e-3 and max-rel 1e-2 read as one allclose bound: bf16 output
# rounding alone is up to 2^-9 relative, so a pure absolute bound of 2e-3 fails
# for |out| >= 1, and a pure relative one fails near 0).
ATOL = 2e-3
RTOL = 1e-2


def poison_tail_slots(w: wl.Workload, tables=None) -> None:
    """bf16 NaN into every slot at or after position seq_len - 1 in each sequence's
    last block: the token being decoded must come from the cache write, and
    unused slots must never be read."""
    tables = w.block_tables if tables is None else tables
    for s in range(w.num_seqs):
        L = int(w.seq_lens[s])
        if L <= 0:
            continue
        last = int(tables[s, (L - 1) // w.block_size])
        off = (L - 1) % w.block_size
        w.key_cache[last, off:] = wl.BF16_NAN
        w.value_cache[last, off:] = wl.BF16_NAN


def oracle_step(w: wl.Workload, tables=None, pairs=None, threads: int = min(32, os.cpu_count() or 1)):
    """The oracle's step: copy pairs, slots of position L-1, cache write, decode.

    Returns (key_cache, value_cache, slots, out fp64)."""
    tables = w.block_tables if tables is None else tables
    kc = w.key_cache.copy()
    vc = w.value_cache.copy()
    if pairs is not None and len(pairs):
        oracle.copy_blocks(kc, vc, pairs)
    slots = oracle.slot_mapping(tables, np.arange(w.num_seqs, dtype=np.int32),
                                w.seq_lens.astype(np.int64) - 1, w.block_size)
    oracle.reshape_and_cache(w.new_key, w.new_value, kc, vc, slots, w.block_size)
    out = oracle.paged_decode(w.query, kc, vc, tables, w.seq_lens, w.scale, threads=threads)
    return kc, vc, slots, out


def bf16_bits_to_f64(bits) -> np.ndarray:
    return oracle.bf16_bits_to_f64(bits)


# Observed error of every attention comparison of the session: (label, elements,
# max |gpu - ref|, max |gpu - ref| / |ref| over all elements with ref != 0, the
# same over elements with |ref| >= ATOL / RTOL = 0.2 (where the relative term of
# the bound is the larger one), and the largest ratio of the error to the
# allclose bound).  conftest prints it at the end of the run, so both literal
# maxima are on record beside the bound.
ERROR_LOG: list[tuple[str, int, float, float, float, float]] = []


def error_report(got: np.ndarray, ref: np.ndarray):
    """(max abs error, max rel error over ref != 0, max rel error over
    |ref| >= 0.2, max error / bound)."""
    err = np.abs(got - ref)
    if not err.size:
        return 0.0, 0.0, 0.0, 0.0
    aref = np.abs(ref)
    nz = aref > 0
    big = aref >= ATOL / RTOL
    max_rel = float(np.max(err[nz] / aref[nz])) if nz.any() else 0.0
    max_rel_big = float(np.max(err[big] / aref[big])) if big.any() else 0.0
    return float(err.max()), max_rel, max_rel_big, float(np.max(err / (ATOL + RTOL * aref)))


def assert_close(gpu_bits: np.ndarray, ref: np.ndarray, what: str = "") -> tuple[float, float]:
    got = bf16_bits_to_f64(gpu_bits)
    ok, max_abs, max_rel, worst = oracle.allclose_report(got, ref, ATOL, RTOL)
    if got.size:
        ERROR_LOG.append((what, int(got.size)) + error_report(got, ref))
    if not ok:
        idx = np.unravel_index(worst, ref.shape)
        raise AssertionError(f"{what}: max_abs={max_abs:.3g} max_rel={max_rel:.3g} worst at {idx}: "
                             f"gpu={got[idx]!r} ref={ref[idx]!r}")
    return max_abs, max_rel
