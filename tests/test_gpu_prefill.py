"""GPU parity of the multi-query paged prefill (tcgen05 kernel) against the
oracle's fp64 causal prefill, element by element."""

import dataclasses

import numpy as np
import pytest
import torch

import oracle
from _helpers import assert_close
from paged_kv_cache_379_b200 import ops
from paged_kv_cache_379_b200 import workload as wl
from paged_kv_cache_379_b200.step import bf16_to_device, bf16_to_host_bits

pytestmark = pytest.mark.gpu
DEV = "cuda"
SENTINEL = np.uint16(0x7F80)  # bf16 +inf: rows the kernel must not write


def _i32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(DEV)


def _case(seed, bs, Hq, Hkv, D, lens, q_lens):
    w = wl.random_decode_case(seed, num_seqs=len(lens), num_heads=Hq, num_kv_heads=Hkv, head_dim=D,
                              block_size=bs, lengths=lens)
    # slots past each sequence's end hold NaN: they must never reach the output
    for s, L in enumerate(w.seq_lens):
        if L > 0 and L % bs:
            last = int(w.block_tables[s, (L - 1) // bs])
            w.key_cache[last, L % bs:] = wl.BF16_NAN
            w.value_cache[last, L % bs:] = wl.BF16_NAN
    q = wl.bf16_normal(np.random.default_rng(seed + 7), (int(sum(q_lens)), Hq, D))
    return w, q


def _run(w, q, q_lens):
    start = np.zeros(len(q_lens) + 1, np.int32)
    start[1:] = np.cumsum(q_lens)
    out = torch.from_numpy(np.full(q.shape, SENTINEL, np.uint16).view(np.int16)).to(DEV).view(torch.bfloat16)
    ops.prefill(bf16_to_device(q, DEV), bf16_to_device(w.key_cache, DEV), bf16_to_device(w.value_cache, DEV),
                _i32(w.block_tables), _i32(w.seq_lens), _i32(start), w.scale, out=out)
    torch.cuda.synchronize()
    return bf16_to_host_bits(out)


def _check(w, q, q_lens, what, active=None):
    got = _run(w, q, q_lens)
    ref = oracle.paged_prefill(q, w.key_cache, w.value_cache, w.block_tables, w.seq_lens, q_lens, w.scale,
                               threads=16)
    rows = np.ones(q.shape[0], bool) if active is None else active
    assert_close(got[rows], ref[rows], what)
    assert (got[~rows] == SENTINEL).all(), f"{what}: rows of skipped sequences were written"
    assert ops.device_status() == 0


# ---- whole prompts, chunks at an offset, single tokens, across groups and shapes ------

LENS = [1, 5, 127, 128, 129, 300, 450, 700, 64]
QLENS = [1, 5, 127, 128, 129, 77, 450, 1, 0]  # whole prompts, a chunk at offset 223, a decode-like row, idle


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("bs", [8, 16, 32])
@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (8, 1), (16, 2), (12, 2), (32, 8)])
def test_prefill_matches_oracle(D, bs, Hq, Hkv):
    w, q = _case(7000 + D + bs + 3 * Hq + Hkv, bs, Hq, Hkv, D, LENS, QLENS)
    _check(w, q, QLENS, f"prefill D={D} bs={bs} G={Hq // Hkv}")


def test_prefill_long_chunk_many_key_tiles():
    """A 600-token chunk at offset 1450: 17 key tiles, query tiles of 16 tokens (G = 8)."""
    w, q = _case(7100, 16, 64, 8, 128, [2050, 33], [600, 33])
    _check(w, q, [600, 33], "long chunk")


def test_prefill_skips_invalid_chunks():
    """q_len > seq_len is skipped; its rows keep their contents."""
    lens, q_lens = [40, 10, 90], [20, 12, 90]
    w, q = _case(7200, 16, 8, 2, 128, lens, q_lens)
    active = np.zeros(sum(q_lens), bool)
    active[:20] = True
    active[32:] = True
    got = _run(w, q, q_lens)
    assert (got[20:32] == SENTINEL).all()
    ref = oracle.paged_prefill(q[active], w.key_cache, w.value_cache, w.block_tables[[0, 2]],
                               w.seq_lens[[0, 2]], [20, 90], w.scale, threads=16)
    assert_close(got[active], ref, "valid chunks beside an invalid one")
    assert ops.device_status() == 0


def test_prefill_chunked_equals_whole_prompt():
    """A prompt prefilled in three chunks gives the rows of one whole-prompt call."""
    L = 520
    w, q = _case(7300, 16, 16, 4, 128, [L], [L])
    whole = _run(w, q, [L])
    parts = []
    for a, b in ((0, 130), (130, 400), (400, L)):
        wc = dataclasses.replace(w, seq_lens=np.array([b], np.int32))
        parts.append(_run(wc, q[a:b], [b - a]))
    ref = oracle.paged_prefill(q, w.key_cache, w.value_cache, w.block_tables, w.seq_lens, [L], w.scale,
                               threads=16)
    assert_close(whole, ref, "whole prompt")
    assert_close(np.concatenate(parts), ref, "three chunks")


def test_prefill_rejects_unsupported_shapes():
    w, q = _case(7400, 4, 4, 4, 64, [8], [8])
    with pytest.raises(ops.PagedKVError):  # block_size 4 is not compiled for prefill
        _run(w, q, [8])
    torch.cuda.synchronize()
    assert ops.device_status() == 0


def test_prefill_bench_workload_sampled_rows():
    """The bench's prefill workload (8 x 2048-token prompts, 64 query / 8 KV heads,
    head_dim 128, block size 16) in its launch configuration, checked on sampled
    rows: windows of 16 query rows at spread positions, each against the oracle's
    prefill of that window (a chunk ending at the window's last position)."""
    import bench
    w, lens, q, nk, nv = bench.make_prefill_case(bench.rank_seed(0))
    B, P = w.num_seqs, lens[0]
    T = q.shape[0]
    # the step's cache write: the prompts' K/V rows at their slots
    seq_ids = np.repeat(np.arange(B), lens).astype(np.int32)
    pos = np.concatenate([np.arange(L) for L in lens]).astype(np.int64)
    slots = oracle.slot_mapping(w.block_tables, seq_ids, pos, w.block_size)
    kc, vc = w.key_cache.copy(), w.value_cache.copy()
    oracle.reshape_and_cache(nk, nv, kc, vc, slots, w.block_size)
    start = np.zeros(B + 1, np.int32)
    start[1:] = np.cumsum(lens)
    out = ops.prefill(bf16_to_device(q, DEV), bf16_to_device(kc, DEV), bf16_to_device(vc, DEV),
                      _i32(w.block_tables), _i32(np.asarray(lens)), _i32(start), w.scale)
    torch.cuda.synchronize()
    got = bf16_to_host_bits(out)
    rng = np.random.default_rng(11)
    for s in range(B):
        for end in (16, int(rng.integers(17, P)), P):
            rows = slice(s * P + end - 16, s * P + end)
            ref = oracle.paged_prefill(q[rows], kc, vc, w.block_tables[s:s + 1], np.array([end], np.int32), [16],
                                       w.scale, threads=16)
            assert_close(got[rows], ref, f"seq {s} rows {end - 16}..{end - 1}")
    assert ops.device_status() == 0


def test_prefill_value_beyond_fp16_range_sets_status():
    """P V runs on fp16 operands: a value-cache entry of magnitude above 65504
    read by the prefill saturates and sets PA_ERR_VALUE_RANGE in the device
    status; rows that do not attend to it still match the oracle.  65280 (the
    largest bf16 value inside the fp16 range) does not set it."""
    lens, q_lens = [200], [200]
    w, q = _case(7500, 16, 8, 2, 128, lens, q_lens)
    last = int(w.block_tables[0, (200 - 1) // 16])
    off = (200 - 1) % 16
    w.value_cache[last, off, 1, 5] = np.uint16(0x47C3)  # 99840: beyond fp16, only the last row attends to it
    got = _run(w, q, q_lens)
    assert ops.device_status() == -12
    ref = oracle.paged_prefill(q, w.key_cache, w.value_cache, w.block_tables, w.seq_lens, q_lens, w.scale,
                               threads=16)
    assert_close(got[:199], ref[:199], "rows before the out-of-range entry")
    w.value_cache[last, off, 1, 5] = np.uint16(0x477F)  # 65280: inside the fp16 range
    _check(w, q, q_lens, "largest in-range value")
