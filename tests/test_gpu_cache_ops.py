"""GPU parity of the integer / byte-moving kernels against the oracle: slot
mapping, cache write and copy-on-write block copies must be bit-exact."""

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_379_b200 import ops
from paged_kv_cache_379_b200 import workload as wl
from paged_kv_cache_379_b200.step import bf16_to_device, bf16_to_host_bits, host_step

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _i32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(DEV)


def _i64(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int64)).to(DEV)


@pytest.mark.parametrize("name", ["tiny", "gqa", "long"])
def test_slot_mapping_decode_form(name):
    w = wl.make(name, fill_cache=False)
    got = ops.slot_mapping(_i32(w.block_tables), w.block_size, seq_lens=_i32(w.seq_lens)).cpu().numpy()
    ref = oracle.slot_mapping(w.block_tables, np.arange(w.num_seqs, dtype=np.int32),
                              w.seq_lens.astype(np.int64) - 1, w.block_size)
    assert np.array_equal(got, ref)


def test_slot_mapping_general_form_and_edges():
    w = wl.make("tiny", fill_cache=False)
    rng = np.random.default_rng(5)
    seq_ids = rng.integers(0, w.num_seqs, size=300).astype(np.int32)
    pos = np.array([rng.integers(0, w.seq_lens[s]) for s in seq_ids], dtype=np.int64)
    pos[:7] = -1                                   # padding tokens
    got = ops.slot_mapping(_i32(w.block_tables), w.block_size, seq_ids=_i32(seq_ids),
                           positions=_i64(pos)).cpu().numpy()
    ref = oracle.slot_mapping(w.block_tables, seq_ids, pos, w.block_size)
    assert np.array_equal(got, ref)
    assert np.all(got[:7] == -1)
    # empty sequence in decode form -> -1
    sl = w.seq_lens.copy()
    sl[2] = 0
    got = ops.slot_mapping(_i32(w.block_tables), w.block_size, seq_lens=_i32(sl)).cpu().numpy()
    assert got[2] == -1


@pytest.mark.parametrize("name", ["tiny", "mha", "gqa"])
def test_reshape_and_cache_bit_exact(name):
    w = wl.make(name)
    slots = oracle.slot_mapping(w.block_tables, np.arange(w.num_seqs, dtype=np.int32),
                                w.seq_lens.astype(np.int64) - 1, w.block_size)
    slots[::5] = -1                               # every 5th token is padding
    kc, vc = bf16_to_device(w.key_cache, DEV), bf16_to_device(w.value_cache, DEV)
    ops.reshape_and_cache(bf16_to_device(w.new_key, DEV), bf16_to_device(w.new_value, DEV), kc, vc, _i64(slots))
    ref_k, ref_v = w.key_cache.copy(), w.value_cache.copy()
    oracle.reshape_and_cache(w.new_key, w.new_value, ref_k, ref_v, slots, w.block_size)
    assert np.array_equal(bf16_to_host_bits(kc), ref_k)
    assert np.array_equal(bf16_to_host_bits(vc), ref_v)


def test_reshape_and_cache_many_tokens():
    """A prefill-sized write: 3000 tokens at scattered slots of a bs-16 cache."""
    rng = np.random.default_rng(8)
    nb, bs, H, D = 400, 16, 8, 128
    kc0 = rng.integers(0, 65535, size=(nb, bs, H, D), dtype=np.uint16)
    vc0 = rng.integers(0, 65535, size=(nb, bs, H, D), dtype=np.uint16)
    slots = rng.permutation(nb * bs)[:3000].astype(np.int64)
    key = rng.integers(0, 65535, size=(3000, H, D), dtype=np.uint16)
    val = rng.integers(0, 65535, size=(3000, H, D), dtype=np.uint16)
    kc, vc = bf16_to_device(kc0, DEV), bf16_to_device(vc0, DEV)
    ops.reshape_and_cache(bf16_to_device(key, DEV), bf16_to_device(val, DEV), kc, vc, _i64(slots))
    oracle.reshape_and_cache(key, val, kc0, vc0, slots, bs)
    assert np.array_equal(bf16_to_host_bits(kc), kc0)
    assert np.array_equal(bf16_to_host_bits(vc), vc0)


@pytest.mark.parametrize("kw", [{}, {"num_seqs": 8, "shared_prompt_len": 1020, "lengths": [1] * 8}])
def test_copy_blocks_bit_exact(kw):
    w = wl.make("shared", **kw)
    _, tables, nblk, slots, pairs = host_step(w, fork_all=not kw)
    assert len(pairs) > 0
    kc, vc = bf16_to_device(w.key_cache, DEV), bf16_to_device(w.value_cache, DEV)
    ops.copy_blocks(kc, vc, _i64(pairs))
    ref_k, ref_v = w.key_cache.copy(), w.value_cache.copy()
    oracle.copy_blocks(ref_k, ref_v, pairs)
    assert np.array_equal(bf16_to_host_bits(kc), ref_k)
    assert np.array_equal(bf16_to_host_bits(vc), ref_v)
    # the sources are unchanged, destinations equal their sources
    assert np.array_equal(ref_k[pairs[:, 1]], w.key_cache[pairs[:, 0]])


def test_copy_blocks_small_block_shapes():
    rng = np.random.default_rng(9)
    for nb, bs, H, D in [(20, 4, 4, 64), (30, 8, 2, 128), (12, 16, 32, 128)]:
        kc0 = rng.integers(0, 65535, size=(nb, bs, H, D), dtype=np.uint16)
        vc0 = rng.integers(0, 65535, size=(nb, bs, H, D), dtype=np.uint16)
        perm = rng.permutation(nb)
        pairs = np.stack([perm[:nb // 3], perm[nb // 3:2 * (nb // 3)]], axis=1).astype(np.int64)
        kc, vc = bf16_to_device(kc0, DEV), bf16_to_device(vc0, DEV)
        ops.copy_blocks(kc, vc, _i64(pairs))
        oracle.copy_blocks(kc0, vc0, pairs)
        assert np.array_equal(bf16_to_host_bits(kc), kc0)
        assert np.array_equal(bf16_to_host_bits(vc), vc0)


# ---- slot mapping + cache write fused (decode form) ---------------------------------

S_EMPTY, S_NEG = 1, 2


def _append_case(name):
    """Sequence S_EMPTY has length 0 and sequence S_NEG a negative table entry
    at its newest position: both get slot -1 (the documented rule of the slot
    mapping) and write nothing.  Returns the workload, lengths, table and the
    expected slots."""
    w = wl.make(name)
    sl = w.seq_lens.copy()
    sl[S_EMPTY] = 0
    pos = sl.astype(np.int64) - 1
    ref = oracle.slot_mapping(w.block_tables, np.arange(w.num_seqs, dtype=np.int32), pos, w.block_size)
    tb = w.block_tables.copy()
    tb[S_NEG, (int(sl[S_NEG]) - 1) // w.block_size] = -1
    ref[S_NEG] = -1
    return w, sl, tb, ref


@pytest.mark.parametrize("name", ["tiny", "gqa"])
def test_append_decode_kv_equals_slot_mapping_then_cache_write(name):
    w, sl, tb, slots_ref = _append_case(name)
    ref_k, ref_v = w.key_cache.copy(), w.value_cache.copy()
    oracle.reshape_and_cache(w.new_key, w.new_value, ref_k, ref_v, slots_ref, w.block_size)
    kc, vc = bf16_to_device(w.key_cache, DEV), bf16_to_device(w.value_cache, DEV)
    slots = torch.full((w.num_seqs,), 12345, dtype=torch.int64, device=DEV)
    ops.append_decode_kv(bf16_to_device(w.new_key, DEV), bf16_to_device(w.new_value, DEV), kc, vc, _i32(tb),
                         _i32(sl), slot_mapping=slots)
    torch.cuda.synchronize()
    assert np.array_equal(slots.cpu().numpy(), slots_ref)
    assert slots_ref[S_EMPTY] == -1 and slots_ref[S_NEG] == -1
    assert np.array_equal(bf16_to_host_bits(kc), ref_k)
    assert np.array_equal(bf16_to_host_bits(vc), ref_v)
    # without the slot output
    kc2, vc2 = bf16_to_device(w.key_cache, DEV), bf16_to_device(w.value_cache, DEV)
    ops.append_decode_kv(bf16_to_device(w.new_key, DEV), bf16_to_device(w.new_value, DEV), kc2, vc2, _i32(tb),
                         _i32(sl))
    torch.cuda.synchronize()
    assert np.array_equal(bf16_to_host_bits(kc2), ref_k)


def test_append_decode_kv_fp8_equals_oracle():
    w, sl, tb, slots_ref = _append_case("gqa")
    rng = np.random.default_rng(3)
    kc8 = wl.fp8_codes(rng, w.key_cache.shape)
    vc8 = wl.fp8_codes(rng, w.value_cache.shape)
    ref_k, ref_v = kc8.copy(), vc8.copy()
    oracle.reshape_and_cache_fp8(w.new_key, w.new_value, ref_k, ref_v, slots_ref, w.block_size, 0.05, 0.3)
    dk = torch.from_numpy(kc8).to(DEV)
    dv = torch.from_numpy(vc8).to(DEV)
    ops.append_decode_kv_fp8(bf16_to_device(w.new_key, DEV), bf16_to_device(w.new_value, DEV), dk, dv, _i32(tb),
                             _i32(sl), 0.05, 0.3)
    torch.cuda.synchronize()
    assert np.array_equal(dk.cpu().numpy(), ref_k)
    assert np.array_equal(dv.cpu().numpy(), ref_v)


# ---- copy-on-write copies + slot mapping + cache write fused (decode form) -----------

def _fused_cow_matches(w, tables, seq_lens, cow_src, slots_ref, pairs_ref):
    """pa_append_decode_kv_cow against the oracle's block copies of pairs_ref
    followed by its cache write at slots_ref: caches and slots bit for bit."""
    ref_k, ref_v = w.key_cache.copy(), w.value_cache.copy()
    if len(pairs_ref):
        oracle.copy_blocks(ref_k, ref_v, np.asarray(pairs_ref, np.int64))
    oracle.reshape_and_cache(w.new_key, w.new_value, ref_k, ref_v, np.asarray(slots_ref, np.int64), w.block_size)
    kc, vc = bf16_to_device(w.key_cache, DEV), bf16_to_device(w.value_cache, DEV)
    slots = torch.full((w.num_seqs,), 777, dtype=torch.int64, device=DEV)
    ops.append_decode_kv_cow(bf16_to_device(w.new_key, DEV), bf16_to_device(w.new_value, DEV), kc, vc,
                             _i32(tables), _i32(seq_lens), _i32(cow_src), slot_mapping=slots)
    torch.cuda.synchronize()
    assert np.array_equal(slots.cpu().numpy(), np.asarray(slots_ref, np.int64))
    assert np.array_equal(bf16_to_host_bits(kc), ref_k)
    assert np.array_equal(bf16_to_host_bits(vc), ref_v)
    assert ops.device_status() == 0


@pytest.mark.parametrize("kw,fork_all", [({}, True),
                                         ({"num_seqs": 8, "shared_prompt_len": 1020, "lengths": [1] * 8}, False)])
def test_append_decode_kv_cow_equals_copies_then_cache_write(kw, fork_all):
    """The shared-prefix step through the host pool: every sequence forked (one
    copy per sequence whose token lands in an existing block), and 8 samples
    writing into their shared partial prompt block (7 copies, the last owner
    writes in place)."""
    w = wl.make("shared", **kw)
    _, tables, _, slots, pairs = host_step(w, fork_all=fork_all)
    cow_src = ops.cow_sources(slots, w.block_size, pairs)
    assert int((cow_src >= 0).sum()) == len(pairs)
    _fused_cow_matches(w, tables, w.seq_lens, cow_src, slots, pairs)


@pytest.mark.parametrize("bs,H,D", [(4, 4, 64), (8, 2, 128), (16, 8, 128), (16, 32, 128)])
def test_append_decode_kv_cow_edges(bs, H, D):
    """Random copy sources on small block shapes, with the edge cases: a
    sequence of length 0 and one with a negative table entry (slot -1: nothing
    written, nothing copied), a copy source outside the pool and one equal to
    its destination (no copy), and sequences without a copy."""
    lens = [1, 5, 0, bs, bs + 1, 3 * bs - 1, 2 * bs, 7, 40, 33]
    w = wl.random_decode_case(310 + bs + H, num_seqs=len(lens), num_heads=H, num_kv_heads=H, head_dim=D,
                              block_size=bs, lengths=lens, spare_blocks=12)
    sl = w.seq_lens.copy()
    pos = sl.astype(np.int64) - 1
    slots_ref = oracle.slot_mapping(w.block_tables, np.arange(w.num_seqs, dtype=np.int32), pos, bs)
    tb = w.block_tables.copy()
    tb[1, (int(sl[1]) - 1) // bs] = -1                      # slot -1: negative table entry
    slots_ref[1] = -1
    assert slots_ref[2] == -1
    free = list(int(b) for b in w.free_blocks)
    cow = np.full(w.num_seqs, -1, np.int32)
    pairs = []
    # sequences 3..6 copy from distinct spare blocks into their write block; sequence 1
    # (slot -1) has a source too, which must be ignored
    for s in (1, 3, 4, 5, 6):
        cow[s] = free.pop()
        if slots_ref[s] >= 0:
            pairs.append((int(cow[s]), int(slots_ref[s] // bs)))
    cow[7] = w.num_blocks + 5                                 # outside the pool: no copy
    cow[8] = int(slots_ref[8] // bs)                          # its own destination: no copy
    _fused_cow_matches(w, tb, sl, cow, slots_ref, pairs)
