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
