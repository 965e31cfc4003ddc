"""GPU parity of the decode that reads shared prefixes once per group of
sequences (pa_decode_shared): against the fp64 oracle element by element, and
bit for bit against the split decode at the same partition size where both
run on the tensor cores (G >= 3: the same arithmetic per query row, only the
work items differ)."""

import numpy as np
import pytest
import torch

import oracle
from _helpers import assert_close, oracle_step, poison_tail_slots
from paged_kv_cache_379_b200 import ops
from paged_kv_cache_379_b200 import workload as wl
from paged_kv_cache_379_b200.step import DecodeBatch, bf16_to_device, bf16_to_host_bits, host_step

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _i32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(DEV)


def _decode_both(w, tables, part, groups=None):
    """(shared-prefix decode, split decode) output bits on the same inputs."""
    q, kc, vc = (bf16_to_device(a, DEV) for a in (w.query, w.key_cache, w.value_cache))
    bt, sl = _i32(tables), _i32(w.seq_lens)
    gs, gp = groups if groups is not None else ops.prefix_groups(tables, w.seq_lens, w.block_size, part)
    ws = ops.new_workspace(w.num_seqs, w.num_heads, w.num_kv_heads, w.head_dim, w.max_seq_len, part, device=DEV)
    shared = ops.decode_shared(q, kc, vc, bt, sl, w.scale, w.max_seq_len, part, _i32(gs), _i32(gp), ws)
    torch.cuda.synchronize()
    got = bf16_to_host_bits(shared)
    ws2 = ops.new_workspace(w.num_seqs, w.num_heads, w.num_kv_heads, w.head_dim, w.max_seq_len, part, device=DEV)
    split = ops.decode_split(q, kc, vc, bt, sl, w.scale, w.max_seq_len, part, ws2)
    torch.cuda.synchronize()
    return got, bf16_to_host_bits(split), (gs, gp)


@pytest.mark.parametrize("part", [256, 512, 1024])
def test_shared_workload_step(part):
    """The shared-prefix step (256 sequences forked from 32 prompts of 1024
    tokens): copy-on-write copies + cache write in one launch, then the decode
    with the groups the host finds (32 groups of 8 sharing 1024 / part
    partitions), against the oracle's copies, cache write and decode."""
    w = wl.make("shared")
    _, tables, _, slots, pairs = host_step(w, fork_all=True)
    poison_tail_slots(w, tables)
    cow = ops.cow_sources(slots, w.block_size, pairs)
    gs, gp = ops.prefix_groups(tables, w.seq_lens, w.block_size, part)
    assert len(gp) == 32 and np.all(gp == 1024 // part) and np.all(np.diff(gs) == 8)
    batch = DecodeBatch(w, DEV, tables=tables, pairs=pairs, cow_src=cow, workspace=False)
    ops.append_decode_kv_cow(batch.new_key, batch.new_value, batch.key_cache, batch.value_cache,
                             batch.block_tables, batch.seq_lens, batch.cow_src, slot_mapping=batch.slots)
    ws = ops.new_workspace(w.num_seqs, w.num_heads, w.num_kv_heads, w.head_dim, w.max_seq_len, part, device=DEV)
    out = ops.decode_shared(batch.query, batch.key_cache, batch.value_cache, batch.block_tables, batch.seq_lens,
                            w.scale, w.max_seq_len, part, _i32(gs), _i32(gp), ws)
    torch.cuda.synchronize()
    ref_k, ref_v, ref_slots, ref_out = oracle_step(w, tables, pairs)
    assert np.array_equal(batch.slots.cpu().numpy(), ref_slots)
    assert np.array_equal(bf16_to_host_bits(batch.key_cache), ref_k)
    assert_close(bf16_to_host_bits(out), ref_out, f"shared step, groups, partition {part}")
    assert ops.device_status() == 0


def _grouped_case(seed, G, Hkv, D, bs, part, sizes, shared_parts, tails):
    """Groups of consecutive sequences: group i has sizes[i] members sharing
    shared_parts[i] partitions of blocks, then private tails of tails[j]
    positions (0 allowed: the sequence ends with the shared part).  Physical
    block ids are shuffled; three unowned blocks hold bf16 NaN."""
    rng = np.random.default_rng(seed)
    lens, rows = [], []
    nb = 0
    for n, k in zip(sizes, shared_parts):
        common = list(range(nb, nb + k * part // bs))
        nb += len(common)
        for _ in range(n):
            t = int(tails[len(lens) % len(tails)])
            L = k * part + t
            own = list(range(nb, nb + (-(-L // bs) - len(common))))
            nb += len(own)
            rows.append(common + own)
            lens.append(L)
    spare = 3
    perm = rng.permutation(nb + spare).astype(np.int32)
    width = max(len(r) for r in rows)
    tables = np.full((len(rows), width), -1, np.int32)
    for s, r in enumerate(rows):
        tables[s, :len(r)] = perm[r]
    B, Hq = len(lens), G * Hkv
    cache_k = wl.bf16_normal(rng, (nb + spare, bs, Hkv, D))
    cache_v = wl.bf16_normal(rng, (nb + spare, bs, Hkv, D))
    cache_k[perm[nb:]] = wl.BF16_NAN
    cache_v[perm[nb:]] = wl.BF16_NAN
    return wl.Workload(name="custom", seed=seed, num_seqs=B, num_heads=Hq, num_kv_heads=Hkv, head_dim=D,
                       block_size=bs, num_blocks=nb + spare, scale=float(1.0 / np.sqrt(D)),
                       seq_lens=np.asarray(lens, np.int32), block_tables=tables,
                       blocks_per_seq=np.array([len(r) for r in rows], np.int32),
                       query=wl.bf16_normal(rng, (B, Hq, D)), new_key=wl.bf16_normal(rng, (B, Hkv, D)),
                       new_value=wl.bf16_normal(rng, (B, Hkv, D)), key_cache=cache_k, value_cache=cache_v,
                       free_blocks=perm[nb:].copy())


@pytest.mark.parametrize("G,Hkv,D,bs", [(4, 2, 128, 16), (8, 1, 128, 16), (1, 4, 128, 16), (2, 2, 64, 8),
                                        (16, 1, 64, 4), (3, 2, 128, 8)])
def test_random_groups_match_oracle_and_split(G, Hkv, D, bs):
    part = 64
    w = _grouped_case(700 + G * 10 + Hkv + D + bs, G, Hkv, D, bs, part,
                      sizes=[5, 1, 9, 2, 3], shared_parts=[3, 2, 1, 4, 2], tails=[0, 1, 17, 63, 64, 100, 5])
    gs, gp = ops.prefix_groups(w.block_tables, w.seq_lens, bs, part)
    assert np.array_equal(np.diff(gs), [5, 1, 9, 2, 3]) and gp.tolist() == [3, 0, 1, 4, 2]
    got, split, _ = _decode_both(w, w.block_tables, part, (gs, gp))
    ref = oracle.paged_decode(w.query, w.key_cache, w.value_cache, w.block_tables, w.seq_lens, w.scale)
    assert_close(got, ref, f"groups G={G} Hkv={Hkv} D={D} bs={bs}")
    if G >= 3:   # both on the tensor cores (the split decode takes the CUDA-core consumers at G <= 2)
        assert np.array_equal(got, split)
    assert ops.device_status() == 0


def test_groups_that_compute_fewer_partitions_than_shared():
    """A group may compute fewer leading partitions than its members share
    (here 1 of 3, or none): the rest run per sequence; same result."""
    part = 64
    w = _grouped_case(808, 4, 2, 128, 16, part, sizes=[6, 4], shared_parts=[3, 2], tails=[7, 0, 64, 90])
    for gp in ([1, 2], [0, 0], [3, 1]):
        got, split, _ = _decode_both(w, w.block_tables, part, (np.array([0, 6, 10], np.int32), np.array(gp, np.int32)))
        assert np.array_equal(got, split), gp
    ref = oracle.paged_decode(w.query, w.key_cache, w.value_cache, w.block_tables, w.seq_lens, w.scale)
    assert_close(got, ref, "groups computing fewer partitions")


def test_many_groups_and_sequences():
    """More groups than the kernel has threads (the enumeration's per-group
    loop takes several rounds) and over a thousand sequences: 300 groups of
    2-6 sequences sharing 1-3 partitions, against the oracle and bit for bit
    against the split decode."""
    part = 64
    rng = np.random.default_rng(31)
    sizes = rng.integers(2, 7, size=300).tolist()
    shared = rng.integers(1, 4, size=300).tolist()
    w = _grouped_case(909, 4, 2, 64, 16, part, sizes=sizes, shared_parts=shared, tails=[0, 3, 16, 40, 64, 70])
    assert w.num_seqs > 1000
    gs, gp = ops.prefix_groups(w.block_tables, w.seq_lens, w.block_size, part)
    assert len(gp) == 300 and np.array_equal(np.diff(gs), sizes) and gp.tolist() == shared
    got, split, _ = _decode_both(w, w.block_tables, part, (gs, gp))
    ref = oracle.paged_decode(w.query, w.key_cache, w.value_cache, w.block_tables, w.seq_lens, w.scale)
    assert_close(got, ref, "300 groups, %d sequences" % w.num_seqs)
    assert np.array_equal(got, split)
    assert ops.device_status() == 0
