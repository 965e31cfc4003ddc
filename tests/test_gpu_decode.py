"""GPU parity of paged decode attention (one-pass, split + reduce, and the
library's own choice) against the fp64 oracle, element by element."""

import numpy as np
import pytest
import torch

import oracle
from _helpers import assert_close, oracle_step, poison_tail_slots
from paged_kv_cache_379_b200 import ops
from paged_kv_cache_379_b200 import workload as wl
from paged_kv_cache_379_b200.step import DecodeBatch, bf16_to_device, bf16_to_host_bits

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _dev_inputs(w):
    return dict(
        query=bf16_to_device(w.query, DEV),
        key_cache=bf16_to_device(w.key_cache, DEV),
        value_cache=bf16_to_device(w.value_cache, DEV),
        block_tables=torch.from_numpy(np.ascontiguousarray(w.block_tables, np.int32)).to(DEV),
        seq_lens=torch.from_numpy(w.seq_lens.astype(np.int32)).to(DEV),
    )


def _run(w, kind, partition=512):
    d = _dev_inputs(w)
    args = (d["query"], d["key_cache"], d["value_cache"], d["block_tables"], d["seq_lens"], w.scale,
            w.max_seq_len)
    if kind == "one_pass":
        out = ops.decode_one_pass(*args)
    elif kind == "split":
        ws = ops.new_workspace(w.num_seqs, w.num_heads, w.num_kv_heads, w.head_dim, w.max_seq_len, partition,
                               device=DEV)
        out = ops.decode_split(*args, partition, ws)
    else:
        ws = ops.new_workspace(w.num_seqs, w.num_heads, w.num_kv_heads, w.head_dim, w.max_seq_len, device=DEV)
        out = ops.decode(*args, workspace=ws)
    torch.cuda.synchronize()
    return bf16_to_host_bits(out)


# ---- the five workloads, whole step, in the benchmark's launch configuration --------

@pytest.mark.parametrize("name", ["tiny", "mha", "gqa", "long", "shared", "shared-fused"])
def test_workload_step_matches_oracle(name):
    """The whole step of each workload as the bench runs it (shared: every
    sequence forked, copy-on-write copies as their own launch, or fused into
    the cache write's launch)."""
    w = wl.make(name.split("-")[0])
    tables, pairs, cow = w.block_tables, None, None
    if name.startswith("shared"):
        from paged_kv_cache_379_b200.step import host_step
        _, tables, _, slots, pairs = host_step(w, fork_all=True)
        if name == "shared-fused":
            cow = ops.cow_sources(slots, w.block_size, pairs)
    poison_tail_slots(w, tables)
    batch = DecodeBatch(w, DEV, tables=tables, pairs=pairs, cow_src=cow)
    out = batch.run_step()
    torch.cuda.synchronize()
    ref_k, ref_v, ref_slots, ref_out = oracle_step(w, tables, pairs)
    assert np.array_equal(batch.slots.cpu().numpy(), ref_slots)
    assert np.array_equal(bf16_to_host_bits(batch.key_cache), ref_k)
    assert np.array_equal(bf16_to_host_bits(batch.value_cache), ref_v)
    assert_close(bf16_to_host_bits(out), ref_out, name)
    assert ops.device_status() == 0


# ---- kernel variants over shapes, groups, block sizes and ragged lengths ------------

LENS = [1, 2, 15, 16, 17, 31, 33, 64, 100, 255, 256, 257, 511, 512, 513, 700, 1025, 2000]


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("bs", [4, 8, 16])
@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (8, 4), (8, 2), (16, 2), (16, 1), (6, 2)])
def test_variants_match_oracle(D, bs, Hq, Hkv):
    seed = 1000 + D + 7 * bs + Hq * 31 + Hkv
    w = wl.random_decode_case(seed, num_seqs=len(LENS), num_heads=Hq, num_kv_heads=Hkv, head_dim=D,
                              block_size=bs, lengths=LENS)
    poison_tail_slots(w)
    # tail slots of positions >= L are poison; the token at L-1 is the cache's own
    for s, L in enumerate(w.seq_lens):
        blk = w.block_tables[s, (L - 1) // bs]
        w.key_cache[blk, (L - 1) % bs] = w.new_key[s]
        w.value_cache[blk, (L - 1) % bs] = w.new_value[s]
    ref = oracle.paged_decode(w.query, w.key_cache, w.value_cache, w.block_tables, w.seq_lens, w.scale,
                              threads=0)
    for kind, part in (("one_pass", 0), ("split", 16), ("split", 64), ("split", 512), ("auto", 0)):
        assert_close(_run(w, kind, part), ref, f"D{D} bs{bs} {Hq}/{Hkv} {kind}/{part}")


@pytest.mark.parametrize("B", [256, 257, 600, 3000])
def test_batch_sizes_around_the_rank_sort_limit(B):
    """The work items of a launch are ordered largest first by a counting sort
    over the remainders' tile counts (the first item of a CTA selected from the
    histogram before the order is scattered), with every CTA's enumeration
    tables in shared memory: batches around a warp multiple and one of 3000
    sequences (tables of ~25 KB per CTA), in one pass, split and the plan's
    choice, against the oracle, ragged lengths with empty sequences."""
    rng = np.random.default_rng(900 + B)
    lens = rng.integers(0, 700, B)
    lens[::37] = 0
    w = wl.random_decode_case(910 + B, num_seqs=B, num_heads=8, num_kv_heads=2, head_dim=128, block_size=16,
                              lengths=lens.tolist(), spare_blocks=4)
    ref = oracle.paged_decode(w.query, w.key_cache, w.value_cache, w.block_tables, w.seq_lens, w.scale,
                              threads=0)
    for kind, part in (("one_pass", 0), ("split", 128), ("auto", 0)):
        assert_close(_run(w, kind, part), ref, f"B={B} {kind}/{part}")
    assert ops.device_status() == 0


def test_zero_length_and_single_token():
    lens = [0, 1, 0, 5, 1]
    w = wl.random_decode_case(77, num_seqs=5, num_heads=8, num_kv_heads=1, head_dim=128, block_size=16,
                              lengths=lens, spare_blocks=2)
    for kind, part in (("one_pass", 0), ("split", 16), ("auto", 0)):
        got = _run(w, kind, part)
        assert np.all(got[0] == 0) and np.all(got[2] == 0)
        for s in (1, 4):   # L = 1: the value row itself, bit for bit
            blk = w.block_tables[s, 0]
            assert np.array_equal(got[s], np.broadcast_to(w.value_cache[blk, 0, 0], got[s].shape))


def test_permutation_of_physical_blocks_is_bitwise_invariant():
    w = wl.random_decode_case(5, num_seqs=6, num_heads=32, num_kv_heads=8, head_dim=128, block_size=16,
                              lengths=[33, 200, 1000, 17, 512, 1500])
    rng = np.random.default_rng(1)
    perm = rng.permutation(w.num_blocks)
    w2 = wl.random_decode_case(5, num_seqs=6, num_heads=32, num_kv_heads=8, head_dim=128, block_size=16,
                               lengths=[33, 200, 1000, 17, 512, 1500])
    w2.key_cache[perm] = w.key_cache
    w2.value_cache[perm] = w.value_cache
    w2.block_tables = np.where(w.block_tables >= 0, perm[np.maximum(w.block_tables, 0)], -1).astype(np.int32)
    for kind, part in (("one_pass", 0), ("split", 128), ("auto", 0)):
        assert np.array_equal(_run(w, kind, part), _run(w2, kind, part))


def test_shared_prefix_identical_outputs():
    w = wl.random_decode_case(6, num_seqs=4, num_heads=32, num_kv_heads=8, head_dim=128, block_size=16,
                              lengths=[700, 700, 700, 700])
    w.block_tables[1:] = w.block_tables[0]
    w.query[1:] = w.query[0]
    for kind, part in (("one_pass", 0), ("split", 256)):
        got = _run(w, kind, part)
        assert all(np.array_equal(got[0], got[i]) for i in range(1, 4))


@pytest.mark.parametrize("Hq,Hkv,part", [(32, 8, 512), (8, 8, 64), (16, 1, 32)])
def test_partitions_and_reduce_match_oracle(Hq, Hkv, part):
    lens = [1, 40, 511, 512, 513, 1300, 0, 2047]
    w = wl.random_decode_case(88, num_seqs=len(lens), num_heads=Hq, num_kv_heads=Hkv, head_dim=128,
                              block_size=16, lengths=lens, spare_blocks=1)
    d = _dev_inputs(w)
    ws = ops.new_workspace(w.num_seqs, Hq, Hkv, 128, w.max_seq_len, part, device=DEV)
    o, m, l = ops.decode_partitions(d["query"], d["key_cache"], d["value_cache"], d["block_tables"],
                                    d["seq_lens"], w.scale, w.max_seq_len, part, ws)
    torch.cuda.synchronize()
    parts = o.shape[2]
    rm, rl, ro = oracle.paged_decode_partials(w.query, w.key_cache, w.value_cache, w.block_tables,
                                              w.seq_lens, w.scale, part, parts)
    gm, gl, go = m.double().cpu().numpy(), l.double().cpu().numpy(), o.double().cpu().numpy()
    empty = np.isneginf(rm)
    assert np.array_equal(np.isneginf(gm), empty)
    assert np.all(gl[empty] == 0) and np.all(go[empty] == 0)
    full = ~empty
    np.testing.assert_allclose(gm[full], rm[full], rtol=1e-5, atol=1e-4)
    np.testing.assert_allclose(gl[full], rl[full], rtol=1e-2)
    norm_ref = ro[full] / rl[full][:, None]
    norm_gpu = go[full] / gl[full][:, None]
    ok, max_abs, _, _ = oracle.allclose_report(norm_gpu, norm_ref, 2e-3, 1e-2)
    assert ok, max_abs
    out = torch.empty_like(d["query"])
    ops.lse_reduce(out, ws, d["seq_lens"], w.max_seq_len, part)
    torch.cuda.synchronize()
    ref = oracle.paged_decode(w.query, w.key_cache, w.value_cache, w.block_tables, w.seq_lens, w.scale)
    assert_close(bf16_to_host_bits(out), ref, "lse_reduce")


@pytest.mark.parametrize("sched", ["round_robin", "dynamic"])
def test_one_pass_full_gqa_batch_matches_oracle(sched):
    """One pass over the whole GQA batch: every CTA runs several long items of
    many table chunks (up to 256 tiles each), so the consumer warps drift apart
    and the ring wraps many times within one item."""
    w = wl.make("gqa")
    d = _dev_inputs(w)
    args = (d["query"], d["key_cache"], d["value_cache"], d["block_tables"], d["seq_lens"], w.scale, w.max_seq_len)
    if sched == "round_robin":
        out = ops.decode_one_pass(*args)
    else:
        counters = torch.zeros(256, dtype=torch.uint8, device=DEV)   # too small to split: one pass, dynamic
        assert ops.decode_plan(w.num_seqs, w.num_heads, w.num_kv_heads, w.head_dim, w.max_seq_len, 256) == 0
        out = ops.decode(*args, workspace=counters)
        out = ops.decode(*args, workspace=counters)                    # counters were left at zero
        assert int(counters.view(torch.int32)[:2].abs().sum().item()) == 0
    torch.cuda.synchronize()
    ref = oracle.paged_decode(w.query, w.key_cache, w.value_cache, w.block_tables, w.seq_lens, w.scale, threads=0)
    assert_close(bf16_to_host_bits(out), ref, f"one pass, {sched}")
    assert ops.device_status() == 0


@pytest.fixture(scope="module")
def long_case():
    """The long-context workload (8 sequences of 32K..128K positions, 32 query /
    8 KV heads) after one step's cache write, and the oracle's output for it."""
    w = wl.make("long")
    poison_tail_slots(w)
    ref_k, ref_v, ref_slots, ref_out = oracle_step(w)
    return w, ref_k, ref_v, ref_slots, ref_out


@pytest.mark.parametrize("partition", [512, 2048])
def test_long_context_split_matches_oracle(long_case, partition):
    """The long-context step in the split form at the workload's stated
    512-token partitions (64..256 partitions per (sequence, head), all merged by
    the log-sum-exp reduce) and at the 2048 the library's plan picks: the fused
    slot mapping + cache write, then partition kernel + reduce, against the
    oracle element by element."""
    w, ref_k, ref_v, ref_slots, ref_out = long_case
    batch = DecodeBatch(w, DEV, workspace=False)
    ws = ops.new_workspace(w.num_seqs, w.num_heads, w.num_kv_heads, w.head_dim, w.max_seq_len, partition,
                           device=DEV)
    ops.append_decode_kv(batch.new_key, batch.new_value, batch.key_cache, batch.value_cache, batch.block_tables,
                         batch.seq_lens, slot_mapping=batch.slots)
    out = ops.decode_split(batch.query, batch.key_cache, batch.value_cache, batch.block_tables, batch.seq_lens,
                           w.scale, w.max_seq_len, partition, ws)
    torch.cuda.synchronize()
    assert np.array_equal(batch.slots.cpu().numpy(), ref_slots)
    assert np.array_equal(bf16_to_host_bits(batch.key_cache), ref_k)
    assert np.array_equal(bf16_to_host_bits(batch.value_cache), ref_v)
    if partition == 512:  # the reduce merges well over 128 partitions per (sequence, head)
        assert int(w.seq_lens.max()) > 128 * 512
    assert_close(bf16_to_host_bits(out), ref_out, f"long, split {partition}")
    assert ops.device_status() == 0


def test_validate_tables():
    w = wl.make("tiny", fill_cache=False)
    d = _dev_inputs(w)
    assert ops.validate_tables(d["block_tables"], d["seq_lens"], w.block_size, w.num_blocks, w.max_seq_len) == 0
    bad = w.block_tables.copy()
    bad[1, 0] = w.num_blocks
    bt = torch.from_numpy(bad).to(DEV)
    assert ops.validate_tables(bt, d["seq_lens"], w.block_size, w.num_blocks, w.max_seq_len) == 1
    assert ops.validate_tables(d["block_tables"], d["seq_lens"], w.block_size, w.num_blocks, 40) == 1
    assert ops.device_status() == 0


def test_bounded_wait_gives_up_and_reports_timeout():
    """A device wait that nothing satisfies gives up after its limit, leaves
    PA_ERR_DEVICE_TIMEOUT in the device status (read once, then cleared), and the
    context stays usable: a decode right after it matches the oracle."""
    assert ops.device_status() == 0
    ops.selftest_bounded_wait()
    assert ops.device_status() == -9
    assert ops.device_status() == 0
    w = wl.make("tiny")
    b = DecodeBatch(w, DEV)
    out = b.run_step()
    torch.cuda.synchronize()
    _, _, _, ref = oracle_step(w)
    assert_close(bf16_to_host_bits(out), ref, "decode after a timed-out wait")
    assert ops.device_status() == 0
