"""Pins of the oracle's block pool: the pages' sharing / copy-on-write rules and
bookkeeping invariants (CPU only)."""

import numpy as np
import pytest

from oracle.pool import OraclePool, PoolExhausted


def _check_invariants(pool, tables, extra_owners=()):
    refs = np.zeros(pool.num_blocks, dtype=np.int64)
    for t in list(tables) + list(extra_owners):
        for b in t:
            refs[b] += 1
    assert refs.tolist() == pool.refcount          # sum of refcounts = table references
    in_use = sum(1 for r in pool.refcount if r > 0)
    assert in_use + pool.get_num_free_blocks() == pool.num_blocks
    assert len(set(pool.free_list)) == len(pool.free_list)
    assert all(pool.refcount[b] == 0 for b in pool.free_list)


def test_free_list_is_lifo_and_exhaustion_raises():
    pool = OraclePool(4, 16, free_order=[2, 0, 3, 1])
    assert pool.allocate(2) == [1, 3]             # pops from the end
    pool.free(3)
    assert pool.allocate(1) == [3]                # the freed block comes back first
    assert pool.get_num_free_blocks() == 2
    with pytest.raises(PoolExhausted):
        pool.allocate(3)


def test_cow_siblings_on_shared_partial_block():
    """8 samples share a prompt whose last block is partial; each writes its first token.

    A block with reference count > 1 is copied before the write and the count drops
    by one; the last remaining owner writes in place: 7 copies for 8 samples.
    """
    bs, prompt = 16, 1020
    pool = OraclePool(128, bs)
    parent = pool.allocate_prompt(prompt)
    tables = [parent] + [pool.fork(parent) for _ in range(7)]
    shared_last = parent[-1]
    assert pool.refcount[shared_last] == 8
    pairs = []
    for t in tables:
        slot, pair, alloc = pool.append_token(t, prompt)
        assert not alloc
        assert slot % bs == prompt % bs
        if pair:
            pairs.append(pair)
    assert len(pairs) == 7
    assert all(src == shared_last for src, _ in pairs)
    assert len({dst for _, dst in pairs}) == 7
    assert pool.refcount[shared_last] == 1
    assert sum(1 for t in tables if t[-1] == shared_last) == 1
    _check_invariants(pool, tables)


def test_fork_snapshot_then_write_copies_the_written_block_only():
    """With a retained parent snapshot, every write into an old block copies it once."""
    bs = 16
    pool = OraclePool(64, bs)
    seq = pool.allocate_prompt(40)                # 3 blocks, last holds 8 tokens
    snap = pool.fork(seq)
    slot, pair, alloc = pool.append_token(seq, 40)
    assert pair is not None and pair[0] == snap[2] and seq[2] == pair[1]
    assert seq[:2] == snap[:2]                    # only the written block forked
    assert pool.refcount[snap[2]] == 1 and pool.refcount[seq[2]] == 1
    _check_invariants(pool, [seq], extra_owners=[snap])
    # a write at a block boundary takes a fresh block: no copy
    seq2 = pool.allocate_prompt(48)
    snap2 = pool.fork(seq2)
    _, pair2, alloc2 = pool.append_token(seq2, 48)
    assert pair2 is None and alloc2 and len(seq2) == 4
    _check_invariants(pool, [seq, seq2], extra_owners=[snap, snap2])


def test_random_operations_keep_invariants():
    rng = np.random.default_rng(3)
    bs = 4
    pool = OraclePool(200, bs, free_order=rng.permutation(200).tolist())
    seqs = []       # (table, length)
    for _ in range(400):
        op = rng.integers(0, 4)
        try:
            if op == 0 or not seqs:
                n = int(rng.integers(1, 20))
                seqs.append([pool.allocate_prompt(n), n])
            elif op == 1:
                i = int(rng.integers(len(seqs)))
                seqs.append([pool.fork(seqs[i][0]), seqs[i][1]])
            elif op == 2:
                i = int(rng.integers(len(seqs)))
                t, n = seqs[i]
                pool.append_token(t, n)
                seqs[i][1] = n + 1
            else:
                i = int(rng.integers(len(seqs)))
                pool.free_sequence(seqs[i][0])
                seqs.pop(i)
        except PoolExhausted:
            pass
        _check_invariants(pool, [t for t, _ in seqs])
    for t, n in seqs:
        assert len(t) == -(-n // bs)


def test_swap_plan_moves_references_between_pools():
    from oracle.pool import swap_plan
    gpu, cpu = OraclePool(16, 4), OraclePool(8, 4)
    a = gpu.allocate_prompt(10)                  # 3 blocks
    b = gpu.fork(a[:2]) + gpu.allocate(1)        # shares 2 of them
    host_b, pairs = swap_plan(gpu, cpu, b)
    assert len(pairs) == 3 and [s for s, _ in pairs] == b
    assert [gpu.refcount[x] for x in a] == [1, 1, 1]      # a keeps its blocks
    assert gpu.get_num_free_blocks() == 16 - 3
    assert [cpu.refcount[x] for x in host_b] == [1, 1, 1]
    back, pairs_in = swap_plan(cpu, gpu, host_b)
    assert cpu.get_num_free_blocks() == 8 and [d for _, d in pairs_in] == back
    _check_invariants(gpu, [a, back])
