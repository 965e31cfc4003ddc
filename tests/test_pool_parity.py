"""The native host block pool (C++ behind the C ABI) against the oracle's plain
Python pool: identical ids, reference counts, slots and copy pairs, bit for bit
(CPU only)."""

import numpy as np
import pytest

import oracle
from oracle.pool import OraclePool, PoolExhausted
from paged_kv_cache_379_b200 import workload as wl
from paged_kv_cache_379_b200._lib import PagedKVError
from paged_kv_cache_379_b200.pool import BlockPool
from paged_kv_cache_379_b200.step import host_step


def test_random_operation_sequences_match():
    rng = np.random.default_rng(17)
    n, bs = 96, 4
    order = rng.permutation(n)
    a = BlockPool(n, bs, free_order=order)
    b = OraclePool(n, bs, free_order=order.tolist())
    seqs_a, seqs_b = [], []
    for _ in range(600):
        op = int(rng.integers(0, 5))
        if op == 0 or not seqs_a:
            k = int(rng.integers(1, 6))
            try:
                ta = a.allocate(k)
            except PagedKVError as e:
                assert e.status == -6
                with pytest.raises(PoolExhausted):
                    b.allocate(k)
                continue
            assert ta == b.allocate(k)
            seqs_a.append(ta)
            seqs_b.append(list(ta))
        elif op == 1:
            i = int(rng.integers(len(seqs_a)))
            seqs_a.append(a.fork(seqs_a[i]))
            seqs_b.append(b.fork(seqs_b[i]))
        elif op == 2:
            i = int(rng.integers(len(seqs_a)))
            j = int(rng.integers(len(seqs_a[i])))
            try:
                ra = a.allocate_or_get_cow(seqs_a[i][j])
            except PagedKVError:
                with pytest.raises(PoolExhausted):
                    b.allocate_or_get_cow(seqs_b[i][j])
                continue
            rb = b.allocate_or_get_cow(seqs_b[i][j])
            assert ra == rb
            seqs_a[i][j] = ra[0]
            seqs_b[i][j] = rb[0]
        else:
            i = int(rng.integers(len(seqs_a)))
            a.free_table(seqs_a.pop(i))
            b.free_sequence(seqs_b.pop(i))
        assert a.get_num_free_blocks() == b.get_num_free_blocks()
    assert a.refcounts() == b.refcount


def test_bad_block_ids_are_rejected():
    p = BlockPool(4, 16)
    with pytest.raises(PagedKVError):
        p.free(2)                       # not allocated
    with pytest.raises(PagedKVError):
        p.fork([7])
    with pytest.raises(ValueError):
        BlockPool(4, 16, free_order=[0, 1, 1, 2])


def _oracle_host_step(w, fork_all):
    """The same step with the oracle pool: adopt tables, optional fork, append a token."""
    tables = [list(w.block_tables[s, :w.blocks_per_seq[s]]) for s in range(w.num_seqs)]
    unowned = list(w.free_blocks)
    owned = sorted(set(range(w.num_blocks)) - set(unowned))
    pool = OraclePool(w.num_blocks, w.block_size, free_order=owned + unowned[::-1])
    # adoption: every table reference is an owner; adopted blocks leave the free list
    for t in tables:
        for blk in t:
            pool.refcount[blk] += 1
    pool.free_list = [x for x in pool.free_list if pool.refcount[x] == 0]
    if fork_all:
        for t in tables:
            pool.fork(t)
    slots, pairs = [], []
    for s, t in enumerate(tables):
        slot, pair, _ = pool.append_token(t, int(w.seq_lens[s]) - 1)
        slots.append(slot)
        if pair:
            pairs.append(pair)
    return pool, tables, slots, pairs


@pytest.mark.parametrize("name,kw,fork_all", [
    ("tiny", {}, False),
    ("shared", {"num_seqs": 64}, True),
    ("shared", {"num_seqs": 8, "shared_prompt_len": 1020, "lengths": [1] * 8}, False),
])
def test_host_step_matches_oracle_pool(name, kw, fork_all):
    w = wl.make(name, fill_cache=False, **kw)
    pool, tables, nblk, slots, pairs = host_step(w, fork_all=fork_all)
    opool, otables, oslots, opairs = _oracle_host_step(w, fork_all)
    assert slots.tolist() == oslots
    assert [tuple(p) for p in pairs.tolist()] == opairs
    for s in range(w.num_seqs):
        assert tables[s, :nblk[s]].tolist() == otables[s]
    assert pool.refcounts() == opool.refcount
    # the device-side address translation agrees with the pool's slots (oracle form)
    got = oracle.slot_mapping(tables, np.arange(w.num_seqs, dtype=np.int32),
                              w.seq_lens.astype(np.int64) - 1, w.block_size)
    assert got.tolist() == oslots
    if name == "shared" and not fork_all:
        assert len(pairs) == 7          # 8 samples write into their shared partial block


def test_shared_workload_pair_count():
    """Fork snapshot + one token: a copy per sequence unless its token opens a new block."""
    w = wl.make("shared", fill_cache=False)
    _, tables, nblk, slots, pairs = host_step(w, fork_all=True)
    opening = int(np.sum((w.seq_lens - 1) % w.block_size == 0))
    assert len(pairs) == w.num_seqs - opening
    assert len(set(pairs[:, 1].tolist())) == len(pairs)
    assert not set(pairs[:, 1].tolist()) & set(pairs[:, 0].tolist())


def test_swap_plan_matches_oracle_and_keeps_bookkeeping():
    from oracle.pool import swap_plan as o_swap_plan
    from paged_kv_cache_379_b200.pool import swap_plan
    rng = np.random.default_rng(11)
    gpu_order, cpu_order = rng.permutation(64), rng.permutation(32)
    g, c = BlockPool(64, 16, free_order=gpu_order), BlockPool(32, 16, free_order=cpu_order)
    og, oc = OraclePool(64, 16, free_order=gpu_order.tolist()), OraclePool(32, 16, free_order=cpu_order.tolist())
    t1 = g.allocate(5)
    assert t1 == og.allocate(5)
    t2 = g.fork(t1[:3]) + g.allocate(2)          # shares 3 blocks with t1
    ot2 = og.fork(t1[:3]) + og.allocate(2)
    assert t2 == ot2
    # swap t2 out to the host pool
    new2, pairs = swap_plan(g, c, t2)
    onew2, opairs = o_swap_plan(og, oc, list(t2))
    assert new2 == onew2 and [tuple(p) for p in pairs.tolist()] == opairs
    assert g.refcounts() == og.refcount and c.refcounts() == oc.refcount
    assert all(g.refcount(b) == 1 for b in t1[:3])     # t1 still owns the shared blocks
    # and back in
    back, pairs_in = swap_plan(c, g, new2)
    oback, opairs_in = o_swap_plan(oc, og, list(new2))
    assert back == oback and [tuple(p) for p in pairs_in.tolist()] == opairs_in
    assert c.get_num_free_blocks() == 32 and g.refcounts() == og.refcount
    # a table repeating a block maps it once, with the repeat count as its refcount
    t3 = g.allocate(1)
    og.allocate(1)
    g.fork(t3)
    og.fork(list(t3))
    new3, p3 = swap_plan(g, c, t3 + t3)
    onew3, op3 = o_swap_plan(og, oc, list(t3 + t3))
    assert new3 == onew3 and len(p3) == 1 and c.refcount(new3[0]) == 2


def test_cow_sources_matches_brute_force():
    """pa_cow_sources: each sequence's copy source is the src of the pair whose
    dst holds its slot; -1 without one or for slot -1; duplicate destinations
    are rejected."""
    from paged_kv_cache_379_b200 import ops
    from paged_kv_cache_379_b200._lib import PagedKVError
    for kw, fork_all in (({}, True), ({"num_seqs": 8, "shared_prompt_len": 1020, "lengths": [1] * 8}, False)):
        w = wl.make("shared", fill_cache=False, **kw)
        _, tables, nblk, slots, pairs = host_step(w, fork_all=fork_all)
        slots = slots.copy()
        slots[0] = -1
        got = ops.cow_sources(slots, w.block_size, pairs)
        want = []
        for s in range(w.num_seqs):
            src = -1
            for a, b in pairs.tolist():
                if slots[s] >= 0 and b == slots[s] // w.block_size:
                    src = a
            want.append(src)
        assert got.tolist() == want
    assert ops.cow_sources(np.array([5, 9], np.int64), 4, np.zeros((0, 2), np.int64)).tolist() == [-1, -1]
    with pytest.raises(PagedKVError):
        ops.cow_sources(np.array([5], np.int64), 4, np.array([[1, 2], [3, 2]], np.int64))


def _groups_brute_force(tables, lens, bs, part):
    """The grouping rule written out: a run takes the next sequence while it
    shares at least one whole partition with the run's first sequence; the
    group's partitions are the minimum shared by its members (0 alone)."""
    bpp = part // bs

    def shared(a, b):
        n = min(lens[a], lens[b]) // part
        k = 0
        while k < n and all(tables[a][k * bpp + j] == tables[b][k * bpp + j] >= 0 for j in range(bpp)):
            k += 1
        return k
    start, parts, s = [], [], 0
    while s < len(lens):
        e, k = s + 1, None
        while e < len(lens) and shared(s, e) >= 1:
            k = shared(s, e) if k is None else min(k, shared(s, e))
            e += 1
        start.append(s)
        parts.append(k or 0)
        s = e
    return start + [len(lens)], parts


def test_prefix_groups_matches_brute_force():
    from paged_kv_cache_379_b200 import ops
    rng = np.random.default_rng(5)
    for trial in range(40):
        bs = int(rng.choice([4, 8, 16]))
        part = bs * int(rng.integers(1, 4))
        B = int(rng.integers(1, 12))
        width = 12
        tables = rng.integers(0, 50, (B, width)).astype(np.int32)
        for s in range(1, B):             # copy a random prefix of the previous row now and then
            if rng.random() < 0.6:
                n = int(rng.integers(0, width + 1))
                tables[s, :n] = tables[s - 1, :n]
        lens = rng.integers(0, width * bs + 1, B).astype(np.int32)
        gs, gp = ops.prefix_groups(tables, lens, bs, part)
        ws, wp = _groups_brute_force(tables.tolist(), lens.tolist(), bs, part)
        assert gs.tolist() == ws and gp.tolist() == wp, trial
    # the shared-prefix workload after the fork and the step's copies: 32 groups of 8
    w = wl.make("shared", fill_cache=False)
    _, tables, _, _, _ = host_step(w, fork_all=True)
    gs, gp = ops.prefix_groups(tables, w.seq_lens, w.block_size, 512)
    assert gs.tolist() == list(range(0, 257, 8)) and gp.tolist() == [2] * 32
