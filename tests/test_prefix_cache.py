"""Prefix caching in the block pool: the oracle's FNV-1a pinned to the published
test vectors, the page's sharing rule on a worked case, and the native pool
against the oracle pool (CPU only)."""

import numpy as np
import pytest

from oracle.pool import OraclePool, PoolExhausted, block_hash as o_block_hash, fnv1a_64
from paged_kv_cache_379_b200._lib import PagedKVError
from paged_kv_cache_379_b200.pool import BlockPool, block_hash


def test_fnv1a_published_vectors():
    # FNV-1a 64-bit reference values for "" and "a", and the definition itself
    assert fnv1a_64(b"") == 0xCBF29CE484222325
    assert fnv1a_64(b"a") == 0xAF63DC4C8601EC8C
    assert fnv1a_64(b"ab") == fnv1a_64(b"b", fnv1a_64(b"a"))


def test_block_hash_matches_oracle_and_chains():
    rng = np.random.default_rng(0)
    toks = rng.integers(0, 50000, size=16)
    h0 = block_hash(0, toks)
    assert h0 == o_block_hash(0, toks)
    assert block_hash(h0, toks) == o_block_hash(h0, toks) != h0
    assert block_hash(0, toks[:-1]) != h0


def _prompts():
    a = list(range(48))
    b = list(range(32)) + list(range(1000, 1016))
    c = list(range(100, 116)) + list(range(16, 32))
    return a, b, c


def test_prefix_cache_worked_case(golden):
    g = golden("prefix_cache_example.txt")
    a, b, c = _prompts()
    for pool in (BlockPool(16, g["block_size"]), OraclePool(16, g["block_size"])):
        ta, ca = pool.allocate_prompt_cached(a)
        assert ca == 0 and len(ta) == 3
        tb, cb = pool.allocate_prompt_cached(b)
        assert cb == g["b_cached_tokens"]
        assert tb[:g["b_reused_blocks"]] == ta[:g["b_reused_blocks"]] and tb[2] != ta[2]
        rc = pool.refcounts() if isinstance(pool, BlockPool) else pool.refcount
        assert [rc[x] for x in (ta[0], ta[1], ta[2], tb[2])] == g["refcount_after_b"]
        tc, cc = pool.allocate_prompt_cached(c)
        assert cc == g["c_cached_tokens"] and not set(tc) & set(ta)
        # a prompt equal to A reuses all three full blocks
        ta2, ca2 = pool.allocate_prompt_cached(a)
        assert ta2 == ta and ca2 == 48
        # a block leaves the cache once it is free: free every owner of A's blocks
        for t in (ta, ta2, tb):
            if isinstance(pool, BlockPool):
                pool.free_table(t)
            else:
                pool.free_sequence(list(t))
        _, c3 = pool.allocate_prompt_cached(a)
        assert c3 == 0


def test_partial_last_block_is_never_shared():
    for pool in (BlockPool(8, 16), OraclePool(8, 16)):
        t1, c1 = pool.allocate_prompt_cached(list(range(20)))
        t2, c2 = pool.allocate_prompt_cached(list(range(20)))
        assert c1 == 0 and c2 == 16
        assert t1[0] == t2[0] and t1[1] != t2[1]


def test_native_and_oracle_prefix_caches_agree():
    rng = np.random.default_rng(7)
    order = rng.permutation(200).tolist()
    a, b = BlockPool(200, 4, free_order=order), OraclePool(200, 4, free_order=order)
    bases = [rng.integers(0, 5, size=24).tolist() for _ in range(4)]
    live = []
    for step in range(300):
        op = rng.integers(0, 3)
        if op < 2 or not live:
            base = bases[int(rng.integers(4))]
            n = int(rng.integers(1, 24))
            toks = base[:n] + rng.integers(0, 5, size=int(rng.integers(0, 6))).tolist()
            try:
                ra = a.allocate_prompt_cached(toks)
            except PagedKVError as e:
                assert e.status == -6
                with pytest.raises(PoolExhausted):
                    b.allocate_prompt_cached(toks)
                continue
            rb = b.allocate_prompt_cached(toks)
            assert ra == rb
            live.append(ra[0])
        else:
            t = live.pop(int(rng.integers(len(live))))
            a.free_table(t)
            b.free_sequence(list(t))
        assert a.refcounts() == b.refcount
        assert a.get_num_free_blocks() == b.get_num_free_blocks()
        assert a.num_cached_blocks() == len(b.cache)
