"""Pins of the oracle to things other than itself (CPU only).

Each test checks the oracle against what the pages fix or what mathematics
fixes: the pages' worked examples (tests/golden/), an independent library
routine (torch's fp64 scaled_dot_product_attention on contiguous K/V), closed
forms, and invariants (permutation of physical blocks, merge of partitions).
"""

import numpy as np
import pytest
import torch

import oracle
from oracle.pool import OraclePool, slot_of
from paged_kv_cache_379_b200 import workload as wl


def _contiguous(case, s, g):
    """Logical K/V rows of sequence s, KV head g, read back through numpy indexing of the table."""
    L = int(case.seq_lens[s])
    bs = case.block_size
    pos = np.arange(L)
    phys = case.block_tables[s, pos // bs]
    k = oracle.bf16_bits_to_f64(case.key_cache[phys, pos % bs, g])
    v = oracle.bf16_bits_to_f64(case.value_cache[phys, pos % bs, g])
    return k, v


def _sdpa_reference(case):
    """torch SDPA (math backend, fp64) per sequence, GQA by enable_gqa."""
    B, Hq, D = case.query.shape
    Hkv = case.num_kv_heads
    out = np.zeros((B, Hq, D))
    for s in range(B):
        L = int(case.seq_lens[s])
        if L == 0:
            continue
        ks, vs = zip(*[_contiguous(case, s, g) for g in range(Hkv)])
        k = torch.from_numpy(np.stack(ks))[None]          # [1, Hkv, L, D]
        v = torch.from_numpy(np.stack(vs))[None]
        q = torch.from_numpy(oracle.bf16_bits_to_f64(case.query[s]))[None, :, None, :]  # [1, Hq, 1, D]
        o = torch.nn.functional.scaled_dot_product_attention(q, k, v, scale=case.scale,
                                                             enable_gqa=(Hq != Hkv))
        out[s] = o[0, :, 0, :].numpy()
    return out


# ---- address translation and allocation: the pages' worked examples ----------

def test_page_table_example(golden):
    g = golden("page_table_example.txt")
    table = np.array([g["page_table"]], dtype=np.int32)
    pos = np.array(g["positions"], dtype=np.int64)
    got = oracle.slot_mapping(table, np.zeros(len(pos), np.int32), pos, g["block_size"])
    assert got.tolist() == g["slots"]
    assert [slot_of(g["page_table"], int(p), g["block_size"]) for p in pos] == g["slots"]


def test_fig6_block_size_4(golden):
    g = golden("fig6_block_size_4.txt")
    bs = g["block_size"]
    pool = OraclePool(16, bs)
    table = pool.allocate_prompt(g["prompt_tokens"])
    assert len(table) == g["logical_blocks"]
    fills = [sum(1 for p in range(g["prompt_tokens"]) if p // bs == j) for j in range(len(table))]
    assert fills == g["fill_per_block"]
    assert len(table) * bs - g["prompt_tokens"] == g["free_slots_in_last_block"]
    free_before = pool.get_num_free_blocks()
    slot8, pair8, alloc8 = pool.append_token(table, 7)
    assert (slot8 // bs, slot8 % bs) == (table[g["token8_logical_block"]], g["token8_offset"])
    assert int(alloc8) == g["token8_allocates"] and pair8 is None
    assert pool.get_num_free_blocks() == free_before
    slot9, pair9, alloc9 = pool.append_token(table, 8)
    assert int(alloc9) == g["token9_allocates"] and pair9 is None
    assert len(table) == g["token9_logical_block"] + 1
    assert (slot9 // bs, slot9 % bs) == (table[g["token9_logical_block"]], g["token9_offset"])
    assert pool.get_num_free_blocks() == free_before - 1
    # the oracle's C translation agrees with the pool's slots
    t = np.array([table], dtype=np.int32)
    got = oracle.slot_mapping(t, np.zeros(2, np.int32), np.array([7, 8]), bs)
    assert got.tolist() == [slot8, slot9]


def test_page_growth_block_size_16(golden):
    g = golden("page_growth_block_size_16.txt")
    pool = OraclePool(8, g["block_size"])
    table = []
    pages = {}
    for token in range(1, 18):          # token n sits at position n - 1
        pool.append_token(table, token - 1)
        pages[token] = len(table)
    assert pages[5] == g["pages_at_token_5"]
    assert pages[16] == g["pages_at_token_16"]
    assert pages[17] == g["pages_at_token_17"]


# ---- decode: an independent library routine and closed forms -----------------

@pytest.mark.parametrize("bs,Hq,Hkv,D,lens", [
    (1, 2, 2, 8, [1, 3, 5]),
    (4, 4, 4, 64, [7, 16, 33, 50]),
    (16, 8, 2, 32, [1, 16, 17, 40]),
    (16, 8, 1, 16, [31, 2]),
])
def test_decode_matches_torch_sdpa(bs, Hq, Hkv, D, lens):
    case = wl.random_decode_case(7, num_seqs=len(lens), num_heads=Hq, num_kv_heads=Hkv,
                                 head_dim=D, block_size=bs, lengths=lens)
    got = oracle.paged_decode(case.query, case.key_cache, case.value_cache,
                              case.block_tables, case.seq_lens, case.scale)
    ref = _sdpa_reference(case)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_decode_identity_table_contiguous():
    """Identity table over a contiguous cache = plain attention over that array."""
    bs, H, D, L = 4, 3, 16, 10
    case = wl.random_decode_case(3, num_seqs=1, num_heads=H, num_kv_heads=H, head_dim=D,
                                 block_size=bs, lengths=[L], spare_blocks=0)
    nb = case.num_blocks
    case.block_tables[0, :nb] = np.arange(nb)
    got = oracle.paged_decode(case.query, case.key_cache, case.value_cache,
                              case.block_tables, case.seq_lens, case.scale)
    k = torch.from_numpy(oracle.bf16_bits_to_f64(case.key_cache.reshape(nb * bs, H, D)[:L]))
    v = torch.from_numpy(oracle.bf16_bits_to_f64(case.value_cache.reshape(nb * bs, H, D)[:L]))
    q = torch.from_numpy(oracle.bf16_bits_to_f64(case.query[0]))
    ref = torch.nn.functional.scaled_dot_product_attention(
        q[:, None, :], k.permute(1, 0, 2), v.permute(1, 0, 2), scale=case.scale)[:, 0, :]
    np.testing.assert_allclose(got[0], ref.numpy(), rtol=1e-12, atol=1e-12)


def test_decode_permutation_invariance():
    """Physical placement does not matter, only logical order (bitwise in the oracle)."""
    case = wl.random_decode_case(11, num_seqs=3, num_heads=4, num_kv_heads=2, head_dim=32,
                                 block_size=4, lengths=[5, 13, 21])
    base = oracle.paged_decode(case.query, case.key_cache, case.value_cache,
                               case.block_tables, case.seq_lens, case.scale)
    rng = np.random.default_rng(0)
    perm = rng.permutation(case.num_blocks)            # old id -> new id
    kc = np.empty_like(case.key_cache)
    vc = np.empty_like(case.value_cache)
    kc[perm] = case.key_cache
    vc[perm] = case.value_cache
    tables = np.where(case.block_tables >= 0, perm[np.maximum(case.block_tables, 0)], -1).astype(np.int32)
    moved = oracle.paged_decode(case.query, kc, vc, tables, case.seq_lens, case.scale)
    assert np.array_equal(base, moved)


def test_decode_closed_forms():
    bs, H, D = 4, 2, 16
    case = wl.random_decode_case(5, num_seqs=4, num_heads=H, num_kv_heads=H, head_dim=D,
                                 block_size=bs, lengths=[1, 9, 9, 9])
    kc, vc = case.key_cache.copy(), case.value_cache.copy()
    q = case.query.copy()
    # seq 1: every key equal -> uniform weights -> mean of V
    t1 = case.block_tables[1, :3]
    kc[t1] = kc[t1[0], 0][None, None]
    # seq 2: zero query -> uniform weights -> mean of V
    q[2] = 0
    # seq 3: key at position 6 aligned with a huge query -> that value row
    t3 = case.block_tables[3]
    q[3] = wl.f32_to_bf16_bits(np.full((H, D), 8.0, np.float32))
    kc[t3[:3]] = wl.f32_to_bf16_bits(np.zeros((3, bs, H, D), np.float32))
    kc[t3[6 // bs], 6 % bs] = wl.f32_to_bf16_bits(np.full((H, D), 1.0, np.float32))
    out = oracle.paged_decode(q, kc, vc, case.block_tables, case.seq_lens, case.scale)
    v = oracle.bf16_bits_to_f64(vc)
    # seq 0: L = 1 -> exactly v_0
    assert np.array_equal(out[0], v[case.block_tables[0, 0], 0])
    for s in (1, 2):
        tb = case.block_tables[s]
        rows = np.stack([v[tb[p // bs], p % bs] for p in range(9)])
        np.testing.assert_allclose(out[s], rows.mean(axis=0), rtol=0, atol=1e-12)
    # logit gap scale*8*16 = 32: the 8 other weights sum to below 1e-13
    np.testing.assert_allclose(out[3], v[t3[1], 2], rtol=0, atol=1e-12)


def test_decode_empty_sequence_is_zero():
    case = wl.random_decode_case(2, num_seqs=2, num_heads=2, num_kv_heads=1, head_dim=8,
                                 block_size=4, lengths=[0, 3], spare_blocks=1)
    out = oracle.paged_decode(case.query, case.key_cache, case.value_cache,
                              case.block_tables, case.seq_lens, case.scale)
    assert np.array_equal(out[0], np.zeros_like(out[0]))
    assert np.all(np.isfinite(out[1]))


def test_decode_ignores_poisoned_unused_slots_and_entries():
    """Slots past L in the last block and table entries past ceil(L/bs) are never read."""
    case = wl.random_decode_case(9, num_seqs=2, num_heads=2, num_kv_heads=2, head_dim=16,
                                 block_size=4, lengths=[6, 10])
    clean = oracle.paged_decode(case.query, case.key_cache, case.value_cache,
                                case.block_tables, case.seq_lens, case.scale)
    kc, vc = case.key_cache.copy(), case.value_cache.copy()
    for s, L in enumerate(case.seq_lens):
        last = case.block_tables[s, (L - 1) // 4]
        kc[last, L % 4 or 4:] = wl.BF16_NAN
        vc[last, L % 4 or 4:] = wl.BF16_NAN
    tables = np.concatenate([case.block_tables, np.full((2, 2), -1, np.int32)], axis=1)
    out = oracle.paged_decode(case.query, kc, vc, tables, case.seq_lens, case.scale)
    assert np.array_equal(out, clean)


def test_shared_prefix_identical_outputs():
    """Two sequences whose tables name the same physical blocks read the same K/V."""
    case = wl.random_decode_case(4, num_seqs=2, num_heads=4, num_kv_heads=2, head_dim=16,
                                 block_size=4, lengths=[11, 11])
    case.block_tables[1] = case.block_tables[0]
    case.query[1] = case.query[0]
    out = oracle.paged_decode(case.query, case.key_cache, case.value_cache,
                              case.block_tables, case.seq_lens, case.scale)
    assert np.array_equal(out[0], out[1])


@pytest.mark.parametrize("psize", [1, 4, 8, 24, 64])
def test_partitions_merge_to_full(psize):
    case = wl.random_decode_case(13, num_seqs=3, num_heads=4, num_kv_heads=2, head_dim=16,
                                 block_size=4, lengths=[1, 23, 50])
    full = oracle.paged_decode(case.query, case.key_cache, case.value_cache,
                               case.block_tables, case.seq_lens, case.scale)
    parts = -(-50 // psize)
    m, l, o = oracle.paged_decode_partials(case.query, case.key_cache, case.value_cache,
                                           case.block_tables, case.seq_lens, case.scale,
                                           psize, parts)
    merged = oracle.lse_merge(m, l, o)
    np.testing.assert_allclose(merged, full, rtol=1e-12, atol=1e-13)
    # one partition covering everything: o / l is the full result
    m1, l1, o1 = oracle.paged_decode_partials(case.query, case.key_cache, case.value_cache,
                                              case.block_tables, case.seq_lens, case.scale, 64, 1)
    np.testing.assert_allclose(o1[..., 0, :] / l1[..., 0, None], full, rtol=1e-12, atol=1e-13)
    # empty partitions carry m = -inf and l = 0
    assert np.all(np.isneginf(m[0, :, 1:])) and np.all(l[0, :, 1:] == 0)


def test_lse_merge_closed_form():
    """Two partitions with known (m, l, o): merge = (e^{m1-M} o1 + e^{m2-M} o2) / (...)."""
    m = np.array([[0.0, np.log(3.0)]])
    l = np.array([[2.0, 1.0]])
    o = np.array([[[2.0, 4.0], [1.0, -1.0]]])
    out = oracle.lse_merge(m, l, o)
    # weights 1 and 3: ((2,4) + 3*(1,-1)) / (2 + 3) = (1, 0.2)
    np.testing.assert_allclose(out[0], [1.0, 0.2], rtol=1e-15)
    assert np.array_equal(oracle.lse_merge(np.full((1, 2), -np.inf), np.zeros((1, 2)),
                                           np.zeros((1, 2, 2)))[0], [0.0, 0.0])


# ---- cache write and block copy ------------------------------------------------

def test_reshape_and_cache_then_decode_sees_new_token():
    """Fig. 6 case: 7 cached tokens at bs 4, token 8 written at position 7, then decoded."""
    bs, H, D = 4, 2, 16
    case = wl.random_decode_case(21, num_seqs=1, num_heads=H, num_kv_heads=H, head_dim=D,
                                 block_size=bs, lengths=[8])
    kc, vc = case.key_cache.copy(), case.value_cache.copy()
    slots = oracle.slot_mapping(case.block_tables, np.zeros(1, np.int32), np.array([7]), bs)
    before_k = kc.copy()
    oracle.reshape_and_cache(case.new_key, case.new_value, kc, vc, slots, bs)
    blk, off = divmod(int(slots[0]), bs)
    assert blk == case.block_tables[0, 1] and off == 3
    assert np.array_equal(kc[blk, off], case.new_key[0])
    assert np.array_equal(vc[blk, off], case.new_value[0])
    changed = np.argwhere(np.any(kc != before_k, axis=(2, 3)))
    assert changed.tolist() in ([[blk, off]], [])
    # negative slot = padding: nothing written
    kc2 = kc.copy()
    oracle.reshape_and_cache(case.new_key, case.new_value, kc2, vc.copy(), np.array([-1]), bs)
    assert np.array_equal(kc2, kc)
    out = oracle.paged_decode(case.query, kc, vc, case.block_tables, case.seq_lens, case.scale)
    # independent: torch SDPA over the logical rows, the new token last
    case.key_cache, case.value_cache = kc, vc
    np.testing.assert_allclose(out, _sdpa_reference(case), rtol=1e-12, atol=1e-12)


def test_copy_blocks_copies_whole_blocks_only():
    rng = np.random.default_rng(1)
    kc = rng.integers(0, 65535, size=(6, 4, 2, 8), dtype=np.uint16)
    vc = rng.integers(0, 65535, size=(6, 4, 2, 8), dtype=np.uint16)
    k0, v0 = kc.copy(), vc.copy()
    oracle.copy_blocks(kc, vc, [(1, 4), (2, 5)])
    assert np.array_equal(kc[4], k0[1]) and np.array_equal(vc[5], v0[2])
    assert np.array_equal(kc[[0, 1, 2, 3]], k0[[0, 1, 2, 3]])
    assert np.array_equal(vc[[0, 1, 2, 3]], v0[[0, 1, 2, 3]])
    oracle.copy_blocks(kc, vc, np.zeros((0, 2), np.int64))
    assert np.array_equal(kc[4], k0[1])


def test_swap_blocks_copies_between_caches():
    rng = np.random.default_rng(2)
    src_k = rng.integers(0, 65535, size=(5, 4, 2, 8), dtype=np.uint16)
    src_v = rng.integers(0, 65535, size=(5, 4, 2, 8), dtype=np.uint16)
    dst_k = rng.integers(0, 65535, size=(3, 4, 2, 8), dtype=np.uint16)
    dst_v = rng.integers(0, 65535, size=(3, 4, 2, 8), dtype=np.uint16)
    d0k, d0v, s0k = dst_k.copy(), dst_v.copy(), src_k.copy()
    oracle.swap_blocks(dst_k, dst_v, src_k, src_v, [(4, 0), (1, 2)])
    assert np.array_equal(dst_k[0], src_k[4]) and np.array_equal(dst_v[2], src_v[1])
    assert np.array_equal(dst_k[1], d0k[1]) and np.array_equal(dst_v[1], d0v[1])
    assert np.array_equal(src_k, s0k)


# ---- FP8 (E4M3) cache: the format's definition ------------------------------------

def test_e4m3_decode_fixed_points():
    # one, the largest finite value, the smallest normal and subnormal, signed zero, NaN
    assert oracle.e4m3_to_f64(0x38) == 1.0
    assert oracle.e4m3_to_f64(0x7E) == 448.0
    assert oracle.e4m3_to_f64(0x08) == 2.0 ** -6
    assert oracle.e4m3_to_f64(0x01) == 2.0 ** -9
    assert oracle.e4m3_to_f64(0x80) == 0.0 and oracle.e4m3_to_f64(0xB8) == -1.0
    assert np.isnan(oracle.e4m3_to_f64(0x7F)) and np.isnan(oracle.e4m3_to_f64(0xFF))
    vals = [oracle.e4m3_to_f64(c) for c in range(127)]
    assert all(a < b for a, b in zip(vals, vals[1:]))            # codes are ordered


def test_e4m3_round_to_nearest_even_and_saturate():
    # every code round-trips; midpoints go to the even code; overflow saturates
    for c in range(127):
        assert oracle.f64_to_e4m3(oracle.e4m3_to_f64(c)) == c
        assert oracle.f64_to_e4m3(-oracle.e4m3_to_f64(c)) == c | 0x80
    one, nxt = oracle.e4m3_to_f64(0x38), oracle.e4m3_to_f64(0x39)    # 1.0 and 1.125
    assert oracle.f64_to_e4m3((one + nxt) / 2) == 0x38              # tie -> even (0x38)
    assert oracle.f64_to_e4m3(one + (nxt - one) * 0.51) == 0x39
    nxt2 = oracle.e4m3_to_f64(0x3A)
    assert oracle.f64_to_e4m3((nxt + nxt2) / 2) == 0x3A              # tie -> even (0x3A)
    assert oracle.f64_to_e4m3(1000.0) == 0x7E and oracle.f64_to_e4m3(-1e9) == 0xFE
    assert oracle.f64_to_e4m3(float("inf")) == 0x7E and oracle.f64_to_e4m3(float("-inf")) == 0xFE
    assert oracle.f64_to_e4m3(464.0) == 0x7E    # halfway to the next binade's step: still 448
    assert oracle.f64_to_e4m3(-0.0) == 0x80 and oracle.f64_to_e4m3(0.0) == 0x00   # signed zero
    assert oracle.f64_to_e4m3(-1e-9) == 0x80 and oracle.f64_to_e4m3(1e-9) == 0x00  # underflow keeps the sign


def test_fp8_decode_equals_bf16_decode_of_the_dequantised_cache():
    """Decoding an E4M3 cache equals decoding the cache its codes stand for."""
    case = wl.random_decode_case(31, num_seqs=3, num_heads=8, num_kv_heads=2, head_dim=16,
                                 block_size=4, lengths=[3, 9, 14], spare_blocks=0)
    rng = np.random.default_rng(4)
    kc8 = rng.integers(0, 126, size=case.key_cache.shape, dtype=np.uint8) | (rng.integers(0, 2, size=case.key_cache.shape, dtype=np.uint8) << 7)
    vc8 = rng.integers(0, 126, size=case.key_cache.shape, dtype=np.uint8)
    ks, vs = 0.5, 0.25          # powers of two: the dequantised values are exact bf16 numbers
    deq = np.vectorize(oracle.e4m3_to_f64)
    kf = (deq(kc8) * ks).astype(np.float32)
    vf = (deq(vc8) * vs).astype(np.float32)
    got = oracle.paged_decode_fp8(case.query, kc8, vc8, case.block_tables, case.seq_lens, case.scale, ks, vs)
    ref = oracle.paged_decode(case.query, wl.f32_to_bf16_bits(kf), wl.f32_to_bf16_bits(vf),
                              case.block_tables, case.seq_lens, case.scale)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_fp8_cache_write_quantises_each_element():
    case = wl.random_decode_case(33, num_seqs=2, num_heads=2, num_kv_heads=2, head_dim=16,
                                 block_size=4, lengths=[5, 6])
    kc = np.zeros(case.key_cache.shape, np.uint8)
    vc = np.zeros(case.key_cache.shape, np.uint8)
    slots = np.array([3, 17], dtype=np.int64)
    oracle.reshape_and_cache_fp8(case.new_key, case.new_value, kc, vc, slots, 4, 0.03, 0.07)
    kinv = np.float32(1.0) / np.float32(0.03)
    for t, slot in enumerate(slots):
        for h in range(2):
            for d in range(16):
                x = np.float32(oracle.bf16_bits_to_f64(case.new_key[t, h, d:d + 1])[0]) * kinv
                assert kc[slot // 4, slot % 4, h, d] == oracle.f64_to_e4m3(float(np.float32(x)))
    assert np.count_nonzero(kc) <= 2 * 2 * 16


# ---- multi-query paged prefill (causal within the chunk) -----------------------------

def _prefill_case(seed, bs, Hq, Hkv, D, lens, q_lens):
    case = wl.random_decode_case(seed, num_seqs=len(lens), num_heads=Hq, num_kv_heads=Hkv, head_dim=D,
                                 block_size=bs, lengths=lens)
    q = wl.bf16_normal(np.random.default_rng(seed + 99), (int(sum(q_lens)), Hq, D))
    return case, q


def _sdpa_prefill(case, q_bits, q_lens):
    """torch SDPA (fp64) per sequence on the gathered rows, with the causal mask
    of a chunk that starts at position L - q_len."""
    Hq, D = q_bits.shape[1:]
    out = np.zeros(q_bits.shape)
    row = 0
    for s, (L, n) in enumerate(zip(case.seq_lens, q_lens)):
        L, n = int(L), int(n)
        if n == 0:
            continue
        ks, vs = zip(*[_contiguous(case, s, g) for g in range(case.num_kv_heads)])
        k = torch.from_numpy(np.stack(ks))[None]
        v = torch.from_numpy(np.stack(vs))[None]
        q = torch.from_numpy(oracle.bf16_bits_to_f64(q_bits[row:row + n])).permute(1, 0, 2)[None]  # [1, Hq, n, D]
        mask = torch.arange(L)[None, :] <= (L - n + torch.arange(n))[:, None]
        o = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=mask, scale=case.scale,
                                                             enable_gqa=(Hq != case.num_kv_heads))
        out[row:row + n] = o[0].permute(1, 0, 2).numpy()
        row += n
    return out


@pytest.mark.parametrize("bs,Hq,Hkv,D", [(4, 4, 4, 16), (16, 8, 2, 64), (8, 16, 1, 32)])
def test_prefill_matches_torch_sdpa_with_chunk_causal_mask(bs, Hq, Hkv, D):
    lens = [1, 7, 16, 40, 33, 5]
    q_lens = [1, 7, 5, 40, 1, 0]      # whole prompts, a mid chunk, single tokens, an idle sequence
    case, q = _prefill_case(21 + bs + D, bs, Hq, Hkv, D, lens, q_lens)
    got = oracle.paged_prefill(q, case.key_cache, case.value_cache, case.block_tables, case.seq_lens,
                               q_lens, case.scale)
    ref = _sdpa_prefill(case, q, q_lens)
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_prefill_of_single_tokens_is_decode():
    case, q = _prefill_case(31, 4, 8, 2, 16, [3, 9, 17], [1, 1, 1])
    got = oracle.paged_prefill(q, case.key_cache, case.value_cache, case.block_tables, case.seq_lens,
                               [1, 1, 1], case.scale)
    dec = oracle.paged_decode(q, case.key_cache, case.value_cache, case.block_tables, case.seq_lens, case.scale)
    assert np.array_equal(got, dec)


def test_prefill_chunks_equal_whole_prompt():
    """A prompt fed as chunks [0, 9), [9, 20), [20, 37) gives the rows of the
    whole-prompt prefill: each token's result depends only on its position."""
    L = 37
    case, q = _prefill_case(41, 8, 4, 2, 32, [L], [L])
    whole = oracle.paged_prefill(q, case.key_cache, case.value_cache, case.block_tables, case.seq_lens,
                                 [L], case.scale)
    for a, b in ((0, 9), (9, 20), (20, 37)):
        part = oracle.paged_prefill(q[a:b], case.key_cache, case.value_cache, case.block_tables,
                                    np.array([b], np.int32), [b - a], case.scale)
        assert np.array_equal(part, whole[a:b])


def test_prefill_first_position_and_permutation():
    case, q = _prefill_case(51, 4, 4, 4, 16, [6, 11], [6, 11])
    got = oracle.paged_prefill(q, case.key_cache, case.value_cache, case.block_tables, case.seq_lens,
                               [6, 11], case.scale)
    for s, row in ((0, 0), (1, 6)):   # position 0 attends to itself only: out = v_0
        _, v = zip(*[_contiguous(case, s, g) for g in range(4)])
        assert np.array_equal(got[row], np.stack([vv[0] for vv in v]))
    perm = np.random.default_rng(1).permutation(case.num_blocks)
    kc = np.empty_like(case.key_cache)
    vc = np.empty_like(case.value_cache)
    kc[perm] = case.key_cache
    vc[perm] = case.value_cache
    tables = np.where(case.block_tables >= 0, perm[np.maximum(case.block_tables, 0)], -1).astype(np.int32)
    moved = oracle.paged_prefill(q, kc, vc, tables, case.seq_lens, [6, 11], case.scale)
    assert np.array_equal(got, moved)
