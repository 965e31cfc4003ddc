"""GPU parity of the FP8 (E4M3) KV cache: the quantising cache write bit for bit,
and paged decode over code caches within the attention tolerance, against the
oracle's FP8 functions."""

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


def _u8(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).to(DEV)


def _i32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(DEV)


def _same_codes(got: np.ndarray, ref: np.ndarray, nan_in: np.ndarray, what: str):
    """Codes equal bit for bit, except that for a NaN input any NaN code passes
    (the sign of a NaN is not part of the conversion's definition)."""
    nan_code = lambda c: (c & 0x7F) == 0x7F  # noqa: E731
    ok = (got == ref) | (nan_in & nan_code(got) & nan_code(ref))
    if not ok.all():
        i = np.flatnonzero(~ok.ravel())[0]
        raise AssertionError(f"{what}: {(~ok).sum()} codes differ, first at {np.unravel_index(i, ref.shape)}: "
                             f"gpu=0x{got.ravel()[i]:02X} ref=0x{ref.ravel()[i]:02X}")


# ---- cache write -----------------------------------------------------------------------

@pytest.mark.parametrize("k_scale,v_scale", [(1.0, 1.0), (0.37, 2.5), (0.0123, 1.0 / 3.0)])
def test_cache_write_every_bf16_pattern(k_scale, v_scale):
    """All 65536 bf16 bit patterns (zeros, subnormals, E4M3 midpoints, values past
    448, infinities, NaNs) through the quantising write, bit-exact."""
    Hkv, D, bs = 1, 128, 16
    T = 65536 // (Hkv * D)
    pats = np.arange(65536, dtype=np.uint32).astype(np.uint16).reshape(T, Hkv, D)
    key, value = pats, pats[::-1].copy()
    nb = T // bs
    slots = np.random.default_rng(7).permutation(nb * bs).astype(np.int64)
    ref_k = np.zeros((nb, bs, Hkv, D), np.uint8)
    ref_v = np.zeros_like(ref_k)
    oracle.reshape_and_cache_fp8(key, value, ref_k, ref_v, slots, bs, k_scale, v_scale)
    kc, vc = _u8(np.zeros_like(ref_k)), _u8(np.zeros_like(ref_v))
    ops.reshape_and_cache_fp8(bf16_to_device(key, DEV), bf16_to_device(value, DEV), kc, vc,
                              torch.from_numpy(slots).to(DEV), k_scale, v_scale)
    torch.cuda.synchronize()
    x = oracle.bf16_bits_to_f64(key)
    nan_k = np.zeros(ref_k.shape, bool)
    nan_k.reshape(-1, Hkv, D)[slots] = np.isnan(x)
    nan_v = np.zeros(ref_v.shape, bool)
    nan_v.reshape(-1, Hkv, D)[slots] = np.isnan(oracle.bf16_bits_to_f64(value))
    _same_codes(kc.cpu().numpy(), ref_k, nan_k, "key codes")
    _same_codes(vc.cpu().numpy(), ref_v, nan_v, "value codes")


def test_cache_write_skips_negative_slots_and_keeps_other_slots():
    rng = np.random.default_rng(11)
    T, Hkv, D, bs, nb = 37, 4, 128, 8, 12
    key = wl.bf16_normal(rng, (T, Hkv, D))
    value = wl.bf16_normal(rng, (T, Hkv, D))
    slots = rng.permutation(nb * bs)[:T].astype(np.int64)
    slots[[3, 17, 30]] = -1
    init_k = wl.fp8_codes(rng, (nb, bs, Hkv, D))
    init_v = wl.fp8_codes(rng, (nb, bs, Hkv, D))
    ref_k, ref_v = init_k.copy(), init_v.copy()
    oracle.reshape_and_cache_fp8(key, value, ref_k, ref_v, slots, bs, 0.02, 0.05)
    kc, vc = _u8(init_k), _u8(init_v)
    ops.reshape_and_cache_fp8(bf16_to_device(key, DEV), bf16_to_device(value, DEV), kc, vc,
                              torch.from_numpy(slots).to(DEV), 0.02, 0.05)
    torch.cuda.synchronize()
    no_nan = np.zeros(ref_k.shape, bool)
    _same_codes(kc.cpu().numpy(), ref_k, no_nan, "key cache")
    _same_codes(vc.cpu().numpy(), ref_v, no_nan, "value cache")


# ---- decode ----------------------------------------------------------------------------

LENS = [0, 1, 2, 15, 16, 17, 31, 33, 64, 100, 255, 257, 513, 700, 1025, 2000]


def _fp8_case(seed, Hq, Hkv, bs, lens, poison=True):
    w = wl.random_decode_case(seed, num_seqs=len(lens), num_heads=Hq, num_kv_heads=Hkv, head_dim=128,
                              block_size=bs, lengths=lens)
    rng = np.random.default_rng(seed + 1)
    kc = wl.fp8_cache(rng, w.num_blocks, bs, Hkv, 128, w.free_blocks)
    vc = wl.fp8_cache(rng, w.num_blocks, bs, Hkv, 128, w.free_blocks)
    if poison:  # slots past each sequence's end hold the NaN code: never read
        for s, L in enumerate(w.seq_lens):
            if L > 0 and L % bs:
                last = int(w.block_tables[s, (L - 1) // bs])
                kc[last, L % bs:] = wl.E4M3_NAN
                vc[last, L % bs:] = wl.E4M3_NAN
    return w, kc, vc


def _decode(w, kc, vc, k_scale, v_scale, partition):
    args = (bf16_to_device(w.query, DEV), _u8(kc), _u8(vc), _i32(w.block_tables), _i32(w.seq_lens), w.scale,
            k_scale, v_scale, w.max_seq_len)
    if partition is None:
        ws = ops.new_workspace(w.num_seqs, w.num_heads, w.num_kv_heads, 128, w.max_seq_len, device=DEV)
        out = ops.decode_fp8(*args, workspace=ws)
    elif partition == 0:
        out = ops.decode_fp8_split(*args, 0, None)
    else:
        ws = ops.new_workspace(w.num_seqs, w.num_heads, w.num_kv_heads, 128, w.max_seq_len, partition,
                               device=DEV)
        out = ops.decode_fp8_split(*args, partition, ws)
    torch.cuda.synchronize()
    return bf16_to_host_bits(out)


@pytest.mark.parametrize("bs", [8, 16])
@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (8, 4), (8, 1), (16, 2), (6, 2), (16, 1)])
@pytest.mark.parametrize("partition", [0, 64, 256, None])
def test_decode_fp8_matches_oracle(bs, Hq, Hkv, partition):
    seed = 5000 + 7 * bs + 31 * Hq + Hkv
    w, kc, vc = _fp8_case(seed, Hq, Hkv, bs, LENS)
    ks, vs = 0.045, 0.3
    ref = oracle.paged_decode_fp8(w.query, kc, vc, w.block_tables, w.seq_lens, w.scale, ks, vs, threads=8)
    got = _decode(w, kc, vc, ks, vs, partition)
    assert_close(got, ref, f"fp8 bs={bs} G={Hq // Hkv} partition={partition}")
    assert ops.device_status() == 0


def test_decode_fp8_subnormal_and_extreme_codes():
    """Codes from the whole finite range: subnormals, 448, negative zero."""
    w, kc, vc = _fp8_case(77, 8, 2, 16, [5, 48, 300])
    rng = np.random.default_rng(78)
    finite = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)
    for s, L in enumerate(w.seq_lens):
        for j in range(-(-int(L) // 16)):
            b = int(w.block_tables[s, j])
            kc[b] = rng.choice(finite, kc[b].shape)
            vc[b] = rng.choice(finite, vc[b].shape)
    ks, vs = 1e-3, 1.0 / 448.0
    ref = oracle.paged_decode_fp8(w.query, kc, vc, w.block_tables, w.seq_lens, w.scale, ks, vs, threads=4)
    for partition in (0, 32):
        assert_close(_decode(w, kc, vc, ks, vs, partition), ref, f"extreme codes, partition={partition}")


def _wide_range_queries(rng, num_seqs, num_heads, head_dim):
    """bf16 queries whose heads reach the edges of the FP8 decode's query split
    (each head is scaled by a power of two so that its largest |q| lies in
    [128, 256) and split into two E4M3 terms: exact within 2^9 of the largest
    element, an error below 2^-17 of it further down).  Head kinds, by h % 5:
      0: one element of magnitude in [2^7, 2^8], the rest log-uniform in
         [2^-10, 2^7] (a range of up to 2^18);
      1: one element in [2^7, 2^8], the rest log-uniform in [2^-2, 2^7]
         (inside 2^9 of the largest: the split is exact);
      2: every element log-uniform in [2^-14, 2^-8] (scaled up by 2^15..2^22);
      3: N(0, 1);
      4: all zeros but one element of 2^-10."""
    q = np.empty((num_seqs, num_heads, head_dim), np.float32)
    sign = lambda *shape: rng.choice(np.array([-1.0, 1.0], np.float32), shape)  # noqa: E731
    for s in range(num_seqs):
        for h in range(num_heads):
            kind = h % 5
            if kind in (0, 1):
                lo = -10.0 if kind == 0 else -2.0
                row = sign(head_dim) * np.exp2(rng.uniform(lo, 7.0, head_dim))
                row[rng.integers(head_dim)] = sign(1)[0] * rng.uniform(128.0, 256.0)
            elif kind == 2:
                row = sign(head_dim) * np.exp2(rng.uniform(-14.0, -8.0, head_dim))
            elif kind == 3:
                row = rng.standard_normal(head_dim)
            else:
                row = np.zeros(head_dim)
                row[rng.integers(head_dim)] = 2.0 ** -10
            q[s, h] = row
    return wl.f32_to_bf16_bits(q)


@pytest.mark.parametrize("Hq,Hkv", [(8, 1), (16, 2), (5, 5)])
@pytest.mark.parametrize("partition", [0, 64])
def test_decode_fp8_wide_range_queries(Hq, Hkv, partition):
    """Queries with one large element and many small ones, heads of tiny
    magnitude, and near-zero heads, through the FP8 decode against the
    oracle, which keeps the exact bf16 query."""
    lens = [1, 16, 33, 200, 513, 1000]
    w, kc, vc = _fp8_case(6100 + Hq + Hkv, Hq, Hkv, 16, lens)
    w.query = _wide_range_queries(np.random.default_rng(6200 + Hq), w.num_seqs, Hq, 128)
    ks, vs = 0.045, 0.3
    ref = oracle.paged_decode_fp8(w.query, kc, vc, w.block_tables, w.seq_lens, w.scale, ks, vs, threads=8)
    got = _decode(w, kc, vc, ks, vs, partition)
    assert_close(got, ref, f"fp8 wide-range q, G={Hq // Hkv} partition={partition}")
    assert ops.device_status() == 0


def test_write_then_decode_fp8():
    """One decode step on an FP8 cache: the new token is quantised into its slot,
    then read back by the decode."""
    Hq, Hkv, bs = 8, 2, 16
    lens = [1, 16, 17, 200, 513]
    w, kc, vc = _fp8_case(91, Hq, Hkv, bs, lens, poison=False)
    slots = oracle.slot_mapping(w.block_tables, np.arange(w.num_seqs, dtype=np.int32),
                                w.seq_lens.astype(np.int64) - 1, bs)
    ks, vs = 0.01, 0.02
    ref_k, ref_v = kc.copy(), vc.copy()
    oracle.reshape_and_cache_fp8(w.new_key, w.new_value, ref_k, ref_v, slots, bs, ks, vs)
    ref = oracle.paged_decode_fp8(w.query, ref_k, ref_v, w.block_tables, w.seq_lens, w.scale, ks, vs, threads=4)
    dk, dv = _u8(kc), _u8(vc)
    ops.reshape_and_cache_fp8(bf16_to_device(w.new_key, DEV), bf16_to_device(w.new_value, DEV), dk, dv,
                              torch.from_numpy(slots).to(DEV), ks, vs)
    out = ops.decode_fp8(bf16_to_device(w.query, DEV), dk, dv, _i32(w.block_tables), _i32(w.seq_lens), w.scale,
                         ks, vs, w.max_seq_len)
    torch.cuda.synchronize()
    assert np.array_equal(dk.cpu().numpy(), ref_k) and np.array_equal(dv.cpu().numpy(), ref_v)
    assert_close(bf16_to_host_bits(out), ref, "write then decode")


def test_decode_fp8_rejects_unsupported_shapes():
    w, kc, vc = _fp8_case(3, 4, 4, 16, [20])
    q = bf16_to_device(w.query, DEV)
    bt, sl = _i32(w.block_tables), _i32(w.seq_lens)
    with pytest.raises(ops.PagedKVError):
        ops.decode_fp8(q, _u8(kc), _u8(vc), bt, sl, w.scale, 0.0, 1.0, 20)  # scale must be > 0
    with pytest.raises(ops.PagedKVError):
        ops.decode_fp8(q, _u8(kc), _u8(vc), bt, sl, w.scale, float("inf"), 1.0, 20)
    w4 = wl.random_decode_case(4, num_seqs=1, num_heads=4, num_kv_heads=4, head_dim=128, block_size=4,
                               lengths=[20])
    kc4 = _u8(np.zeros((w4.num_blocks, 4, 4, 128), np.uint8))
    with pytest.raises(ops.PagedKVError):  # block_size 4 is not compiled for FP8
        ops.decode_fp8(bf16_to_device(w4.query, DEV), kc4, kc4, _i32(w4.block_tables), _i32(w4.seq_lens),
                       w4.scale, 1.0, 1.0, 20)
    w64 = wl.random_decode_case(5, num_seqs=1, num_heads=4, num_kv_heads=4, head_dim=64, block_size=16,
                                lengths=[20])
    kc64 = _u8(np.zeros((w64.num_blocks, 16, 4, 64), np.uint8))
    with pytest.raises(ops.PagedKVError):  # head_dim 64 is not compiled for FP8
        ops.decode_fp8(bf16_to_device(w64.query, DEV), kc64, kc64, _i32(w64.block_tables), _i32(w64.seq_lens),
                       w64.scale, 1.0, 1.0, 20)
    torch.cuda.synchronize()
    assert ops.device_status() == 0


def test_fp8_bench_workload_full_batch():
    """The bench's FP8 row in its launch configuration: the gqa batch (128
    sequences, 64 query / 8 KV heads) over E4M3 caches, one decode step through
    the fused slot mapping + quantising cache write, then the planned decode;
    caches bit-exact and every output element against the oracle."""
    import bench
    w = wl.make("gqa", seed=bench.rank_seed(0), fill_cache=False)
    rng = np.random.Generator(np.random.PCG64(bench.rank_seed(0) + 17))
    kc = wl.fp8_cache(rng, w.num_blocks, w.block_size, w.num_kv_heads, w.head_dim, w.free_blocks)
    vc = wl.fp8_cache(rng, w.num_blocks, w.block_size, w.num_kv_heads, w.head_dim, w.free_blocks)
    ks, vs = 0.25, 0.25
    slots = oracle.slot_mapping(w.block_tables, np.arange(w.num_seqs, dtype=np.int32),
                                w.seq_lens.astype(np.int64) - 1, w.block_size)
    ref_k, ref_v = kc.copy(), vc.copy()
    oracle.reshape_and_cache_fp8(w.new_key, w.new_value, ref_k, ref_v, slots, w.block_size, ks, vs)
    ref = oracle.paged_decode_fp8(w.query, ref_k, ref_v, w.block_tables, w.seq_lens, w.scale, ks, vs, threads=0)
    dk, dv = _u8(kc), _u8(vc)
    bt, sl = _i32(w.block_tables), _i32(w.seq_lens)
    ops.append_decode_kv_fp8(bf16_to_device(w.new_key, DEV), bf16_to_device(w.new_value, DEV), dk, dv, bt, sl, ks, vs)
    ws = ops.new_workspace(w.num_seqs, w.num_heads, w.num_kv_heads, w.head_dim, w.max_seq_len, device=DEV)
    out = ops.decode_fp8(bf16_to_device(w.query, DEV), dk, dv, bt, sl, w.scale, ks, vs, w.max_seq_len, workspace=ws)
    torch.cuda.synchronize()
    assert np.array_equal(dk.cpu().numpy(), ref_k) and np.array_equal(dv.cpu().numpy(), ref_v)
    assert_close(bf16_to_host_bits(out), ref, "gqa FP8 batch")
    assert ops.device_status() == 0
