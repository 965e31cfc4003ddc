"""GPU parity of the GPU <-> pinned host block swap (bit-exact against the oracle)."""

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_379_b200 import ops
from paged_kv_cache_379_b200._lib import PagedKVError

pytestmark = pytest.mark.gpu


def _cache(rng, nb, shape_tail):
    return rng.integers(0, 65535, size=(nb,) + shape_tail, dtype=np.uint16)


def _bf16(a, device=None, pin=False):
    t = torch.from_numpy(a.view(np.int16).copy()).view(torch.bfloat16)
    if pin:
        t = t.pin_memory()
    return t.to(device) if device else t


def _bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("bs,H,D", [(16, 8, 128), (4, 4, 64)])
def test_swap_out_and_in_bit_exact(bs, H, D):
    rng = np.random.default_rng(bs + H + D)
    gk, gv = _cache(rng, 96, (bs, H, D)), _cache(rng, 96, (bs, H, D))
    hk, hv = _cache(rng, 40, (bs, H, D)), _cache(rng, 40, (bs, H, D))
    dev_k, dev_v = _bf16(gk, "cuda"), _bf16(gv, "cuda")
    host_k, host_v = _bf16(hk, pin=True), _bf16(hv, pin=True)
    # swap out: 25 GPU blocks to distinct host blocks; pairs in device memory
    out_pairs = np.stack([rng.permutation(96)[:25], rng.permutation(40)[:25]], axis=1).astype(np.int64)
    ops.swap_blocks(host_k, host_v, dev_k, dev_v, torch.from_numpy(out_pairs).cuda())
    torch.cuda.synchronize()
    oracle.swap_blocks(hk, hv, gk, gv, out_pairs)
    assert np.array_equal(_bits(host_k), hk) and np.array_equal(_bits(host_v), hv)
    # swap in: host blocks back to other GPU blocks; pairs in pinned host memory
    in_pairs = np.stack([out_pairs[:, 1], rng.permutation(96)[:25]], axis=1).astype(np.int64)
    ops.swap_blocks(dev_k, dev_v, host_k, host_v, torch.from_numpy(in_pairs).pin_memory())
    torch.cuda.synchronize()
    oracle.swap_blocks(gk, gv, hk, hv, in_pairs)
    assert np.array_equal(_bits(dev_k), gk) and np.array_equal(_bits(dev_v), gv)


def test_swap_rejects_pageable_host_memory():
    rng = np.random.default_rng(3)
    dev_k = _bf16(_cache(rng, 8, (16, 8, 128)), "cuda")
    dev_v = _bf16(_cache(rng, 8, (16, 8, 128)), "cuda")
    host_k = _bf16(_cache(rng, 8, (16, 8, 128)))      # pageable
    host_v = _bf16(_cache(rng, 8, (16, 8, 128)))
    pairs = torch.tensor([[0, 1]], dtype=torch.int64, device="cuda")
    lib = ops.load()
    rc = lib.pa_swap_blocks(host_k.data_ptr(), host_v.data_ptr(), dev_k.data_ptr(), dev_v.data_ptr(),
                            pairs.data_ptr(), 1, 8, 128, 16, 8, 8, torch.cuda.current_stream().cuda_stream)
    assert rc == -11
    with pytest.raises(ValueError):
        ops.swap_blocks(host_k, host_v, dev_k, dev_v, pairs)


def test_swap_bench_plan_round_trip_full_size():
    """The bench's swap row at full size: a quarter of the GQA batch's blocks
    out to pinned host memory and back into the GPU pool through the host
    pool's plans, compared bit for bit with the oracle's copies applied to host
    copies of the same caches (the host cache and the whole GPU cache after
    each direction)."""
    import bench
    from paged_kv_cache_379_b200 import workload as wlmod
    w = wlmod.make("gqa", seed=bench.rank_seed(0, "gqa"))
    tables, swapped, n_host, out_pairs, in_pairs = bench.swap_row_plan(w)
    gk, gv = w.key_cache.copy(), w.value_cache.copy()
    dev_k, dev_v = _bf16(gk, "cuda"), _bf16(gv, "cuda")
    hk = np.zeros((n_host,) + gk.shape[1:], np.uint16)
    hv = np.zeros_like(hk)
    host_k, host_v = _bf16(hk, pin=True), _bf16(hv, pin=True)
    ops.swap_blocks(host_k, host_v, dev_k, dev_v, torch.from_numpy(out_pairs).cuda())
    torch.cuda.synchronize()
    oracle.swap_blocks(hk, hv, gk, gv, out_pairs)
    assert np.array_equal(_bits(host_k), hk) and np.array_equal(_bits(host_v), hv)
    ops.swap_blocks(dev_k, dev_v, host_k, host_v, torch.from_numpy(in_pairs).cuda())
    torch.cuda.synchronize()
    oracle.swap_blocks(gk, gv, hk, hv, in_pairs)
    assert np.array_equal(_bits(dev_k), gk) and np.array_equal(_bits(dev_v), gv)
    # every swapped sequence's blocks hold their content again, at the blocks
    # the swap-in chose
    moved = dict(zip(out_pairs[:, 0].tolist(), out_pairs[:, 1].tolist()))
    back = dict(zip(in_pairs[:, 0].tolist(), in_pairs[:, 1].tolist()))
    for s in swapped[:4]:
        for b in tables[s][tables[s] >= 0]:
            assert np.array_equal(gk[back[moved[int(b)]]], w.key_cache[b])
