"""The multi-GPU path of the benchmark, on CPU: two gloo ranks, each with its own
independent batch (weak scaling, no collective on the data path); the measured
time is the max over ranks and the work the sum over ranks."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        import oracle
        from paged_kv_cache_379_b200 import workload as wl

        w = wl.make("gqa", seed=bench.rank_seed(rank), num_seqs=4, fill_cache=True)
        # each rank's decode touches only its own batch (oracle stands in for the GPU here)
        out = oracle.paged_decode(w.query, w.key_cache, w.value_cache, w.block_tables, w.seq_lens, w.scale)
        step_bytes = bench.algorithmic_bytes(w.seq_lens, w.block_size, w.num_heads, w.num_kv_heads, w.head_dim)
        fake_ms = 10.0 + 5.0 * rank
        t, e, b, n = bench.aggregate_over_ranks(fake_ms, 2 * fake_ms, step_bytes, w.num_seqs, "cpu", dist)
        np.savez(os.path.join(out_dir, f"r{rank}.npz"), out=out, lens=w.seq_lens, step_bytes=step_bytes,
                 agg=np.array([t, e, b, n]))
    finally:
        dist.destroy_process_group()


def test_two_rank_weak_scaling_aggregation(tmp_path):
    world = 2
    mp.spawn(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    r = [np.load(tmp_path / f"r{i}.npz") for i in range(world)]
    # independent batches: different lengths / outputs per rank, same shapes
    assert r[0]["out"].shape == r[1]["out"].shape
    assert not np.array_equal(r[0]["lens"], r[1]["lens"])
    for i in range(world):
        t, e, b, n = r[i]["agg"]
        assert t == pytest.approx(15.0) and e == pytest.approx(30.0)     # max over ranks
        assert b == pytest.approx(float(r[0]["step_bytes"] + r[1]["step_bytes"]))  # summed
        assert n == 8
