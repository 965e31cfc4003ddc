"""The units bench.py reports: algorithmic bytes of a decode call, useful FLOPs
of a causal prefill, and the code-only hash that keys recorded ncu counters."""

import numpy as np

import bench


def test_algorithmic_bytes_hand_case():
    # 2 sequences of 5 and 17 positions, block size 4: 2 + 5 blocks touched;
    # 4 query / 2 KV heads, head_dim 8, bf16
    got = bench.algorithmic_bytes([5, 17], 4, 4, 2, 8)
    kv = 7 * 4 * 2 * 8 * 2 * 2          # blocks x bs x Hkv x D x (K, V) x 2 bytes
    q_and_out = 2 * 2 * 4 * 8 * 2        # (query, output) x B x Hq x D x 2 bytes
    tables_and_lens = 7 * 4 + 2 * 4      # one int32 per block touched, one length per sequence
    assert got == kv + q_and_out + tables_and_lens
    # an FP8 cache halves the KV term only
    assert bench.algorithmic_bytes([5, 17], 4, 4, 2, 8, 1) == kv // 2 + q_and_out + tables_and_lens
    # an empty sequence touches no block
    assert bench.algorithmic_bytes([0], 16, 8, 8, 128) == 2 * 8 * 128 * 2 + 4


def test_unique_bytes_counts_shared_blocks_once():
    # two sequences of 5 and 7 positions, block size 4, sharing their first block
    # (id 3): blocks touched 2 + 2, distinct 3; 2 query / 2 KV heads, head_dim 8
    tables = np.array([[3, 5], [3, 6]], np.int32)
    got = bench.unique_bytes(tables, [5, 7], 4, 2, 2, 8)
    kv = 3 * 4 * 2 * 8 * 2 * 2
    q_and_out = 2 * 2 * 2 * 8 * 2
    tables_and_lens = 4 * 4 + 2 * 4
    assert got == kv + q_and_out + tables_and_lens
    # without sharing it equals the algorithmic bytes
    assert bench.unique_bytes(np.array([[1, 2], [3, 4]], np.int32), [5, 7], 4, 2, 2, 8) == \
        bench.algorithmic_bytes([5, 7], 4, 2, 2, 8)


def test_prefill_flops_matches_brute_force():
    rng = np.random.default_rng(3)
    for _ in range(20):
        B = int(rng.integers(1, 5))
        lens = rng.integers(1, 200, B)
        q_lens = [int(rng.integers(1, L + 1)) for L in lens]
        pairs = 0
        for L, n in zip(lens, q_lens):
            for i in range(n):               # new token i sits at position L - n + i
                pairs += (L - n + i) + 1     # and sees positions 0 .. L - n + i
        assert bench.prefill_flops(lens, q_lens, 8, 64) == 4 * 64 * 8 * pairs
    # the bench's workload: 8 whole 2048-token prompts, 64 heads, d128
    n = 2048
    assert bench.prefill_flops([n] * 8, [n] * 8, 64, 128) == 4 * 128 * 64 * 8 * n * (n + 1) // 2


def test_code_hash_ignores_comments_and_layout_only():
    a = "int f(int x) {\n  // twice\n  return 2 * x; /* doubled */\n}\n"
    b = "int f(int x)   {   return 2 * x;\n\n}  // changed comment\n"
    c = "int f(int x) { return 3 * x; }"
    assert bench._code_only(a) == bench._code_only(b)
    assert bench._code_only(a) != bench._code_only(c)
    assert len(bench.kernel_source_hash()) == 16


def test_reference_arm_prints_one_contract_line():
    """`bench.py --impl reference` times the oracle on the host and prints one
    JSON line with the contract's keys (no GPU needed)."""
    import subprocess
    import sys

    r = subprocess.run([sys.executable, bench.__file__, "--impl", "reference", "--steps", "3", "--warmup", "3"],
                       capture_output=True, text=True, timeout=600)
    _check_reference_line(r)


def test_reference_arm_on_the_shared_prefix_step():
    """The reference arm decodes the shared-prefix step with the step's tables
    (each token's block present: fresh or copied), on a small batch."""
    import subprocess
    import sys

    r = subprocess.run([sys.executable, bench.__file__, "--impl", "reference", "--workload", "shared",
                        "--num-seqs", "16", "--steps", "3", "--warmup", "3"],
                       capture_output=True, text=True, timeout=600)
    d = _check_reference_line(r)
    assert d["config"]["num_seqs_per_gpu"] == 16


def _check_reference_line(r):
    import json
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["steps"] == 3 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    return d


def test_swap_row_plan_moves_each_swapped_block_out_and_back():
    from paged_kv_cache_379_b200 import workload as wlmod
    w = wlmod.make("gqa", seed=bench.rank_seed(0, "gqa"))
    tables, swapped, n_host, out_pairs, in_pairs = bench.swap_row_plan(w)
    # swap-out: the swapped sequences' blocks (distinct, none shared in this
    # batch), each to its own host block
    want = np.concatenate([tables[s][tables[s] >= 0] for s in swapped])
    assert sorted(out_pairs[:, 0].tolist()) == sorted(want.tolist())
    assert len(set(out_pairs[:, 1].tolist())) == out_pairs.shape[0] == n_host
    assert out_pairs[:, 1].min() >= 0 and out_pairs[:, 1].max() < n_host
    # swap-in: every host block back to a distinct GPU block of the pool
    assert sorted(in_pairs[:, 0].tolist()) == sorted(out_pairs[:, 1].tolist())
    assert len(set(in_pairs[:, 1].tolist())) == in_pairs.shape[0]
    assert in_pairs[:, 1].min() >= 0 and in_pairs[:, 1].max() < w.num_blocks


def test_prefix_row_reuses_the_full_blocks_of_every_later_sample():
    from oracle.pool import OraclePool
    from paged_kv_cache_379_b200.pool import BlockPool
    # 3 prompts of 100 tokens (6 full blocks of 16 + 1 partial), 4 samples each
    reqs = bench.prefix_row_prompts(5, prompts=3, samples=4, prompt_len=100)
    with BlockPool(64, 16) as pool:
        first = bench.prefix_step(pool, reqs, pool.free_table)
        again = bench.prefix_step(pool, reqs, pool.free_table)   # everything was freed: the same again
        assert pool.get_num_free_blocks() == 64
    op = OraclePool(64, 16)

    def ofree(t):
        for b in t:
            op.free(b)
    assert first == again == bench.prefix_step(op, reqs, ofree) == (3 * 4 * 7, 3 * 3 * 6 * 16)
