#!/usr/bin/env python
"""Benchmark of the paged-KV decode hot path on B200.

One step = slot mapping (new token's position -> cache slot) and cache write of
the new K/V (one fused launch) -> paged decode attention (one pass, or partition kernel + LSE
reduce, as the library chooses), over one batch of the GQA 70B-style layer
workload: 128 sequences, 64 query / 8 KV heads, head_dim 128, block_size 16,
lengths lognormal (median 1024, sigma 0.8) clipped to [16, 4096], shuffled
block pool 1.2x.  Inputs are seeded synthetic data already resident in HBM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload tiny|mha|gqa|long|shared|gqa-fp8|prefill|cow|swap|prefix]
                    [--partition P] [--l2-flush]

The default workload is the line above.  The other decode workloads run the
same step: `tiny` (4 sequences, block size 4), `mha` (64 sequences, 32/32
heads), `long` (8 sequences of 32K..128K positions; --partition 512 is the
workload's stated split), `shared` (256 sequences forked from 32 shared
1024-token prompts: the step starts with the copy-on-write block copies; its
roofline counts every shared block once).  --l2-flush empties L2 before every
step.  More rows of the path: `gqa-fp8` (the gqa batch with an FP8 E4M3
cache: slot mapping + quantising cache write -> decode over codes; KV GB/s of
1-byte elements), `prefill` (8 x 2048-token prompts with the gqa heads: slot
mapping -> cache write of the prompts' K/V -> causal paged prefill on the
tensor cores; useful TFLOP/s), `cow` (the shared step's block copies alone),
`swap` (a quarter of the gqa batch's blocks swapped out to pinned host memory
and back through the host pool's plans; GB/s over the host link against the
copy engines' rate for the same bytes) and `prefix` (host only: 32 prompts x
8 samples through the pool's prefix cache; prompts/s).

Prints ONE JSON line (rank 0).  `value` = KV GB/s: the decode's algorithmic
bytes per step (KV blocks touched + queries + block tables + outputs) over the
step time, summed over ranks / max over ranks.  The oracle (plain fp64 CPU
code) is timed on a bounded sample as `cpu_baseline`; `--impl reference`
times it as the reference arm.
"""

from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "paged-decode KV GB/s (% of B200 HBM peak) and seqs/s, GQA 64q/8kv d128 b128"
WORKLOAD = "gqa"
FALLBACK_HBM_GBS = 6650.0
SPEC_HBM_GBS = 8000.0
L2_BYTES = 126 * 1024 * 1024
PROFILE_SUMMARY = os.path.join(ROOT, "profiles", "paged_decode_gqa_ncu.md")
KERNEL_SOURCES = [os.path.join(ROOT, "paged_kv_cache_379_b200", "csrc", f)
                  for f in ("decode.cuh", "common.cuh", "pagedkv.cu", "cache_ops.cuh", "prefill.cuh", "tc05.cuh")]
PROFILE_FP8 = os.path.join(ROOT, "profiles", "paged_decode_fp8_gqa_ncu.md")
PROFILE_PREFILL = os.path.join(ROOT, "profiles", "paged_prefill_prompt2k_ncu.md")
PROFILE_SHARED = os.path.join(ROOT, "profiles", "paged_decode_shared_prefix_ncu.md")
PROFILE_LONG = os.path.join(ROOT, "profiles", "paged_decode_long_ncu.md")
METRIC_FP8 = "paged-decode KV GB/s, FP8 E4M3 KV cache (per-tensor scales), GQA 64q/8kv d128 b16"
METRIC_PREFILL = "paged-prefill useful TFLOP/s (causal), 8 x 2048-token prompts, GQA 64q/8kv d128 b16"
PREFILL_SHAPE = dict(num_seqs=8, prompt=2048, num_heads=64, num_kv_heads=8, head_dim=128, block_size=16)


DECODE_ROWS = ("tiny", "mha", "gqa", "long", "shared")
ROW_METRICS = {
    "tiny": "paged-decode KV GB/s and seqs/s, tiny 4 seqs 4q/4kv d64 bs4",
    "mha": "paged-decode KV GB/s (% of B200 HBM peak) and seqs/s, MHA 32q/32kv d128 b64",
    "gqa": METRIC,
    "long": "paged-decode KV GB/s (% of B200 HBM peak) and seqs/s, long-context 32q/8kv d128 b8 L 32K-128K, split-K",
    "shared": "shared-prefix CoW decode step: KV GB/s (unique and logical) and seqs/s, 256 seqs 32q/8kv d128",
}


def workload_description(w) -> str:
    heads = (f"{w.num_heads} query / {w.num_kv_heads} KV heads, head_dim {w.head_dim}, "
             f"block_size {w.block_size}")
    if w.name == "tiny":
        return (f"{w.num_seqs} seqs of lengths {{7, 16, 33, 50}}, {heads}, pool of {w.num_blocks} blocks, "
                "tables drawn without replacement")
    if w.name == "mha":
        return f"{w.num_seqs} seqs, {heads}, lengths uniform in [128, 2048], shuffled pool of {w.num_blocks} blocks (1.25x)"
    if w.name == "long":
        return (f"{w.num_seqs} seqs, {heads}, lengths uniform in [32768, 131072], shuffled pool of "
                f"{w.num_blocks} blocks (1.2x)")
    if w.name == "shared":
        return (f"{w.num_seqs} seqs = 32 prompts of 1024 tokens x 8 samples (prompt blocks shared), private tails "
                f"uniform in [1, 256], {heads}, shuffled pool of {w.num_blocks} blocks (1.2x); every sequence "
                "forked before the step, so its token's write copies the block it lands in")
    return (f"{w.num_seqs} seqs, {heads}, lengths lognormal(median 1024, sigma 0.8) clipped [16, 4096], "
            f"shuffled pool of {w.num_blocks} blocks (1.2x)")


def decode_config(w, world: int, l2_flush: bool) -> dict:
    """The workload's description: the same dict in both arms."""
    return {
        "workload": f"{w.name}: {workload_description(w)}",
        "num_seqs_per_gpu": w.num_seqs, "num_heads": w.num_heads, "num_kv_heads": w.num_kv_heads,
        "head_dim": w.head_dim, "block_size": w.block_size, "sum_seq_len": int(w.seq_lens.sum()),
        "max_seq_len": w.max_seq_len,
        "l2": "flushed before every step (2x L2 written outside the step's events)" if l2_flush else
              "no flush: each step reads more than L2 (126 MB)" if w.name in ("mha", "gqa", "long", "shared") else
              "no flush: the tiny working set stays in L2 across steps",
        "parallelism": f"dp{world}: independent batch per GPU, no collective on the data path",
    }


def unique_bytes(tables, seq_lens, block_size, num_heads, num_kv_heads, head_dim, kv_elem_bytes: int = 2) -> int:
    """algorithmic_bytes with every physical block counted once, however many
    sequences' tables point at it (what HBM must supply at least when
    sequences share blocks)."""
    lens = np.asarray(seq_lens, dtype=np.int64)
    blocks = -(-lens // block_size)
    ids = np.concatenate([np.asarray(tables[s, :blocks[s]]) for s in range(len(lens))]) if len(lens) else []
    kv = int(np.unique(ids).size) * block_size * num_kv_heads * head_dim * 2 * kv_elem_bytes
    qo = 2 * len(lens) * num_heads * head_dim * 2
    return kv + qo + int(blocks.sum()) * 4 + 4 * len(lens)


def algorithmic_bytes(seq_lens, block_size, num_heads, num_kv_heads, head_dim, kv_elem_bytes: int = 2) -> int:
    """KV blocks touched (K and V) + queries + outputs + block-table entries read + seq_lens.

    kv_elem_bytes: 2 for a bf16 cache, 1 for an FP8 (E4M3) cache."""
    blocks = -(-np.asarray(seq_lens, dtype=np.int64) // block_size)
    kv = int(blocks.sum()) * block_size * num_kv_heads * head_dim * 2 * kv_elem_bytes
    qo = 2 * len(seq_lens) * num_heads * head_dim * 2
    tables = int(blocks.sum()) * 4 + 4 * len(seq_lens)
    return kv + qo + tables


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def _code_only(text: str) -> str:
    """C/C++ source with comments and blank-space runs removed: what the compiler
    sees, so that a comment edit does not invalidate recorded counters."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def kernel_source_hash() -> str:
    """Hash of the kernel sources' code (comments and layout ignored)."""
    h = hashlib.sha256()
    for p in KERNEL_SOURCES:
        with open(p, encoding="utf-8") as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def profiled_traffic(path=PROFILE_SUMMARY, key="dram_bytes_per_decode_call"):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel sources (else None)."""
    try:
        text = open(path).read()
    except OSError:
        return None
    m_hash = re.search(r"kernel_source_sha256_16\s*=\s*([0-9a-f]+)", text)
    m_bytes = re.search(key + r"\s*=\s*([0-9]+)", text)
    if not m_hash or not m_bytes or m_hash.group(1) != kernel_source_hash():
        return None
    return int(m_bytes.group(1))


def measured_tensor_peak():
    """Sustained dense bf16 TFLOP/s (a kernel timed inside a long loop)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["bf16_tflops_sustained"]), "measured (MEASURED_PEAKS.json bf16_tflops_sustained)"
    except Exception:
        return 1400.0, "fallback (sustained bf16 figure of the profiling recipe)"


# ------------------------------------------------------------------ clocks

REASON_BITS = {
    0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
    0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
    0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
}
BAD_REASONS = {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"}


class ClockSampler:
    """Samples the SM clock and the clock-event reasons through NVML (the data
    nvidia-smi reports) every 5 ms on a background thread, and on request
    from the timing thread (sample_now)."""

    def __init__(self, cuda_index: int):
        import torch
        self.samples = []
        self.ok = False
        self.max_mhz = None
        try:
            import pynvml as nv
            nv.nvmlInit()
            handle = None
            try:
                props = torch.cuda.get_device_properties(cuda_index)
                bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
                handle = nv.nvmlDeviceGetHandleByPciBusId(bus)
            except Exception:
                handle = nv.nvmlDeviceGetHandleByIndex(cuda_index)
            self.nv, self.h = nv, handle
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(handle, nv.NVML_CLOCK_SM))
            self.ok = True
        except Exception as e:  # pragma: no cover - depends on the box
            self.err = repr(e)
        self._stop = threading.Event()
        self._t = None

    def _reasons(self):
        nv = self.nv
        for fn in ("nvmlDeviceGetCurrentClocksEventReasons", "nvmlDeviceGetCurrentClocksThrottleReasons"):
            if hasattr(nv, fn):
                return int(getattr(nv, fn)(self.h))
        return 0

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append((time.perf_counter(), float(self.nv.nvmlDeviceGetClockInfo(
                    self.h, self.nv.NVML_CLOCK_SM)), self._reasons()))
            except Exception:
                pass
            time.sleep(0.005)

    def sample_now(self):
        """One sample from the calling thread: taken inside the timed region
        right after the steps are enqueued, while the GPU still runs them, so
        that a timed region shorter than the background period has samples."""
        if self.ok:
            try:
                self.samples.append((time.perf_counter(), float(self.nv.nvmlDeviceGetClockInfo(
                    self.h, self.nv.NVML_CLOCK_SM)), self._reasons()))
            except Exception:
                pass

    def start(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()

    def stop(self):
        if self._t:
            self._stop.set()
            self._t.join()

    def window(self, t0: float, t1: float) -> dict:
        s = [x for x in self.samples if t0 <= x[0] <= t1]
        if not s:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0,
                    "note": "no NVML samples in the timed window" if self.ok else getattr(self, "err", "")}
        bits = 0
        for x in s:
            bits |= x[2]
        reasons = sorted(name for b, name in REASON_BITS.items() if bits & b and name != "gpu_idle")
        return {"sm_mhz": statistics.median(x[1] for x in s), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(s)}


# ------------------------------------------------------------------ our arm

def aggregate_over_ranks(total_ms, e2e_ms, step_bytes, num_seqs, device, dist=None):
    """Whole-job figures: times are the max over ranks, work is summed over ranks."""
    import torch
    res = torch.tensor([float(total_ms), float(e2e_ms)], dtype=torch.float64, device=device)
    tot = torch.tensor([float(step_bytes), float(num_seqs)], dtype=torch.float64, device=device)
    if dist is not None:
        dist.all_reduce(res, op=dist.ReduceOp.MAX)
        dist.all_reduce(tot, op=dist.ReduceOp.SUM)
    t, e = res.tolist()
    b, n = tot.tolist()
    return t, e, b, n


def rank_seed(rank: int, name: str = WORKLOAD) -> int:
    """Each rank decodes its own independent batch of the same shape (weak scaling)."""
    from paged_kv_cache_379_b200 import workload as wlmod
    return wlmod.SEED_BASE + wlmod.NAMES.index(name) + 1000 * rank


def run_decode(args, rank: int, world: int, local_rank: int) -> dict | None:
    """One decode row: tiny, mha, gqa (the default line), long or shared.

    Step = [copy-on-write block copies (shared)] -> slot mapping + cache write
    of each sequence's new token (one launch) -> decode (the library's plan, or
    the split form at --partition).  Device events around every stage of every
    timed step; the whole K-step window between barriers gives the step time
    (with --l2-flush: the sum of the per-step event intervals, the flush
    writes sitting between them)."""
    import torch

    from paged_kv_cache_379_b200 import ops
    from paged_kv_cache_379_b200 import workload as wlmod
    from paged_kv_cache_379_b200.step import DecodeBatch, host_step

    name = args.workload
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    dist = None
    if world > 1:
        import torch.distributed as dist
    w = wlmod.make(name, seed=rank_seed(rank, name), num_seqs=args.num_seqs or None)
    tables, pairs_h, cow_h = w.block_tables, None, None
    if name == "shared":
        # the host pool's step: every sequence forked, so each token's write into
        # an existing block takes a copy (the pool's (src, dst) pairs); fused, the
        # copies run in the cache write's launch from per-sequence sources
        _, tables, _, slots_h, pairs_h = host_step(w, fork_all=True)
        if not args.unfused_cow:
            cow_h = ops.cow_sources(slots_h, w.block_size, pairs_h)
    batch = DecodeBatch(w, dev, tables=tables, pairs=pairs_h, workspace=False, cow_src=cow_h)
    stream = torch.cuda.current_stream(dev)
    part = int(args.partition)
    groups = None
    if name == "shared" and not args.no_groups:
        # the shared prompts are read once per group of sequences (pa_decode_shared),
        # the host pool's groups at the prompt's length unless --partition says otherwise
        part = part or 1024
        gs_h, gp_h = ops.prefix_groups(tables, w.seq_lens, w.block_size, part)
        groups = (torch.from_numpy(gs_h).to(dev), torch.from_numpy(gp_h).to(dev))
    if part:
        ws = ops.new_workspace(w.num_seqs, w.num_heads, w.num_kv_heads, w.head_dim, w.max_seq_len, part,
                               device=dev)
        plan = part
    else:
        ws = ops.new_workspace(w.num_seqs, w.num_heads, w.num_kv_heads, w.head_dim, w.max_seq_len, device=dev)
        plan = ops.decode_plan(w.num_seqs, w.num_heads, w.num_kv_heads, w.head_dim, w.max_seq_len, ws.numel())
    n_pairs = 0 if batch.pairs is None else int(batch.pairs.shape[0])
    fused = batch.cow_src is not None
    launches_per_step = (1 if n_pairs and not fused else 0) + 1 + (2 if plan else 1)
    step_bytes = algorithmic_bytes(w.seq_lens, w.block_size, w.num_heads, w.num_kv_heads, w.head_dim)
    uniq = unique_bytes(tables, w.seq_lens, w.block_size, w.num_heads, w.num_kv_heads, w.head_dim)
    roof_bytes = uniq if name == "shared" else step_bytes
    blk_bytes = w.block_size * w.num_kv_heads * w.head_dim * 2
    copy_bytes = n_pairs * blk_bytes * 2 * 2     # K and V blocks, each read and written

    def device_step(S, ev=None):
        """One step on input set S (tensors on the device); ev: per-stage events."""
        if ev is not None:
            ev[0].record(stream)
        if S["pairs"] is not None and S["cow"] is None:
            ops.copy_blocks(batch.key_cache, batch.value_cache, S["pairs"], stream=stream)
        if ev is not None:
            ev[1].record(stream)
        if S["cow"] is not None:
            ops.append_decode_kv_cow(S["k"], S["v"], batch.key_cache, batch.value_cache, S["bt"], S["sl"],
                                     S["cow"], slot_mapping=S["slots"], stream=stream)
        else:
            ops.append_decode_kv(S["k"], S["v"], batch.key_cache, batch.value_cache, S["bt"], S["sl"],
                                 slot_mapping=S["slots"], stream=stream)
        if ev is not None:
            ev[2].record(stream)
        if groups is not None:
            ops.decode_shared(S["q"], batch.key_cache, batch.value_cache, S["bt"], S["sl"], w.scale,
                              batch.max_seq_len, part, S["gs"], S["gp"], ws, out=S["out"], stream=stream)
        elif part:
            ops.decode_split(S["q"], batch.key_cache, batch.value_cache, S["bt"], S["sl"], w.scale,
                             batch.max_seq_len, part, ws, out=S["out"], stream=stream)
        else:
            ops.decode(S["q"], batch.key_cache, batch.value_cache, S["bt"], S["sl"], w.scale, batch.max_seq_len,
                       out=S["out"], workspace=ws, stream=stream)
        if ev is not None:
            ev[3].record(stream)

    resident = dict(q=batch.query, k=batch.new_key, v=batch.new_value, bt=batch.block_tables, sl=batch.seq_lens,
                    pairs=batch.pairs, cow=batch.cow_src, slots=batch.slots, out=batch.out,
                    gs=None if groups is None else groups[0], gp=None if groups is None else groups[1])
    K, W = args.steps, args.warmup
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)]
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev) if args.l2_flush else None

    def step(i, events=False):
        if flush is not None:
            flush.fill_((0 if i is None else i) & 255)   # evicts the previous step's lines from L2
        device_step(resident, evs[i] if (events and i is not None) else None)

    sampler = ClockSampler(local_rank)
    sampler.start()
    # The timed window runs the steps' kernels back to back, as a serving loop
    # does (each kernel may start under the end of the one before it); a
    # second pass of the same K steps with events between the kernels gives
    # each stage's own duration (the roofline's kernel time) -- and, with the
    # L2 flushed between steps, the step time as the sum of the event
    # intervals, which leaves the flush writes out.
    total_ms, clocks, remeasured = _timed_loop(step, K, W, stream, dev, dist, sampler)
    torch.cuda.synchronize(dev)
    for i in range(K):
        step(i, events=True)
    torch.cuda.synchronize(dev)
    stage = np.array([[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(3)] for i in range(K)])
    copy_ms, append_ms, dec_ms = (float(x) for x in stage.mean(axis=0))
    if flush is not None:
        total_ms = float(stage.sum())

    # e2e: the same step through the C ABI with host buffers.  Every step's
    # inputs (query, new K/V, block tables, lengths, copy pairs) come from pinned
    # host memory and its output goes back to pinned host memory inside the timed
    # region.  As a serving loop would, the inputs sit in one pinned staging
    # buffer (16-byte aligned sections, one copy per step), and the copies run on
    # their own streams over three buffer sets: while step i computes, step i-1's
    # output comes back and step i+1's inputs go up (with two sets, a step's
    # upload waits for the download two steps back, so both copies sit on a
    # two-step cycle with one compute: ~104 us per 97 us step on the GQA
    # batch).  The KV cache stays resident.
    e2e = None
    if not args.no_e2e:
        parts = [("q", w.query.view(np.int16), torch.bfloat16, batch.query.shape),
                 ("k", w.new_key.view(np.int16), torch.bfloat16, batch.new_key.shape),
                 ("v", w.new_value.view(np.int16), torch.bfloat16, batch.new_value.shape),
                 ("bt", np.ascontiguousarray(tables, np.int32), torch.int32, batch.block_tables.shape),
                 ("sl", w.seq_lens.astype(np.int32), torch.int32, batch.seq_lens.shape)]
        if fused:
            parts.append(("cow", np.ascontiguousarray(cow_h, np.int32), torch.int32, batch.cow_src.shape))
        if groups is not None:
            parts.append(("gs", gs_h, torch.int32, groups[0].shape))
            parts.append(("gp", gp_h, torch.int32, groups[1].shape))
        elif n_pairs:
            parts.append(("pairs", np.ascontiguousarray(pairs_h, np.int64), torch.int64, batch.pairs.shape))
        offs, nbytes_in = {}, 0
        for pname, a, _, _ in parts:
            offs[pname] = (nbytes_in, a.nbytes)
            nbytes_in += -(-a.nbytes // 16) * 16
        h_in = torch.zeros(nbytes_in, dtype=torch.uint8).pin_memory()
        h_np = h_in.numpy()
        for pname, a, _, _ in parts:
            o, n = offs[pname]
            h_np[o:o + n] = np.frombuffer(np.ascontiguousarray(a).tobytes(), np.uint8)
        NB = 3   # buffer sets in flight
        h_out = [torch.empty(batch.out.shape, dtype=torch.int16).pin_memory() for _ in range(NB)]
        h2d = nbytes_in
        d2h = h_out[0].numel() * h_out[0].element_size()

        def input_set():
            buf = torch.empty(nbytes_in, dtype=torch.uint8, device=dev)
            S = {pname: buf[offs[pname][0]:offs[pname][0] + offs[pname][1]].view(dt).view(shape)
                 for pname, _, dt, shape in parts}
            S.setdefault("pairs", None)
            S.setdefault("cow", None)
            S.setdefault("gs", None)
            S.setdefault("gp", None)
            S.update(buf=buf, slots=torch.empty_like(batch.slots), out=torch.empty_like(batch.out))
            return S
        sets = [input_set() for _ in range(NB)]
        up = torch.cuda.Stream(dev)
        down = torch.cuda.Stream(dev)
        ev_in = [torch.cuda.Event() for _ in range(NB)]
        ev_done = [torch.cuda.Event() for _ in range(NB)]
        ev_free = [torch.cuda.Event() for _ in range(NB)]

        def e2e_step(i):
            b = i % NB
            S = sets[b]
            up.wait_event(ev_free[b])            # this buffer set's previous output is back on the host
            with torch.cuda.stream(up):
                S["buf"].copy_(h_in, non_blocking=True)
                ev_in[b].record(up)
            stream.wait_event(ev_in[b])
            device_step(S)
            ev_done[b].record(stream)
            down.wait_event(ev_done[b])
            with torch.cuda.stream(down):
                h_out[b].copy_(S["out"].view(torch.int16), non_blocking=True)
                ev_free[b].record(down)

        def barrier():
            torch.cuda.synchronize(dev)
            if dist is not None:
                dist.barrier()
            torch.cuda.synchronize(dev)

        for i in range(W):
            e2e_step(i)
        barrier()
        f0 = torch.cuda.Event(enable_timing=True)
        f1 = torch.cuda.Event(enable_timing=True)
        f0.record(up)
        for i in range(K):
            e2e_step(i)
        down.wait_event(ev_free[(K - 1) % NB])
        f1.record(down)
        barrier()
        e2e = {"ms": f0.elapsed_time(f1), "h2d": h2d, "d2h": d2h}
    sampler.stop()

    total_ms, e2e_max_ms, all_bytes, all_seqs = aggregate_over_ranks(
        total_ms, e2e["ms"] if e2e else 0.0, step_bytes, w.num_seqs, dev, dist)
    if rank != 0:
        return None

    ms_per_step = total_ms / K
    gbs = all_bytes * K / (total_ms * 1e-3) / 1e9
    achieved = roof_bytes / (dec_ms * 1e-3) / 1e9
    peak, peak_src = measured_peak()
    # DRAM bytes per decode call from the committed ncu captures, for the
    # configurations they were taken on (whole batch, no L2 flush)
    traffic = None
    if not args.num_seqs and not args.l2_flush:
        if name == "gqa" and not part:
            traffic = profiled_traffic()
        elif name == "shared" and groups is not None and part == 1024:
            traffic = profiled_traffic(PROFILE_SHARED)
        elif name == "long" and not int(args.partition):
            traffic = profiled_traffic(PROFILE_LONG)
    path = f"split, partition {plan} (partition kernel + LSE reduce)" if plan else "one pass"
    if groups is not None:
        path = (f"shared-prefix groups ({len(gp_h)} groups; the shared {int(gp_h.max())} x {part}-token "
                f"partitions computed once per KV head for 16 / G sequences at a time) + split, partition {part}")
    if fused:
        step_desc = "append_decode_kv_cow (copy-on-write copies + slot mapping + cache write, one launch) -> decode"
    else:
        step_desc = ("copy_blocks (CoW pairs) -> " if n_pairs else "") + \
            "append_decode_kv (slot mapping + cache write, one launch) -> decode"
    line = {
        "metric": ROW_METRICS[name] + (f" {part}" if name == "long" and part else ""),
        "value": round(gbs, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": K,
        "warmup": W,
        "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16 values, the workload's lengths, shuffled block pool)",
        "config": decode_config(w, world, bool(args.l2_flush)),
        "reduced_batch": (f"first {w.num_seqs} sequences only (--num-seqs): a profiling case, not the workload"
                          if args.num_seqs else None),
        "decode_path": path + ("" if groups is not None else
                               " (forced by --partition)" if args.partition else " (the library's plan)"),
        "step": step_desc,
        "algorithmic_bytes_per_step": step_bytes,
        "seqs_per_s": round(all_seqs * K / (total_ms * 1e-3), 1),
        "frac_of_spec_hbm": round(gbs / world / SPEC_HBM_GBS, 4),
        "stage_ms_note": "each stage's own duration: a second pass of the K steps with events between the kernels",
        "stage_ms": ({"append_decode_kv_cow": round(append_ms, 5), "decode": round(dec_ms, 5)} if fused else
                     {"copy_blocks": round(copy_ms, 5) if n_pairs else None, "append_decode_kv": round(append_ms, 5),
                      "decode": round(dec_ms, 5)}),
        "clocks": clocks,
        "gpu_launches": launches_per_step * K,
        "roofline": {
            "bound": "hbm",
            "kernel": ("pa_decode_shared (partition kernel with shared-prefix items + LSE reduce)" if groups is not None
                       else "pa_decode (partition kernel + LSE reduce)" if plan else "pa_decode (one-pass kernel)"),
            "achieved": round(achieved, 2),
            "peak": peak,
            "unit": "GB/s",
            "frac": round(achieved / peak, 4),
            "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)" if peak_src == "measured" else peak_src,
            "traffic": traffic,
            "algorithmic_bytes": roof_bytes,
            "avg_launch_ms": round(dec_ms, 5),
        },
    }
    if name == "shared":
        line["roofline"]["bytes_basis"] = ("unique physical bytes: every shared block counted once "
                                           f"({uniq} of {step_bytes} logical bytes)")
        line["logical_kv_gbs_decode"] = round(step_bytes / (dec_ms * 1e-3) / 1e9, 2)
        line["unique_gbs_step"] = round(uniq * world * K / (total_ms * 1e-3) / 1e9, 2)
        cow_ms = append_ms if fused else copy_ms      # fused: the copies and the 256-row cache write
        line["copy_on_write"] = {"pairs": n_pairs, "bytes_read_and_written": copy_bytes,
                                 "fused_with_cache_write": fused,
                                 "ms": round(cow_ms, 5),
                                 "gbs": round(copy_bytes / (cow_ms * 1e-3) / 1e9, 2) if cow_ms > 0 else None,
                                 "share_of_step": round(cow_ms / (copy_ms + append_ms + dec_ms), 4),
                                 # back to back the copies overlap the decode's start: what they
                                 # add to the step is the step minus the decode's own duration
                                 "exposed_ms_back_to_back": round(max(0.0, total_ms / K - dec_ms), 5),
                                 "exposed_share_back_to_back": round(max(0.0, total_ms / K - dec_ms) / (total_ms / K), 4),
                                 "note": ("share_of_step: the copy launch's own duration (events between the "
                                          "kernels) over the sum of the stages; exposed_*: the whole step back "
                                          "to back minus the decode's own duration")}
    if remeasured:
        line["clocks_note"] = "first timed region saw a thermal/hw slowdown reason; re-measured once"
    if e2e:
        line["e2e"] = {"value": round(all_bytes * K / (e2e_max_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
                       "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
                       "ms_per_step": round(e2e_max_ms / K, 5),
                       "how": "pa_* C-ABI calls on pinned host inputs; host-to-device and device-to-host copies "
                              "on their own streams, three buffer sets in flight" +
                              ("; no L2 flush between these steps" if flush is not None else "")}
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, tables, budget_s=args.cpu_budget)
    return line


# ------------------------------------------------------- the other path rows

def _timed_loop(step, K, W, stream, dev, dist, sampler):
    """W untimed steps, then K timed steps between barriers; step(i) gets the
    step index (or None in warm-up).  Returns (total_ms, clocks, remeasured)."""
    import torch

    def barrier():
        torch.cuda.synchronize(dev)
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize(dev)

    for _ in range(W):
        step(None)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)

    def region():
        barrier()
        t0 = time.perf_counter()
        e0.record(stream)
        for i in range(K):
            step(i)
        e1.record(stream)
        sampler.sample_now()           # all steps enqueued; the GPU is still running them
        barrier()
        return t0, time.perf_counter()

    t0, t1 = region()
    clocks = sampler.window(t0, t1)
    remeasured = False
    if set(clocks["reasons"]) & BAD_REASONS:
        first = clocks
        t0, t1 = region()
        clocks = sampler.window(t0, t1)
        clocks["first_attempt"] = first
        remeasured = True
    return e0.elapsed_time(e1), clocks, remeasured


def prefill_flops(seq_lens, q_lens, num_heads, head_dim) -> int:
    """Useful FLOPs of a causal prefill: 4 * D * Hq per (query row, visible key)."""
    total = 0
    for L, n in zip(seq_lens, q_lens):
        L, n = int(L), int(n)
        ctx = L - n
        total += n * ctx + n * (n + 1) // 2
    return 4 * head_dim * num_heads * total


def make_prefill_case(seed):
    """8 prompts of 2048 tokens (chunk = whole prompt), 64/8 heads, d128, bs16,
    tables drawn from a shuffled pool of 1.2x the blocks needed."""
    from paged_kv_cache_379_b200 import workload as wlmod
    sh = PREFILL_SHAPE
    B, P, bs = sh["num_seqs"], sh["prompt"], sh["block_size"]
    lens = [P] * B
    w = wlmod.random_decode_case(seed, num_seqs=B, num_heads=sh["num_heads"], num_kv_heads=sh["num_kv_heads"],
                                 head_dim=sh["head_dim"], block_size=bs, lengths=lens,
                                 spare_blocks=int(0.2 * B * P / bs))
    rng = np.random.Generator(np.random.PCG64(seed + 1))
    T = B * P
    query = wlmod.bf16_normal(rng, (T, sh["num_heads"], sh["head_dim"]))
    new_k = wlmod.bf16_normal(rng, (T, sh["num_kv_heads"], sh["head_dim"]))
    new_v = wlmod.bf16_normal(rng, (T, sh["num_kv_heads"], sh["head_dim"]))
    return w, lens, query, new_k, new_v


def run_row(args, rank: int, world: int, local_rank: int) -> dict | None:
    """gqa-fp8 or prefill, timed like the main line (device events, max over ranks)."""
    import torch

    from paged_kv_cache_379_b200 import ops
    from paged_kv_cache_379_b200 import workload as wlmod
    from paged_kv_cache_379_b200.step import bf16_to_device

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    dist = None
    if world > 1:
        import torch.distributed as dist
    stream = torch.cuda.current_stream(dev)
    K, W = args.steps, args.warmup
    ev0 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ev1 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    i32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(dev)  # noqa: E731

    if args.workload == "gqa-fp8":
        w = wlmod.make("gqa", seed=rank_seed(rank), fill_cache=False)
        rng = np.random.Generator(np.random.PCG64(rank_seed(rank) + 17))
        kc_h = wlmod.fp8_cache(rng, w.num_blocks, w.block_size, w.num_kv_heads, w.head_dim, w.free_blocks)
        vc_h = wlmod.fp8_cache(rng, w.num_blocks, w.block_size, w.num_kv_heads, w.head_dim, w.free_blocks)
        kc, vc = torch.from_numpy(kc_h).to(dev), torch.from_numpy(vc_h).to(dev)
        ks, vs = 0.25, 0.25
        q, nk, nv = (bf16_to_device(a, dev) for a in (w.query, w.new_key, w.new_value))
        bt, sl = i32(w.block_tables), i32(w.seq_lens)
        slots = torch.empty(w.num_seqs, dtype=torch.int64, device=dev)
        out = torch.empty_like(q)
        ws = ops.new_workspace(w.num_seqs, w.num_heads, w.num_kv_heads, w.head_dim, w.max_seq_len, device=dev)
        plan = ops.decode_plan(w.num_seqs, w.num_heads, w.num_kv_heads, w.head_dim, w.max_seq_len, ws.numel())
        units = algorithmic_bytes(w.seq_lens, w.block_size, w.num_heads, w.num_kv_heads, w.head_dim, 1)
        launches = 1 + (2 if plan else 1)

        def step(i):
            ops.append_decode_kv_fp8(nk, nv, kc, vc, bt, sl, ks, vs, slot_mapping=slots, stream=stream)
            if i is not None:
                ev0[i].record(stream)
            ops.decode_fp8(q, kc, vc, bt, sl, w.scale, ks, vs, w.max_seq_len, out=out, workspace=ws,
                           stream=stream)
            if i is not None:
                ev1[i].record(stream)
    else:
        w, lens, qh, nkh, nvh = make_prefill_case(rank_seed(rank))
        B, T = w.num_seqs, qh.shape[0]
        kc, vc = bf16_to_device(w.key_cache, dev), bf16_to_device(w.value_cache, dev)
        q, nk, nv = (bf16_to_device(a, dev) for a in (qh, nkh, nvh))
        bt, sl = i32(w.block_tables), i32(lens)
        start = np.zeros(B + 1, np.int32)
        start[1:] = np.cumsum(lens)
        qs = i32(start)
        seq_ids = i32(np.repeat(np.arange(B), lens))
        positions = torch.from_numpy(np.concatenate([np.arange(L) for L in lens]).astype(np.int64)).to(dev)
        slots = torch.empty(T, dtype=torch.int64, device=dev)
        out = torch.empty_like(q)
        units = prefill_flops(lens, lens, w.num_heads, w.head_dim)
        launches = 3

        def step(i):
            ops.slot_mapping(bt, w.block_size, positions=positions, seq_ids=seq_ids, out=slots, stream=stream)
            ops.reshape_and_cache(nk, nv, kc, vc, slots, stream=stream)
            if i is not None:
                ev0[i].record(stream)
            ops.prefill(q, kc, vc, bt, sl, qs, w.scale, out=out, stream=stream)
            if i is not None:
                ev1[i].record(stream)

    sampler = ClockSampler(local_rank)
    sampler.start()
    total_ms, clocks, remeasured = _timed_loop(step, K, W, stream, dev, dist, sampler)
    sampler.stop()
    kern_ms = float(np.mean([ev0[i].elapsed_time(ev1[i]) for i in range(K)]))
    total_ms, _, all_units, all_seqs = aggregate_over_ranks(total_ms, 0.0, units, w.num_seqs, dev, dist)
    if rank != 0:
        return None
    fp8 = args.workload == "gqa-fp8"
    value = all_units * K / (total_ms * 1e-3) / (1e9 if fp8 else 1e12)
    achieved = units / (kern_ms * 1e-3) / (1e9 if fp8 else 1e12)
    if fp8:
        peak, peak_src = measured_peak()
        peak_src = f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)" if peak_src == "measured" else peak_src
        traffic = profiled_traffic(PROFILE_FP8)
    else:
        peak, peak_src = measured_tensor_peak()
        traffic = profiled_traffic(PROFILE_PREFILL, "dram_bytes_per_prefill_call")
    line = {
        "metric": METRIC_FP8 if fp8 else METRIC_PREFILL,
        "value": round(value, 2),
        "unit": "GB/s" if fp8 else "TFLOP/s",
        "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": round(total_ms / K, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3 KV, bf16 q/out, fp16 MMA" if fp8 else "bf16",
        "data": "synthetic (seeded)",
        "config": ({"workload": f"gqa-fp8: {workload_description(w)}; E4M3 codes, k_scale = v_scale = 0.25",
                    "decode_path": f"split, partition {plan}" if plan else "one pass",
                    "step": "append_decode_kv_fp8 (slot mapping + quantising cache write) -> decode_fp8",
                    "algorithmic_bytes_per_step": units,
                    "l2": f"inputs larger than L2 ({units / 1e9:.2f} GB read per step); no flush"}
                   if fp8 else
                   {"workload": "prefill: 8 prompts x 2048 tokens (whole-prompt chunks), 64 query / 8 KV heads, "
                                "head_dim 128, block_size 16, shuffled pool 1.2x",
                    "step": "slot_mapping (16384 tokens) -> reshape_and_cache -> prefill",
                    "useful_flops_per_step": units,
                    "l2": "compute bound; K/V (67 MB) re-read from L2 by every query tile; no flush"}),
        "clocks": clocks,
        "gpu_launches": launches * K,
        "roofline": {"bound": "hbm" if fp8 else "tensor",
                     "kernel": "pa_decode_fp8" if fp8 else "pa_prefill (paged_prefill_kernel)",
                     "achieved": round(achieved, 2), "peak": peak, "unit": "GB/s" if fp8 else "TFLOP/s",
                     "frac": round(achieved / peak, 4), "peak_source": peak_src, "traffic": traffic,
                     "avg_launch_ms": round(kern_ms, 5)},
        "e2e": None,
        "e2e_note": "end-to-end host-buffer timing is measured on the default workload only",
    }
    if remeasured:
        line["clocks_note"] = "first timed region saw a thermal/hw slowdown reason; re-measured once"
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = (cpu_baseline_fp8(w, kc_h, vc_h, ks, vs, args.cpu_budget) if fp8 else
                                cpu_baseline_prefill(w, qh, args.cpu_budget))
    return line


def run_cow(args, rank: int, world: int, local_rank: int) -> dict | None:
    """The copy-on-write block copies of the shared-prefix step (256 sequences
    forked from 32 prompts, each writing into a shared block), L2 flushed
    before every launch; per-launch device time by events (max over ranks)."""
    import torch

    from paged_kv_cache_379_b200 import ops
    from paged_kv_cache_379_b200 import workload as wlmod
    from paged_kv_cache_379_b200.step import DecodeBatch, host_step

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    dist = None
    if world > 1:
        import torch.distributed as dist
    stream = torch.cuda.current_stream(dev)
    K, W = args.steps, args.warmup
    w = wlmod.make("shared", seed=wlmod.SEED_BASE + wlmod.NAMES.index("shared") + 1000 * rank)
    _, tables, _, _, pairs = host_step(w, fork_all=True)
    batch = DecodeBatch(w, dev, tables=tables, pairs=pairs)
    n_pairs = int(pairs.shape[0])
    blk_bytes = w.block_size * w.num_kv_heads * w.head_dim * 2
    units = n_pairs * blk_bytes * 2 * 2  # K and V blocks, each read and written
    flush = torch.empty(L2_BYTES * 2, dtype=torch.uint8, device=dev)
    ev0 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ev1 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]

    def step(i):
        flush.fill_((i or 0) & 255)  # evicts the copies' blocks from L2
        if i is not None:
            ev0[i].record(stream)
        ops.copy_blocks(batch.key_cache, batch.value_cache, batch.pairs, stream=stream)
        if i is not None:
            ev1[i].record(stream)

    sampler = ClockSampler(local_rank)
    sampler.start()
    total_ms, clocks, remeasured = _timed_loop(step, K, W, stream, dev, dist, sampler)
    sampler.stop()
    kern_ms = float(np.mean([ev0[i].elapsed_time(ev1[i]) for i in range(K)]))
    if dist is not None:
        t = torch.tensor([kern_ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        kern_ms = float(t.item())
    if rank != 0:
        return None
    achieved = units / (kern_ms * 1e-3) / 1e9
    peak, peak_src = measured_peak()
    line = {
        "metric": "copy-on-write block copy GB/s (read + written), shared-prefix step",
        "value": round(achieved * world, 2), "unit": "GB/s", "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": round(kern_ms, 5), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16 (bit copy)", "data": "synthetic (seeded)",
        "config": {"workload": f"shared: {w.num_seqs} sequences forked from 32 prompts of 1024 tokens, "
                               f"{n_pairs} (src, dst) block pairs of {blk_bytes} bytes per cache",
                   "step": "copy_blocks of the step's pairs (K and V caches)",
                   "l2": f"flushed before every launch ({2 * L2_BYTES >> 20} MiB written, outside the events)",
                   "value_from": "per-launch device time (events around the copy only)"},
        "clocks": clocks,
        "gpu_launches": K,
        "roofline": {"bound": "hbm", "kernel": "pa_copy_blocks (copy_blocks_kernel)", "achieved": round(achieved, 2),
                     "peak": peak, "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "peak_source": peak_src, "traffic": None, "avg_launch_ms": round(kern_ms, 5)},
        "e2e": None,
        "e2e_note": "end-to-end host-buffer timing is measured on the default workload only",
    }
    if remeasured:
        line["clocks_note"] = "first timed region saw a thermal/hw slowdown reason; re-measured once"
    return line


def swap_row_plan(w):
    """The swap row's host work: the pool adopts the batch's step tables, every
    4th sequence is swapped out to a host pool sized for exactly those blocks,
    then all of them back in.  Returns (tables, swapped sequences, host blocks,
    swap-out pairs, swap-in pairs), the pairs int64 [P, 2]."""
    from paged_kv_cache_379_b200.pool import BlockPool, swap_plan
    from paged_kv_cache_379_b200.step import host_step

    gpu_pool, tables, nblk, _, _ = host_step(w)
    swapped = np.arange(0, w.num_seqs, 4)                  # a quarter of the batch
    n_host = int(nblk[swapped].sum())
    with BlockPool(n_host, w.block_size) as host_pool:
        outs, ins, host_tables = [], [], []
        for s in swapped:
            host_table, po = swap_plan(gpu_pool, host_pool, tables[s, :nblk[s]])
            host_tables.append(host_table)
            outs.append(po)
        for host_table in host_tables:
            _, pi = swap_plan(host_pool, gpu_pool, host_table)
            ins.append(pi)
    gpu_pool.close()
    return tables, swapped, n_host, np.concatenate(outs).astype(np.int64), np.concatenate(ins).astype(np.int64)


def run_swap(args, rank: int, world: int, local_rank: int) -> dict | None:
    """Preemption by swapping (the CPU-GPU block allocator of [深度解析
    «BlockAllocator 源码核心»]): the blocks of a quarter of the GQA batch's
    sequences move to a pinned host cache through the host pool's swap plan
    (pa_pool_swap_plan) and back into the GPU pool (pa_swap_blocks both ways).
    A step is the swap-out plus the swap-in; device time by events around each
    launch.  The denominator is measured in the same run: the copy engines'
    rate (cudaMemcpyAsync between a device buffer and pinned host memory) for
    the same bytes, each direction."""
    import torch

    from paged_kv_cache_379_b200 import ops
    from paged_kv_cache_379_b200 import workload as wlmod
    from paged_kv_cache_379_b200.step import DecodeBatch

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    dist = None
    if world > 1:
        import torch.distributed as dist
    stream = torch.cuda.current_stream(dev)
    K, W = args.steps, args.warmup
    w = wlmod.make("gqa", seed=rank_seed(rank, "gqa"))
    tables, swapped, n_host, out_pairs, in_pairs = swap_row_plan(w)
    batch = DecodeBatch(w, dev, tables=tables)
    shape = (n_host,) + tuple(batch.key_cache.shape[1:])
    host_k = torch.zeros(shape, dtype=torch.bfloat16).pin_memory()
    host_v = torch.zeros(shape, dtype=torch.bfloat16).pin_memory()
    d_out = torch.from_numpy(out_pairs).to(dev)
    d_in = torch.from_numpy(in_pairs).to(dev)
    blk_bytes = w.block_size * w.num_kv_heads * w.head_dim * 2
    bytes_out = int(out_pairs.shape[0]) * blk_bytes * 2     # K and V blocks over the link, GPU -> host
    bytes_in = int(in_pairs.shape[0]) * blk_bytes * 2       # and back
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]

    def step(i):
        if i is not None:
            ev[i][0].record(stream)
        ops.swap_blocks(host_k, host_v, batch.key_cache, batch.value_cache, d_out, stream=stream)
        if i is not None:
            ev[i][1].record(stream)
        ops.swap_blocks(batch.key_cache, batch.value_cache, host_k, host_v, d_in, stream=stream)
        if i is not None:
            ev[i][2].record(stream)

    sampler = ClockSampler(local_rank)
    sampler.start()
    total_ms, clocks, remeasured = _timed_loop(step, K, W, stream, dev, dist, sampler)
    sampler.stop()
    out_ms = float(np.mean([ev[i][0].elapsed_time(ev[i][1]) for i in range(K)]))
    in_ms = float(np.mean([ev[i][1].elapsed_time(ev[i][2]) for i in range(K)]))

    # the copy engines on the same bytes, contiguous: the link's measured rate
    dbuf = torch.empty(max(bytes_out, bytes_in), dtype=torch.uint8, device=dev)
    hbuf = torch.empty(max(bytes_out, bytes_in), dtype=torch.uint8).pin_memory()
    ce = []
    for _ in range(3):
        e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        e[0].record(stream)
        hbuf[:bytes_out].copy_(dbuf[:bytes_out], non_blocking=True)
        e[1].record(stream)
        dbuf[:bytes_in].copy_(hbuf[:bytes_in], non_blocking=True)
        e[2].record(stream)
        torch.cuda.synchronize(dev)
        ce.append((e[0].elapsed_time(e[1]), e[1].elapsed_time(e[2])))
    ce_out_ms = float(np.median([c[0] for c in ce]))
    ce_in_ms = float(np.median([c[1] for c in ce]))
    vals = torch.tensor([out_ms, in_ms, total_ms], dtype=torch.float64, device=dev)
    if dist is not None:
        dist.all_reduce(vals, op=dist.ReduceOp.MAX)
    out_ms, in_ms, total_ms = (float(v) for v in vals.tolist())
    if rank != 0:
        return None
    ms_per_step = total_ms / K
    step_bytes = bytes_out + bytes_in
    achieved = step_bytes / ((out_ms + in_ms) * 1e-3) / 1e9
    peak = step_bytes / ((ce_out_ms + ce_in_ms) * 1e-3) / 1e9
    line = {
        "metric": "block swap GB/s over the host link (GPU -> pinned host and back), preempting a quarter "
                  "of the GQA batch",
        "value": round(step_bytes * world / (ms_per_step * 1e-3) / 1e9, 2), "unit": "GB/s", "n_gpus": world,
        "steps": K, "warmup": W, "ms_per_step": round(ms_per_step, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16 (bit copy)", "data": "synthetic (seeded)",
        "config": {"workload": f"gqa: {workload_description(w)}; the blocks of {len(swapped)} of its "
                               f"{w.num_seqs} sequences ({n_host} blocks of {blk_bytes} bytes per cache) "
                               f"swapped out to a pinned host cache and back in",
                   "step": "pa_swap_blocks GPU -> host (the pool's swap-out plan), then host -> GPU (its "
                           "swap-in plan), K and V caches",
                   "l2": "no flush: each step moves more than L2 (126 MB) each way"},
        "stage_ms": {"swap_out": round(out_ms, 5), "swap_in": round(in_ms, 5)},
        "clocks": clocks,
        "gpu_launches": 2 * K,
        "roofline": {"bound": "host link", "kernel": "pa_swap_blocks (swap_blocks_kernel), both directions",
                     "achieved": round(achieved, 2), "peak": round(peak, 2), "unit": "GB/s",
                     "frac": round(achieved / peak, 4),
                     "peak_source": "measured in this run: cudaMemcpyAsync of the same bytes, contiguous, "
                                    f"device <-> pinned host ({ce_out_ms:.3f} ms out, {ce_in_ms:.3f} ms in)",
                     "traffic": None, "avg_launch_ms": round((out_ms + in_ms) / 2, 5),
                     "per_direction_gbs": {"out": round(bytes_out / (out_ms * 1e-3) / 1e9, 2),
                                           "in": round(bytes_in / (in_ms * 1e-3) / 1e9, 2),
                                           "copy_engine_out": round(bytes_out / (ce_out_ms * 1e-3) / 1e9, 2),
                                           "copy_engine_in": round(bytes_in / (ce_in_ms * 1e-3) / 1e9, 2)}},
        "e2e": None,
        "e2e_note": "the swap already runs between device and host buffers; end-to-end host-buffer timing is "
                    "measured on the decode rows",
    }
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_swap(w, out_pairs, n_host, max(2.0, args.cpu_budget / 2))
    if remeasured:
        line["clocks_note"] = "first timed region saw a thermal/hw slowdown reason; re-measured once"
    return line


def prefix_row_prompts(seed: int, prompts: int = 32, samples: int = 8, prompt_len: int = 1024):
    """The prefix-cache row's requests: `prompts` seeded prompts of random token
    ids, each requested `samples` times in a row (parallel sampling)."""
    rng = np.random.default_rng(seed)
    toks = rng.integers(0, 32000, size=(prompts, prompt_len), dtype=np.int32)
    return [toks[p] for p in range(prompts) for _ in range(samples)]


def prefix_step(pool, requests, free_table):
    """One step of the prefix-cache row: every request's table through the
    pool's prefix cache, then every table freed.  Returns (blocks, cached
    tokens)."""
    tables, cached, blocks = [], 0, 0
    for toks in requests:
        t, c = pool.allocate_prompt_cached(toks)
        tables.append(t)
        cached += c
        blocks += len(t)
    for t in tables:
        free_table(t)
    return blocks, cached


def run_prefix(args, rank: int, world: int, local_rank: int) -> dict | None:
    """Prefix-hash caching in the host pool ([深度解析 «Copy-on-Write 与 Prefix
    Caching»]): 32 prompts of 1024 tokens, each requested by 8 samples in a row;
    every request hashes its full blocks (chained FNV-1a) and reuses the live
    blocks of an equal prefix, then all tables are freed.  Host code only: the
    step is timed by the host clock, and no kernel runs."""
    from paged_kv_cache_379_b200.pool import BlockPool

    if rank != 0:
        return None
    K, W = args.steps, args.warmup
    bs = 16
    requests = prefix_row_prompts(rank_seed(rank, "shared"))
    n_tokens = sum(len(t) for t in requests)
    num_blocks = int(1.2 * n_tokens // bs)
    with BlockPool(num_blocks, bs) as pool:
        for _ in range(W):
            prefix_step(pool, requests, pool.free_table)
        t0 = time.perf_counter()
        for _ in range(K):
            blocks, cached = prefix_step(pool, requests, pool.free_table)
        el = time.perf_counter() - t0
    ms_per_step = el / K * 1e3
    line = {
        "metric": "prefix-cached prompt allocations per second (host block pool)",
        "value": round(len(requests) * K / el, 1), "unit": "prompts/s", "n_gpus": world, "steps": K,
        "warmup": W, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int32 token ids, uint64 hashes", "data": "synthetic (seeded token ids)",
        "config": {"workload": f"prefix: {len(requests) // 8} prompts of 1024 tokens x 8 samples in a row, "
                               f"block_size {bs}, pool of {num_blocks} blocks",
                   "step": "pa_pool_allocate_prompt_cached for every request, then pa_pool_free_table for "
                           "every table"},
        "tokens_hashed_per_s": round(n_tokens * K / el, 1),
        "blocks_per_step": blocks,
        "hit_rate": round(cached / n_tokens, 4),
        "gpu_launches": 0,
        "gpu_note": "host code: the pool is the C++ library's, called through its C ABI; no kernel runs",
        "roofline": None,
        "e2e": None,
    }
    if not args.no_cpu_baseline:
        from oracle.pool import OraclePool
        opool = OraclePool(num_blocks, bs)

        def ofree(t):
            for b in t:
                opool.free(b)
        sub = requests[:64]                    # 8 prompts x 8 samples
        n, t0 = 0, time.perf_counter()
        while time.perf_counter() - t0 < max(2.0, args.cpu_budget / 2):
            prefix_step(opool, sub, ofree)
            n += len(sub)
        el_o = time.perf_counter() - t0
        line["cpu_baseline"] = {"value": round(n / el_o, 1), "unit": "prompts/s", "cores": 1, "kind": "oracle",
                                "sample": f"{n} requests (8 of the prompts x 8 samples, repeated), {el_o:.1f} s, "
                                          "pure Python, one thread"}
    return line


# ---------------------------------------------------------------- the oracle

def _oracle_decode_rate(w, tables, threads: int, budget_s: float):
    """The oracle's decode over chunks of the batch's sequences, cycling, until
    budget_s seconds of oracle time: (bytes/s, seqs/s, sequences, seconds)."""
    import oracle
    chunk = max(1, min(8, int(2e5 // max(float(w.seq_lens.mean()), 1.0))))
    done_bytes, done_seqs, elapsed, i = 0, 0, 0.0, 0
    while elapsed < budget_s:
        idx = (np.arange(chunk) + i) % w.num_seqs
        t = time.perf_counter()
        oracle.paged_decode(w.query[idx], w.key_cache, w.value_cache, tables[idx], w.seq_lens[idx],
                            w.scale, threads=threads)
        elapsed += time.perf_counter() - t
        done_bytes += algorithmic_bytes(w.seq_lens[idx], w.block_size, w.num_heads, w.num_kv_heads, w.head_dim)
        done_seqs += len(idx)
        i += chunk
    return done_bytes / elapsed, done_seqs / elapsed, done_seqs, elapsed


def cpu_baseline(w, tables, budget_s: float = 15.0) -> dict:
    """The oracle (fp64 CPU, as it stands) on a bounded sample of the same
    workload (tables: the step's block tables): once with OpenMP over
    (sequence, head) on all host cores, once single-threaded."""
    import oracle
    threads = oracle.num_threads()
    bps, sps, n, el = _oracle_decode_rate(w, tables, threads, budget_s)
    bps1, sps1, n1, el1 = _oracle_decode_rate(w, tables, 1, max(2.0, budget_s / 3))
    return {"value": round(bps / 1e9, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
            "sample": f"{n} sequence decodes cycling through the {w.num_seqs}-sequence {w.name} batch "
                      f"(decode only), {el:.1f} s, fp64, OpenMP over (sequence, head)",
            "seqs_per_s": round(sps, 2),
            "single_thread": {"value": round(bps1 / 1e9, 4), "unit": "GB/s", "cores": 1,
                              "seqs_per_s": round(sps1, 3),
                              "sample": f"{n1} sequence decodes, {el1:.1f} s, fp64, one thread"}}


def cpu_baseline_swap(w, out_pairs, n_host: int, budget_s: float) -> dict:
    """The oracle's block copy (as it stands) between two host arrays of the
    workload's caches, the swap-out pairs in chunks, until budget_s seconds."""
    import oracle
    hk = np.zeros((n_host,) + w.key_cache.shape[1:], dtype=np.uint16)
    hv = np.zeros_like(hk)
    blk_bytes = w.block_size * w.num_kv_heads * w.head_dim * 2
    done, elapsed, i = 0, 0.0, 0
    chunk = 64
    while elapsed < budget_s:
        idx = (np.arange(chunk) + i) % out_pairs.shape[0]
        t = time.perf_counter()
        oracle.swap_blocks(hk, hv, w.key_cache, w.value_cache, out_pairs[idx])
        elapsed += time.perf_counter() - t
        done += chunk * blk_bytes * 2
        i += chunk
    return {"value": round(done / elapsed / 1e9, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"{done // (blk_bytes * 2)} block pairs of the swap-out plan, K and V, host to host, "
                      f"{elapsed:.1f} s, one thread"}


def cpu_baseline_fp8(w, kc, vc, ks, vs, budget_s: float) -> dict:
    import oracle
    threads = oracle.num_threads()
    done, seqs, elapsed, i = 0, 0, 0.0, 0
    while elapsed < budget_s:
        idx = (np.arange(8) + i) % w.num_seqs
        t = time.perf_counter()
        oracle.paged_decode_fp8(w.query[idx], kc, vc, w.block_tables[idx], w.seq_lens[idx], w.scale, ks, vs,
                                threads=threads)
        elapsed += time.perf_counter() - t
        done += algorithmic_bytes(w.seq_lens[idx], w.block_size, w.num_heads, w.num_kv_heads, w.head_dim, 1)
        seqs += len(idx)
        i += 8
    return {"value": round(done / elapsed / 1e9, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
            "sample": f"{seqs} FP8 sequence decodes cycling through the gqa batch, {elapsed:.1f} s, fp64"}


def cpu_baseline_prefill(w, q, budget_s: float) -> dict:
    """The oracle's prefill on windows of 16 query rows at spread positions."""
    import oracle
    threads = oracle.num_threads()
    P = PREFILL_SHAPE["prompt"]
    flops, rows, elapsed, i = 0, 0, 0.0, 0
    while elapsed < budget_s:
        s = i % w.num_seqs
        end = 16 + (i * 389) % (P - 16)
        qrows = q[s * P + end - 16: s * P + end]
        t = time.perf_counter()
        oracle.paged_prefill(qrows, w.key_cache, w.value_cache, w.block_tables[s:s + 1],
                             np.array([end], np.int32), [16], w.scale, threads=threads)
        elapsed += time.perf_counter() - t
        flops += prefill_flops([end], [16], w.num_heads, w.head_dim)
        rows += 16
        i += 1
    return {"value": round(flops / elapsed / 1e12, 6), "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "sample": f"{rows} query rows (windows of 16 at spread positions of the 2048-token prompts), "
                      f"{elapsed:.1f} s, fp64"}


def run_reference(args, rank: int, world: int) -> dict | None:
    """Reference arm: the oracle timed as it stands, each step a bounded sample
    of the same workload; rank 0 alone runs it."""
    if rank != 0:
        return None
    import oracle
    from paged_kv_cache_379_b200 import workload as wlmod

    oracle.build()
    name = args.workload
    w = wlmod.make(name, seed=rank_seed(0, name), num_seqs=args.num_seqs or None)
    tables = w.block_tables
    if name == "shared":   # the step's tables: each token's block exists (fresh or copied)
        from paged_kv_cache_379_b200.step import host_step
        _, tables, _, _, _ = host_step(w, fork_all=True)
    threads = oracle.num_threads()
    # sample size per step: one sequence, or more while a step stays short
    per_step_budget = max(0.02, 120.0 / max(args.steps + args.warmup, 1))
    t = time.perf_counter()
    oracle.paged_decode(w.query[:1], w.key_cache, w.value_cache, tables[:1], w.seq_lens[:1], w.scale,
                        threads=threads)
    one = time.perf_counter() - t
    mean_len = float(w.seq_lens.mean())
    per_seq = one * mean_len / max(int(w.seq_lens[0]), 1)
    S = int(max(1, min(w.num_seqs, per_step_budget // max(per_seq, 1e-9))))

    def step(j):
        idx = (np.arange(S) + j * S) % w.num_seqs
        oracle.paged_decode(w.query[idx], w.key_cache, w.value_cache, tables[idx], w.seq_lens[idx],
                            w.scale, threads=threads)
        return algorithmic_bytes(w.seq_lens[idx], w.block_size, w.num_heads, w.num_kv_heads, w.head_dim)

    for j in range(args.warmup):
        step(j)
    t0 = time.perf_counter()
    nbytes = 0
    for j in range(args.steps):
        nbytes += step(args.warmup + j)
    dt = time.perf_counter() - t0
    value = nbytes / dt / 1e9
    sample = f"{S} sequence(s) of the {name} batch per step, cycling; fp64 oracle decode"
    return {
        "impl": "reference", "metric": ROW_METRICS[name] + (f" {args.partition}" if name == "long" and args.partition
                                                            else ""), "value": round(value, 4), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1) bf16 values, the workload's lengths, shuffled block pool)",
        "config": decode_config(w, world, bool(args.l2_flush)),
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=10.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--workload", choices=list(DECODE_ROWS) + ["gqa-fp8", "prefill", "cow", "swap", "prefix"],
                    default="gqa")
    ap.add_argument("--partition", type=int, default=0,
                    help="decode rows: force the split form with this many positions per partition "
                         "(0 = the library's plan)")
    ap.add_argument("--num-seqs", type=int, default=0,
                    help="decode rows: only the first N sequences of the workload (a smaller case for "
                         "profiler captures; the line then says so)")
    ap.add_argument("--no-groups", action="store_true",
                    help="shared: decode without the shared-prefix groups (pa_decode / pa_decode_split)")
    ap.add_argument("--unfused-cow", action="store_true",
                    help="shared: the copy-on-write copies as their own launch (pa_copy_blocks) before the "
                         "cache write, instead of fused into it")
    ap.add_argument("--l2-flush", action="store_true",
                    help="decode rows: flush L2 before every step; the step time is then the sum of the "
                         "per-step event intervals")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.partition and (args.partition < 16 or args.partition % 16):
        ap.error("--partition must be a positive multiple of 16")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if args.workload not in DECODE_ROWS:
            ap.error("--impl reference times the oracle's decode: use a decode workload")
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return

    import torch
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    from paged_kv_cache_379_b200.build import build as build_lib
    if rank == 0 or world == 1:
        build_lib()
    if world > 1:
        dist.barrier()
    try:
        if args.workload in DECODE_ROWS:
            line = run_decode(args, rank, world, local_rank)
        elif args.workload == "cow":
            line = run_cow(args, rank, world, local_rank)
        elif args.workload == "swap":
            line = run_swap(args, rank, world, local_rank)
        elif args.workload == "prefix":
            line = run_prefix(args, rank, world, local_rank)
        else:
            line = run_row(args, rank, world, local_rank)
    finally:
        if world > 1:
            dist.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
