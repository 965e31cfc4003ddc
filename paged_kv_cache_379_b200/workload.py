"""Seeded synthetic inputs for the paged-KV decode path.

This module draws random numbers and random structure only -- values, sequence
lengths and which physical blocks each sequence owns.  It contains none of the
method's arithmetic (no slot computation, no cache write, no attention), so the
tests can feed the very same arrays to the CUDA path and to the independent
oracle.  It depends on numpy alone.

Five workloads, named by what they are:

* ``tiny``   -- 4 sequences of lengths {7, 16, 33, 50}, 4/4 heads, head_dim 64,
  block_size 4, a pool of 64 physical blocks; tables are a seeded draw without
  replacement from the pool.
* ``mha``    -- 64 sequences, 32/32 heads, head_dim 128, block_size 16, lengths
  uniform in [128, 2048]; pool 1.25x the blocks needed, shuffled.
* ``gqa``    -- 128 sequences, 64 query / 8 KV heads, head_dim 128, block_size 16,
  lengths lognormal with median 1024 and sigma 0.8, rounded and clipped to
  [16, 4096]; pool 1.2x, shuffled.
* ``long``   -- 8 sequences, 32 query / 8 KV heads, head_dim 128, block_size 16,
  lengths uniform in [32768, 131072]; pool 1.2x, shuffled.
* ``shared`` -- 32 prompts of 1024 tokens, each shared by 8 samples (256
  sequences whose tables start with the same 64 prompt blocks), private tails of
  uniform [1, 256] tokens; 32/8 heads, head_dim 128, block_size 16; pool 1.2x.

Values are N(0, 1) float32 rounded to bf16 (round to nearest even); they are
kept as raw uint16 bit patterns.  Every sequence length counts the token being
decoded: its K/V are the ``new_key`` / ``new_value`` rows, and it sits at
logical position ``seq_len - 1``.  Blocks nobody owns are filled with bf16 NaN
so that a read of a wrong block shows up.
"""

from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

BF16_NAN = np.uint16(0x7FC0)
NAMES = ("tiny", "mha", "gqa", "long", "shared")
SEED_BASE = 379


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns, round to nearest even (NaN kept NaN)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    rounded = ((u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)).astype(np.uint16)
    nan = np.isnan(x)
    if nan.any():
        rounded[nan] = BF16_NAN
    return rounded


def bf16_normal(rng: np.random.Generator, shape, chunk: int = 1 << 22) -> np.ndarray:
    """N(0, 1) values rounded to bf16.

    The values are drawn in fixed-size chunks, each from its own PCG64 stream
    seeded from `rng`, on a thread pool; the result depends only on `rng`'s
    state, not on the number of threads.
    """
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    starts = list(range(0, n, chunk))
    seeds = rng.integers(0, 2**63 - 1, size=max(len(starts), 1), dtype=np.int64)

    def fill(i):
        start = starts[i]
        stop = min(n, start + chunk)
        g = np.random.Generator(np.random.PCG64(int(seeds[i])))
        out[start:stop] = f32_to_bf16_bits(g.standard_normal(stop - start, dtype=np.float32))

    if len(starts) <= 1:
        for i in range(len(starts)):
            fill(i)
    else:
        workers = min(len(starts), os.cpu_count() or 1, 32)
        with ThreadPoolExecutor(max_workers=workers) as ex:
            list(ex.map(fill, range(len(starts))))
    return out.reshape(shape)


def _fill_cache(rng, num_blocks, bs, hkv, d, free):
    """Cache contents: random bf16 in owned blocks, bf16 NaN in unowned ones."""
    cache = np.empty((num_blocks, bs, hkv, d), dtype=np.uint16)
    is_free = np.zeros(num_blocks, dtype=bool)
    is_free[np.asarray(free, dtype=np.int64)] = True
    owned = np.flatnonzero(~is_free)
    cache[is_free] = BF16_NAN
    cache[owned] = bf16_normal(rng, (owned.size, bs, hkv, d))
    return cache


E4M3_NAN = np.uint8(0x7F)


def fp8_codes(rng: np.random.Generator, shape, zero_exp_frac: float = 0.05) -> np.ndarray:
    """Random E4M3 codes (uint8): sign uniform, mantissa field uniform in 0..7,
    exponent field uniform in 3..9 (magnitudes 2^-4 .. 2^2 * 1.875), except a
    fraction `zero_exp_frac` of codes with exponent field 0 (zero and
    subnormals).  Never the NaN pattern (exponent 15, mantissa 7)."""
    n = int(np.prod(shape))
    sign = rng.integers(0, 2, n, dtype=np.uint8) << 7
    exp = rng.integers(3, 10, n, dtype=np.uint8)
    exp[rng.random(n) < zero_exp_frac] = 0
    man = rng.integers(0, 8, n, dtype=np.uint8)
    return (sign | (exp << 3) | man).astype(np.uint8).reshape(shape)


def fp8_cache(rng: np.random.Generator, num_blocks: int, bs: int, hkv: int, d: int, free) -> np.ndarray:
    """An E4M3 code cache: random codes in owned blocks, the NaN code in unowned ones."""
    cache = np.empty((num_blocks, bs, hkv, d), dtype=np.uint8)
    is_free = np.zeros(num_blocks, dtype=bool)
    is_free[np.asarray(free, dtype=np.int64)] = True
    owned = np.flatnonzero(~is_free)
    cache[is_free] = E4M3_NAN
    cache[owned] = fp8_codes(rng, (owned.size, bs, hkv, d))
    return cache


@dataclass
class Workload:
    name: str
    seed: int
    num_seqs: int
    num_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    scale: float
    seq_lens: np.ndarray          # int32 [B], including the token being decoded
    block_tables: np.ndarray      # int32 [B, max_blocks], -1 past each sequence's blocks
    blocks_per_seq: np.ndarray    # int32 [B], number of valid entries in each table row
    query: np.ndarray             # uint16 bf16 bits [B, Hq, D]
    new_key: np.ndarray           # uint16 bf16 bits [B, Hkv, D]
    new_value: np.ndarray         # uint16 bf16 bits [B, Hkv, D]
    key_cache: np.ndarray         # uint16 bf16 bits [nb, bs, Hkv, D]
    value_cache: np.ndarray       # uint16 bf16 bits [nb, bs, Hkv, D]
    free_blocks: np.ndarray       # int32: unowned blocks, in free-list order
    extra: dict = field(default_factory=dict)

    @property
    def max_blocks(self) -> int:
        return int(self.block_tables.shape[1])

    @property
    def max_seq_len(self) -> int:
        return int(self.seq_lens.max(initial=0))

    @property
    def group(self) -> int:
        return self.num_heads // self.num_kv_heads


def _ceil_div(a, b):
    return -(-np.asarray(a, dtype=np.int64) // b)


def _lengths(name: str, rng: np.random.Generator, B: int) -> np.ndarray:
    if name == "tiny":
        return np.array([7, 16, 33, 50], dtype=np.int32)
    if name == "mha":
        return rng.integers(128, 2048, size=B, endpoint=True).astype(np.int32)
    if name == "gqa":
        x = np.rint(np.exp(np.log(1024.0) + 0.8 * rng.standard_normal(B)))
        return np.clip(x, 16, 4096).astype(np.int32)
    if name == "long":
        return rng.integers(32768, 131072, size=B, endpoint=True).astype(np.int32)
    raise ValueError(name)


_SHAPES = {
    #          B    Hq  Hkv  D   bs
    "tiny": (4, 4, 4, 64, 4),
    "mha": (64, 32, 32, 128, 16),
    "gqa": (128, 64, 8, 128, 16),
    "long": (8, 32, 8, 128, 16),
    "shared": (256, 32, 8, 128, 16),
}
_POOL_FACTOR = {"mha": 1.25, "gqa": 1.2, "long": 1.2, "shared": 1.2}


def make(name: str, seed: int | None = None, *, num_seqs: int | None = None,
         lengths=None, fill_cache: bool = True, shared_prompt_len: int = 1024,
         shared_samples: int = 8) -> Workload:
    """Build one named workload.  ``num_seqs`` / ``lengths`` shrink it for tests."""
    if name not in _SHAPES:
        raise ValueError(f"unknown workload {name!r}; choose from {NAMES}")
    if seed is None:
        seed = SEED_BASE + NAMES.index(name)
    rng = np.random.Generator(np.random.PCG64(seed))
    B, Hq, Hkv, D, bs = _SHAPES[name]
    if num_seqs is not None:
        B = int(num_seqs)
    extra: dict = {}

    if name == "shared":
        samples = shared_samples
        prompts = max(1, B // samples)
        B = prompts * samples
        tails = rng.integers(1, 256, size=B, endpoint=True) if lengths is None else np.asarray(lengths)
        seq_lens = (shared_prompt_len + tails).astype(np.int32)
        prompt_blocks = int(_ceil_div(shared_prompt_len, bs))
        # blocks already holding data before this step: the prompt's, plus the
        # tail's private ones for the seq_len - 1 cached tokens
        cached = seq_lens.astype(np.int64) - 1
        tail_blocks = _ceil_div(cached, bs) - prompt_blocks
        tail_blocks = np.maximum(tail_blocks, 0)
        needed = prompts * prompt_blocks + int(tail_blocks.sum())
        # room for one new block or one copy per sequence in the step
        num_blocks = int(np.ceil(_POOL_FACTOR[name] * (needed + B)))
        perm = rng.permutation(num_blocks).astype(np.int32)
        take = 0
        width = int(_ceil_div(seq_lens.max(), bs))
        tables = np.full((B, width), -1, dtype=np.int32)
        nblk = np.zeros(B, dtype=np.int32)
        for p in range(prompts):
            pblocks = perm[take:take + prompt_blocks]
            take += prompt_blocks
            for i in range(samples):
                s = p * samples + i
                tb = int(tail_blocks[s])
                tables[s, :prompt_blocks] = pblocks
                tables[s, prompt_blocks:prompt_blocks + tb] = perm[take:take + tb]
                take += tb
                nblk[s] = prompt_blocks + tb
        free = perm[take:]
        extra.update(prompts=prompts, samples=samples, prompt_len=shared_prompt_len,
                     prompt_blocks=prompt_blocks)
        if name == "shared" and shared_prompt_len % bs:
            extra["partial_prompt_block"] = True
    else:
        seq_lens = _lengths(name, rng, B) if lengths is None else np.asarray(lengths, dtype=np.int32)
        B = int(seq_lens.shape[0])
        need = _ceil_div(seq_lens, bs).astype(np.int32)
        total = int(need.sum())
        num_blocks = 64 if name == "tiny" else int(np.ceil(_POOL_FACTOR[name] * total))
        num_blocks = max(num_blocks, total)
        perm = rng.permutation(num_blocks).astype(np.int32)
        width = int(need.max(initial=1)) if B else 1
        tables = np.full((B, max(width, 1)), -1, dtype=np.int32)
        take = 0
        for s in range(B):
            tables[s, :need[s]] = perm[take:take + need[s]]
            take += int(need[s])
        nblk = need
        free = perm[take:]

    query = bf16_normal(rng, (B, Hq, D))
    new_key = bf16_normal(rng, (B, Hkv, D))
    new_value = bf16_normal(rng, (B, Hkv, D))
    cache_shape = (num_blocks, bs, Hkv, D)
    if fill_cache:
        key_cache = _fill_cache(rng, num_blocks, bs, Hkv, D, free)
        value_cache = _fill_cache(rng, num_blocks, bs, Hkv, D, free)
    else:
        key_cache = np.zeros(cache_shape, dtype=np.uint16)
        value_cache = np.zeros(cache_shape, dtype=np.uint16)
    return Workload(name=name, seed=seed, num_seqs=B, num_heads=Hq, num_kv_heads=Hkv,
                    head_dim=D, block_size=bs, num_blocks=num_blocks,
                    scale=float(1.0 / np.sqrt(D)), seq_lens=seq_lens.astype(np.int32),
                    block_tables=tables, blocks_per_seq=np.asarray(nblk, dtype=np.int32),
                    query=query, new_key=new_key, new_value=new_value,
                    key_cache=key_cache, value_cache=value_cache,
                    free_blocks=np.asarray(free, dtype=np.int32), extra=extra)


def random_decode_case(seed: int, *, num_seqs: int, num_heads: int, num_kv_heads: int,
                       head_dim: int, block_size: int, lengths, spare_blocks: int = 3) -> Workload:
    """A small custom case (tests): given lengths, shuffled pool with a few spare blocks."""
    rng = np.random.Generator(np.random.PCG64(seed))
    seq_lens = np.asarray(lengths, dtype=np.int32)
    assert seq_lens.shape[0] == num_seqs
    need = _ceil_div(seq_lens, block_size).astype(np.int32)
    total = int(need.sum())
    num_blocks = total + spare_blocks
    perm = rng.permutation(num_blocks).astype(np.int32)
    width = max(int(need.max(initial=1)), 1)
    tables = np.full((num_seqs, width), -1, dtype=np.int32)
    take = 0
    for s in range(num_seqs):
        tables[s, :need[s]] = perm[take:take + need[s]]
        take += int(need[s])
    free = perm[take:]
    Hq, Hkv, D = num_heads, num_kv_heads, head_dim
    query = bf16_normal(rng, (num_seqs, Hq, D))
    new_key = bf16_normal(rng, (num_seqs, Hkv, D))
    new_value = bf16_normal(rng, (num_seqs, Hkv, D))
    key_cache = _fill_cache(rng, num_blocks, block_size, Hkv, D, free)
    value_cache = _fill_cache(rng, num_blocks, block_size, Hkv, D, free)
    return Workload(name="custom", seed=seed, num_seqs=num_seqs, num_heads=Hq, num_kv_heads=Hkv,
                    head_dim=D, block_size=block_size, num_blocks=num_blocks,
                    scale=float(1.0 / np.sqrt(D)), seq_lens=seq_lens, block_tables=tables,
                    blocks_per_seq=need, query=query, new_key=new_key, new_value=new_value,
                    key_cache=key_cache, value_cache=value_cache, free_blocks=free)

