"""The split decode that allocates nothing (pa_decode_split_noalloc), checked
against the split decode that takes a caller workspace (pa_decode_split).

pa_decode_split_noalloc is for callers that cannot allocate device memory on
their decode path -- cudaMalloc can synchronise the device and stall a serving
loop, and some hosts fix the device memory a component may own up front -- so
it keeps its scratch in one fixed array inside the library.  This file sorts
last, so a run that stops at the first failure has run every other test first.
"""

import numpy as np
import pytest
import torch

import oracle
from _helpers import ATOL, RTOL
from paged_kv_cache_379_b200 import ops
from paged_kv_cache_379_b200 import workload as wl
from paged_kv_cache_379_b200._lib import PagedKVError
from paged_kv_cache_379_b200.step import bf16_to_device, bf16_to_host_bits

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _inputs(w):
    return (bf16_to_device(w.query, DEV), bf16_to_device(w.key_cache, DEV), bf16_to_device(w.value_cache, DEV),
            torch.from_numpy(np.ascontiguousarray(w.block_tables, np.int32)).to(DEV),
            torch.from_numpy(w.seq_lens.astype(np.int32)).to(DEV))


def test_noalloc_split_matches_workspace_split_on_two_calls():
    # 32 sequences of the GQA workload: the split workspace (~8.5 MB at
    # partition 512) fits the library's 16 MiB scratch
    w = wl.make("gqa", num_seqs=32)
    part = 512
    q, kc, vc, bt, sl = _inputs(w)
    need = ops.decode_workspace_size(w.num_seqs, w.num_heads, w.num_kv_heads, w.head_dim, w.max_seq_len, part)
    assert need <= ops.NOALLOC_SCRATCH_BYTES
    ws = ops.new_workspace(w.num_seqs, w.num_heads, w.num_kv_heads, w.head_dim, w.max_seq_len, part,
                           device=DEV)
    ref = ops.decode_split(q, kc, vc, bt, sl, w.scale, w.max_seq_len, part, ws)
    torch.cuda.synchronize()
    ref_bits = bf16_to_host_bits(ref)
    for call in range(2):
        got = ops.decode_split_noalloc(q, kc, vc, bt, sl, w.scale, w.max_seq_len, part)
        torch.cuda.synchronize()
        ok, max_abs, max_rel, _ = oracle.allclose_report(
            oracle.bf16_bits_to_f64(bf16_to_host_bits(got)), oracle.bf16_bits_to_f64(ref_bits), ATOL, RTOL)
        assert ok, f"call {call}: max_abs {max_abs:.3g} max_rel {max_rel:.3g}"
    assert ops.device_status() == 0


def test_noalloc_split_rejects_a_problem_beyond_its_scratch():
    # all 128 sequences at partition 16: ~270 MB of split workspace
    w = wl.make("gqa", fill_cache=False)
    q, kc, vc, bt, sl = _inputs(w)
    assert ops.decode_workspace_size(w.num_seqs, w.num_heads, w.num_kv_heads, w.head_dim, w.max_seq_len, 16) > \
        ops.NOALLOC_SCRATCH_BYTES
    with pytest.raises(PagedKVError) as err:
        ops.decode_split_noalloc(q, kc, vc, bt, sl, w.scale, w.max_seq_len, 16)
    assert err.value.status == -10
