"""The split decode that allocates nothing (pa_decode_split_noalloc).

pa_decode_split_noalloc is for callers that cannot allocate device memory on
their decode path -- cudaMalloc can synchronise the device and stall a serving
loop, and some hosts fix the device memory a component may own up front -- so
it keeps its scratch in one fixed array inside the library.  Two calls in a
row, on problems of different sizes and partition sizes (so that the second
call's partial results sit at other offsets of the array than the first
call's), are each compared bit for bit with pa_decode_split on the same inputs
and element by element with the fp64 oracle.  This file sorts last, so a run
that stops at the first failure has run every other test first.
"""

import numpy as np
import pytest
import torch

import oracle
from _helpers import assert_close
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


def _problems():
    # 1) 32 sequences of the GQA workload at partition 512: ~8.5 MB of split
    #    workspace, inside the 16 MiB scratch.
    # 2) 12 shorter sequences of another seed with MHA-like heads at partition
    #    256: a smaller layout, so stale partials of call 1 lie where call 2's
    #    m, l and o sections now start.
    w1 = wl.make("gqa", num_seqs=32)
    w2 = wl.random_decode_case(4242, num_seqs=12, num_heads=16, num_kv_heads=4, head_dim=128, block_size=16,
                               lengths=[1, 17, 255, 256, 257, 700, 1000, 1500, 33, 512, 513, 1200])
    return [(w1, 512), (w2, 256)]


def test_noalloc_split_matches_workspace_split_and_oracle_on_two_calls():
    for call, (w, part) in enumerate(_problems()):
        q, kc, vc, bt, sl = _inputs(w)
        need = ops.decode_workspace_size(w.num_seqs, w.num_heads, w.num_kv_heads, w.head_dim, w.max_seq_len, part)
        assert need <= ops.NOALLOC_SCRATCH_BYTES
        ws = ops.new_workspace(w.num_seqs, w.num_heads, w.num_kv_heads, w.head_dim, w.max_seq_len, part,
                               device=DEV)
        ref = ops.decode_split(q, kc, vc, bt, sl, w.scale, w.max_seq_len, part, ws)
        got = ops.decode_split_noalloc(q, kc, vc, bt, sl, w.scale, w.max_seq_len, part)
        torch.cuda.synchronize()
        got_bits = bf16_to_host_bits(got)
        # the same kernels on the same items: the same bits
        assert np.array_equal(got_bits, bf16_to_host_bits(ref)), f"call {call}"
        want = oracle.paged_decode(w.query, w.key_cache, w.value_cache, w.block_tables, w.seq_lens, w.scale)
        assert_close(got_bits, want, f"no-alloc split, call {call} (partition {part})")
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
