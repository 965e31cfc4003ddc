"""The C-ABI library loads and exports every symbol include/pagedkv.h declares;
argument checks answer on the host without touching a GPU (CPU only)."""

import ctypes
import os
import re

import pytest

from paged_kv_cache_379_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pagedkv.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pa_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    return _lib.load()


def test_header_declares_the_boundary():
    names = _declared()
    for required in ("pa_reshape_and_cache", "pa_decode", "pa_copy_blocks", "pa_slot_mapping",
                     "pa_decode_one_pass", "pa_decode_split", "pa_lse_reduce", "pa_pool_create"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    raw = ctypes.CDLL(_lib.LIB_PATH)
    missing = [n for n in _declared() if not hasattr(raw, n)]
    assert not missing, missing
    # and the binding knows every one of them
    assert set(_declared()) <= set(_lib.SIGNATURES)


def test_status_strings(lib):
    assert _lib.status_string(0) == "ok"
    for code in range(-1, -13, -1):
        assert _lib.status_string(code) != "unknown status"
    assert lib.pa_version() >= 10000


def test_argument_errors_without_gpu(lib):
    P = ctypes.c_void_p
    # null pointers
    assert lib.pa_decode(None, None, None, None, None, None, 1.0, 16, 8, 4, 64, 128, 8, 100, 128,
                         None, 0, None) == -1
    fake = P(4096)
    # num_heads not a multiple of num_kv_heads
    assert lib.pa_decode(fake, fake, fake, fake, fake, fake, 1.0, 16, 8, 4, 63, 128, 8, 100, 128,
                         None, 0, None) == -2
    # unsupported head_dim / block_size / group
    assert lib.pa_decode_one_pass(fake, fake, fake, fake, fake, fake, 1.0, 16, 8, 4, 64, 96, 8, 100,
                                  128, None) == -3
    assert lib.pa_decode_one_pass(fake, fake, fake, fake, fake, fake, 1.0, 32, 8, 4, 64, 128, 8, 100,
                                  128, None) == -3
    assert lib.pa_decode_one_pass(fake, fake, fake, fake, fake, fake, 1.0, 16, 2, 4, 64, 128, 8, 100,
                                  128, None) == -3
    # misaligned pointer
    assert lib.pa_decode_one_pass(P(4100), fake, fake, fake, fake, fake, 1.0, 16, 8, 4, 64, 128, 8,
                                  100, 128, None) == -8
    # split without workspace, bad partition size
    assert lib.pa_decode_split(fake, fake, fake, fake, fake, fake, 1.0, 16, 8, 4, 64, 128, 8, 100,
                               128, 512, None, 0, None) == -4
    assert lib.pa_decode_split(fake, fake, fake, fake, fake, fake, 1.0, 16, 8, 4, 64, 128, 8, 100,
                               128, 100, fake, 1 << 30, None) == -2
    # empty work is a no-op
    assert lib.pa_slot_mapping(None, None, 4, 1, None, None, None, 0, 16, None) == 0
    assert lib.pa_slot_mapping(fake, fake, 4, 1, None, None, fake, 5, 16, None) == -2
    assert lib.pa_copy_blocks(fake, fake, None, 0, 8, 128, 16, 10, None) == 0
    assert lib.pa_reshape_and_cache(None, None, None, None, None, 0, 8, 128, 16, 10, None) == 0
    assert lib.pa_reshape_and_cache(fake, fake, fake, fake, fake, 3, 8, 128, 16, 0, None) == -2


def test_fp8_argument_errors_without_gpu(lib):
    P = ctypes.c_void_p
    fake = P(4096)
    # (out, q, kc, vc, bt, sl, scale, k_scale, v_scale, bs, Hkv, B, Hq, D, max_blocks, nb, max_len, ws, ws_bytes, st)
    assert lib.pa_decode_fp8(fake, fake, fake, fake, fake, fake, 1.0, 1.0, 1.0, 16, 8, 4, 64, 64, 8, 100, 128,
                             None, 0, None) == -3       # head_dim 64 not compiled for FP8
    assert lib.pa_decode_fp8(fake, fake, fake, fake, fake, fake, 1.0, 1.0, 1.0, 4, 8, 4, 64, 128, 8, 100, 128,
                             None, 0, None) == -3       # block_size 4 not compiled for FP8
    assert lib.pa_decode_fp8(fake, fake, fake, fake, fake, fake, 1.0, 0.0, 1.0, 16, 8, 4, 64, 128, 8, 100, 128,
                             None, 0, None) == -2       # scales must be positive and finite
    assert lib.pa_decode_fp8(fake, fake, fake, fake, fake, fake, 1.0, 1.0, float("nan"), 16, 8, 4, 64, 128, 8,
                             100, 128, None, 0, None) == -2
    assert lib.pa_decode_fp8_split(fake, fake, fake, fake, fake, fake, 1.0, 1.0, 1.0, 16, 8, 4, 64, 128, 8, 100,
                                   128, 512, None, 0, None) == -4   # split form needs a workspace
    # (k, v, kc, vc, slots, T, Hkv, D, bs, nb, k_scale, v_scale, st)
    assert lib.pa_reshape_and_cache_fp8(fake, fake, fake, fake, fake, 3, 8, 128, 16, 10, -1.0, 1.0, None) == -2
    assert lib.pa_reshape_and_cache_fp8(fake, fake, fake, fake, fake, 3, 1, 8, 16, 10, 1.0, 1.0, None) == -3
    assert lib.pa_reshape_and_cache_fp8(None, None, None, None, None, 0, 8, 128, 16, 10, 1.0, 1.0, None) == 0


def test_fp8_code_generator_never_draws_nan():
    import numpy as np
    from paged_kv_cache_379_b200 import workload as wl
    c = wl.fp8_codes(np.random.default_rng(0), (200000,))
    assert c.dtype == np.uint8 and not ((c & 0x7F) == 0x7F).any()
    exps = np.unique((c >> 3) & 15)
    assert 0 in exps and set(exps) <= {0, 3, 4, 5, 6, 7, 8, 9}


def test_workspace_size(lib):
    # 256-byte scheduler header, then for 4 seqs x 8 heads x ceil(1000/512)=2 parts:
    # o = 64*128*4 B, m and l = 64*4 B each (each 256-aligned)
    assert lib.pa_decode_workspace_size(4, 8, 2, 128, 1000, 512) == 256 + 64 * 128 * 4 + 2 * 256
    assert lib.pa_decode_workspace_size(4, 8, 2, 128, 0, 512) == 256 + 32 * 128 * 4 + 2 * 256
    assert lib.pa_decode_workspace_size(0, 8, 2, 128, 10, 512) == 0


def test_prefill_argument_errors_without_gpu(lib):
    P = ctypes.c_void_p
    fake = P(4096)
    # (out, q, kc, vc, bt, sl, q_start, scale, bs, Hkv, B, Hq, D, max_blocks, nb, T, stream)
    ok_args = (fake, fake, fake, fake, fake, fake, fake, 0.1, 16, 8, 4, 64, 128, 8, 100, 64, None)

    def call(**kw):
        names = ["out", "q", "kc", "vc", "bt", "sl", "qs", "scale", "bs", "hkv", "b", "hq", "d", "mb", "nb", "t",
                 "st"]
        args = dict(zip(names, ok_args))
        args.update(kw)
        return lib.pa_prefill(*[args[n] for n in names])

    assert call(d=96) == -3            # head_dim not compiled
    assert call(bs=4) == -3            # block_size not compiled
    assert call(hq=136, hkv=8) == -3   # G = 17 > 16
    assert call(hq=63) == -2           # num_heads not a multiple of num_kv_heads
    for bad in (0.0, -0.125, float("nan"), float("inf")):
        assert call(scale=bad) == -2   # the scale must be finite and > 0
    assert call(nb=0) == -2
    assert call(t=0) == 0              # no query rows: nothing to do
    assert call(b=0) == 0
    assert call(out=None) == -1
    assert call(q=P(4100)) == -8       # misaligned query


def test_shared_prefix_and_cow_argument_errors_without_gpu(lib):
    P = ctypes.c_void_p
    fake = P(4096)
    # pa_decode_shared(out, q, kc, vc, bt, sl, scale, bs, Hkv, B, Hq, D, max_blocks, nb, max_len, part,
    #                  group_start, group_parts, num_groups, ws, ws_bytes, st)
    args = [fake, fake, fake, fake, fake, fake, 1.0, 16, 8, 4, 64, 128, 8, 100, 128, 512, fake, fake, 2, fake,
            1 << 30, None]

    def shared(changes):
        a = list(args)
        for i, v in changes.items():
            a[i] = v
        return lib.pa_decode_shared(*a)
    assert shared({16: None}) == -1      # groups given without their starts
    assert shared({18: 5}) == -2         # more groups than sequences
    assert shared({18: -1}) == -2
    assert shared({15: 100}) == -2       # partition size not a multiple of 16
    assert shared({19: None, 20: 0}) == -4   # the split form needs a workspace
    assert shared({11: 96}) == -3        # head_dim not compiled
    # pa_append_decode_kv_cow(k, v, kc, vc, bt, sl, cow_src, slots, B, max_blocks, Hkv, D, bs, nb, st)
    assert lib.pa_append_decode_kv_cow(None, None, None, None, None, None, None, None, 0, 8, 8, 128, 16, 10,
                                       None) == 0
    assert lib.pa_append_decode_kv_cow(fake, fake, fake, fake, fake, fake, None, None, 3, 8, 8, 128, 16, 0,
                                       None) == -2
    assert lib.pa_append_decode_kv_cow(None, fake, fake, fake, fake, fake, None, None, 3, 8, 8, 128, 16, 10,
                                       None) == -1
    assert lib.pa_append_decode_kv_cow(fake, fake, fake, fake, fake, fake, None, None, 70000, 8, 8, 128, 16, 10,
                                       None) == -2   # one grid row per sequence
    assert lib.pa_append_decode_kv_cow(P(4100), fake, fake, fake, fake, fake, None, None, 3, 8, 8, 128, 16, 10,
                                       None) == -8


def test_prefix_groups_argument_errors(lib):
    import numpy as np
    t = np.zeros((2, 4), np.int32)
    lens = np.array([8, 8], np.int32)
    out_s = np.zeros(3, np.int32)
    out_p = np.zeros(2, np.int32)
    n = ctypes.c_int(0)
    ptr = lambda a: a.ctypes.data_as(ctypes.c_void_p)  # noqa: E731
    # partition size not a multiple of the block size
    assert lib.pa_prefix_groups(ptr(t), 2, 4, ptr(lens), 4, 6, ptr(out_s), ptr(out_p), ctypes.byref(n)) == -2
    assert lib.pa_prefix_groups(ptr(t), 2, 4, ptr(lens), 4, 8, None, ptr(out_p), ctypes.byref(n)) == -1
    assert lib.pa_prefix_groups(ptr(t), 2, 4, ptr(lens), 4, 8, ptr(out_s), ptr(out_p), ctypes.byref(n)) == 0
    assert n.value == 1 and out_s.tolist() == [0, 2, 0] and out_p[0] == 1
