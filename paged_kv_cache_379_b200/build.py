"""Build libpagedkv.so in-tree with nvcc for sm_100a.

    python -m paged_kv_cache_379_b200.build [--force]

The library is one CUDA translation unit (csrc/pagedkv.cu, which includes the
kernels) plus the host block pool (csrc/block_pool.cpp), linked into
paged_kv_cache_379_b200/libpagedkv.so against the CUDA runtime only.
"""

from __future__ import annotations

import os
import shutil
import subprocess
import sys
import tempfile

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
LIB = os.path.join(HERE, "libpagedkv.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libpagedkv.so")


def sources() -> list[str]:
    out = [os.path.join(CSRC, f) for f in sorted(os.listdir(CSRC))
           if f.endswith((".cu", ".cuh", ".cpp", ".h"))]
    out.append(os.path.join(INCLUDE, "pagedkv.h"))
    return out


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(s) > t for s in sources())


def build(force: bool = False, verbose: bool = False, ptxas_verbose: bool = False) -> str:
    if not force and not needs_build():
        return LIB
    nvcc = _nvcc()
    with tempfile.TemporaryDirectory(prefix="pagedkv_build_") as tmp:
        objs = []
        cu_flags = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O3",
                           "--expt-relaxed-constexpr", "-I", INCLUDE]
        if ptxas_verbose:
            cu_flags += ["-Xptxas", "-v"]
        cxx = shutil.which("g++") or "g++"
        for src, compiler, flags in ((os.path.join(CSRC, "pagedkv.cu"), nvcc, cu_flags),
                                     (os.path.join(CSRC, "block_pool.cpp"), cxx,
                                      ["-O3", "-std=c++17", "-fPIC", "-I", INCLUDE])):
            obj = os.path.join(tmp, os.path.basename(src) + ".o")
            cmd = [compiler, "-c", src, "-o", obj] + flags
            if verbose:
                print(" ".join(cmd), flush=True)
            subprocess.check_call(cmd)
            objs.append(obj)
        out_tmp = os.path.join(tmp, "libpagedkv.so")
        cmd = [nvcc, "-shared"] + ARCH + ["-o", out_tmp] + objs + ["-lcudart"]
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.check_call(cmd)
        shutil.copyfile(out_tmp, LIB + ".tmp")
        os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    force = "--force" in sys.argv
    print(build(force=force, verbose=True, ptxas_verbose="--ptxas-v" in sys.argv))
