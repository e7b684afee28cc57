"""Builds the in-tree CUDA library ``libthdattn.so`` for sm_100a with nvcc.

Usage: ``python -m sliding_window_gqa_cu_b200.build [--force] [--verbose-ptxas]``.
"""
from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libthdattn.so")
SOURCES = [os.path.join(CSRC, "thd_attn_api.cu"), os.path.join(CSRC, "thd_attn_noalloc.cu"),
           os.path.join(CSRC, "thd_prologue.cu"), os.path.join(CSRC, "thd_sparse_mla.cu"),
           os.path.join(CSRC, "thd_host_pipeline.cu"), os.path.join(CSRC, "thd_attn_merge.cu"),
           os.path.join(CSRC, "scheduler.cpp")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in ("thd_attn_kernel.cuh", "thd_attn_split_kernel.cuh",
                                                  "thd_attn_bwd_kernels.cuh",
                                                  "sm100_ptx.cuh", "scheduler.h", "tma_map.h")] \
    + [os.path.join(ROOT, "include", "thd_attn.h")]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in DEPS if os.path.exists(p))


def build(force: bool = False, verbose_ptxas: bool = False, out: str = LIB,
          defines: tuple = ()) -> str:
    """Build the library (if a source is newer) into ``out``; ``defines`` are
    extra ``-D`` flags (e.g. ``("THD_DEBUG=1",)`` for the debug build, which a
    different ``out`` keeps apart from the regular library)."""
    if out == LIB and not defines and not force and not needs_build():
        return LIB
    if out != LIB and not force and os.path.exists(out) and \
            all(os.path.getmtime(p) <= os.path.getmtime(out) for p in DEPS if os.path.exists(p)):
        return out
    cmd = [nvcc_path(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo",
           "-std=c++17", "-Xcompiler", "-fPIC,-O2", "-shared", "--expt-relaxed-constexpr",
           *[f"-D{d}" for d in defines],
           "-I", os.path.join(ROOT, "include"), "-o", out + ".tmp", *SOURCES]
    if verbose_ptxas:
        cmd[1:1] = ["-Xptxas", "-v"]
    subprocess.run(cmd, check=True)
    os.replace(out + ".tmp", out)
    return out


def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose-ptxas", action="store_true")
    a = ap.parse_args(argv)
    print(build(force=a.force, verbose_ptxas=a.verbose_ptxas))
    return 0


if __name__ == "__main__":
    sys.exit(main())
