"""Build libattn_b200.so in-tree for sm_100a with nvcc.

    python -m exact_softmax_attention_causal_b200.csrc.build [--verbose-ptxas]

The shared library lands next to the Python binding
(exact_softmax_attention_causal_b200/libattn_b200.so). The CUDA runtime is
linked statically; the driver entry point for tensor-map encoding is looked
up at run time, so the build needs no GPU and no libcuda.
"""

from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
PKG = os.path.dirname(HERE)
ROOT = os.path.dirname(PKG)
LIB = os.path.join(PKG, "libattn_b200.so")
SOURCES = ["attn_api.cu", "prefill_sm100.cu", "decode_sm100.cu", "decode_noalloc.cu", "mla_sm100.cu", "backward_sm100.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found")
    return cand


def build(verbose_ptxas: bool = False, force: bool = False) -> str:
    srcs = [os.path.join(HERE, s) for s in SOURCES]
    deps = srcs + [os.path.join(HERE, h) for h in ("ptx.cuh", "internal.h")] + [os.path.join(ROOT, "include", "attn.h")]
    if not force and os.path.exists(LIB) and all(os.path.getmtime(LIB) >= os.path.getmtime(d) for d in deps):
        return LIB
    cmd = [nvcc(), "-O3", "-std=c++17", *ARCH, "-lineinfo", "-shared", "-Xcompiler", "-fPIC",
           "-Xcompiler", "-fvisibility=hidden", "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include"),
           "-o", LIB + ".tmp", *srcs]
    if verbose_ptxas:
        cmd += ["-Xptxas", "-v"]
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--verbose-ptxas", action="store_true")
    ap.add_argument("--force", action="store_true")
    a = ap.parse_args()
    print(build(a.verbose_ptxas, a.force))
    sys.exit(0)
