"""Build libkvq.so in-tree for sm_100a.

Steps: compile and run the codebook generator (the library's own Gaussian
Lloyd-Max solver) into ``_build/kvq_codebooks_gen.h``, then compile the CUDA
sources into ``libkvq.so`` next to this file. Run: python -m bit_kv_cache_19_b200.build
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libkvq.so")
SOURCES = ["api.cu", "quantize.cu", "decode.cu", "dense.cu", "noalloc.cu", "window.cu"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _run(cmd):
    print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    gen_src = os.path.join(CSRC, "gen_codebooks.cpp")
    gen_bin = os.path.join(BUILD, "gen_codebooks")
    header = os.path.join(BUILD, "kvq_codebooks_gen.h")
    lm = os.path.join(CSRC, "lloydmax_newton.h")
    if force or _stale(gen_bin, [gen_src, lm]):
        _run(["g++", "-O2", "-std=c++17", "-o", gen_bin, gen_src])
    if force or _stale(header, [gen_bin]):
        out = subprocess.run([gen_bin], check=True, capture_output=True, text=True).stdout
        with open(header, "w") as f:
            f.write(out)
    srcs = [os.path.join(CSRC, s) for s in SOURCES]
    headers = sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h")))
    deps = srcs + headers + [header, os.path.join(ROOT, "include", "kvq.h")]
    if force or _stale(LIB, deps):
        from concurrent.futures import ThreadPoolExecutor
        objs, cmds = [], []
        for s in srcs:
            o = os.path.join(BUILD, os.path.basename(s) + ".o")
            cmd = [NVCC, *ARCH, "-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC",
                   "-Xcompiler", "-fvisibility=hidden", "-I", os.path.join(ROOT, "include"),
                   "-I", BUILD, "-c", s, "-o", o]
            if verbose_ptxas:
                cmd.insert(1, "-Xptxas=-v")
            cmds.append(cmd)
            objs.append(o)
        # the translation units compile independently (decode.cu takes longest)
        with ThreadPoolExecutor(max_workers=min(len(cmds), os.cpu_count() or 1)) as ex:
            list(ex.map(_run, cmds))
        _run([NVCC, *ARCH, "-shared", "-o", LIB, *objs, "-cudart", "static"])
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose_ptxas="-v" in sys.argv)
