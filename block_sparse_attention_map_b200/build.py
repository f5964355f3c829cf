"""Build libbsa.so in-tree with nvcc for sm_100a (no torch extension machinery).

``python -m block_sparse_attention_map_b200.build`` or ``build()`` from Python.
The shared library lands next to this file so it travels with the source tree.
"""

from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
LIB = os.path.join(HERE, "libbsa.so")
SOURCES = ["api.cu", "plan.cu", "fwd.cu", "bwd.cu", "static_scratch.cu"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.isabs(cand) and os.path.exists(cand) or not os.path.isabs(cand)):
            return cand
    return "nvcc"


def flags(verbose_ptxas: bool = False):
    f = [
        "-std=c++17", "-O3", "-lineinfo",
        "-gencode", "arch=compute_100a,code=sm_100a",
        "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
        "--expt-relaxed-constexpr",
        "-I", INCLUDE,
    ]
    if verbose_ptxas:
        f += ["-Xptxas", "-v"]
    return f


def build(verbose: bool = False, verbose_ptxas: bool = False, jobs: int = 4) -> str:
    """Compile every source to an object, link libbsa.so; returns its path."""
    objdir = os.path.join(HERE, "_build")
    os.makedirs(objdir, exist_ok=True)
    procs = []
    objs = []
    for src in SOURCES:
        obj = os.path.join(objdir, src.replace(".cu", ".o"))
        objs.append(obj)
        cmd = [nvcc(), "-c", os.path.join(CSRC, src), "-o", obj] + flags(verbose_ptxas)
        if verbose:
            print(" ".join(cmd), flush=True)
        procs.append((src, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT)))
    failed = []
    for src, p in procs:
        out, _ = p.communicate()
        text = out.decode(errors="replace")
        if p.returncode != 0:
            failed.append((src, text))
        elif text.strip() and (verbose or verbose_ptxas):
            print(text)
    if failed:
        msg = "\n".join(f"--- {s}\n{t}" for s, t in failed)
        raise RuntimeError(f"nvcc failed:\n{msg}")
    link = [nvcc(), "-shared", "-o", LIB] + objs + [
        "-gencode", "arch=compute_100a,code=sm_100a", "-cudart", "static",
        "-Xcompiler", "-fPIC"]
    if verbose:
        print(" ".join(link), flush=True)
    subprocess.run(link, check=True)
    return LIB


if __name__ == "__main__":
    build(verbose="-v" in sys.argv, verbose_ptxas="--ptxas" in sys.argv)
    print(LIB)
