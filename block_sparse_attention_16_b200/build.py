"""Build liblbsa.so in-tree with nvcc for sm_100a.

    python -m block_sparse_attention_16_b200.build [--force]

Compiles every ``csrc/*.cu`` to an object under ``_build/`` and links them
into ``block_sparse_attention_16_b200/liblbsa.so`` (static cudart, no libcuda
link: the TMA encoder is fetched through the runtime's driver entry point).
Rebuilds only what changed.
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
OUT = os.path.join(PKG, "liblbsa.so")
OBJ = os.path.join(ROOT, "_build")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
         "-Xcompiler", "-fPIC", "-I", os.path.join(ROOT, "include")]


def _headers_mtime():
    hs = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]
    hs.append(os.path.join(ROOT, "include", "lbsa.h"))
    return max(os.path.getmtime(h) for h in hs)


def build(force: bool = False, verbose: bool = False, defines=(), out: str | None = None,
          obj_dir: str | None = None) -> str:
    """Build liblbsa.so; `defines` (e.g. ["LBSA_SCORE_POLY_EVERY=4"]) and `out` /
    `obj_dir` build a variant library elsewhere."""
    global OUT, OBJ
    out_path, obj_path = out or OUT, obj_dir or OBJ
    saved = OUT, OBJ
    OUT, OBJ = out_path, obj_path
    try:
        return _build(force, verbose, [f"-D{d}" for d in defines])
    finally:
        OUT, OBJ = saved


def _build(force, verbose, dflags) -> str:
    os.makedirs(OBJ, exist_ok=True)
    srcs = sorted(f for f in os.listdir(CSRC) if f.endswith(".cu"))
    hdr = _headers_mtime()
    objs = []
    for f in srcs:
        src = os.path.join(CSRC, f)
        obj = os.path.join(OBJ, f[:-3] + ".o")
        objs.append(obj)
        if force or not os.path.exists(obj) or os.path.getmtime(obj) < max(os.path.getmtime(src), hdr):
            cmd = [NVCC, *FLAGS, *dflags, "-c", src, "-o", obj]
            if verbose:
                print(" ".join(cmd), flush=True)
            subprocess.run(cmd, check=True)
    if force or not os.path.exists(OUT) or os.path.getmtime(OUT) < max(os.path.getmtime(o) for o in objs):
        cmd = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-Xcompiler", "-fPIC",
               *objs, "-o", OUT]
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.run(cmd, check=True)
    return OUT


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
