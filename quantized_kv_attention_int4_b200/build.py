"""Build libflashloop_b200.so in-tree with nvcc for sm_100a.

Usage: python -m quantized_kv_attention_int4_b200.build [--verbose-ptxas]
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_NAME = "libflashloop_b200.so"
LIB_PATH = os.path.join(PKG, LIB_NAME)
SOURCES = ["api.cu", "encode.cu", "dense.cu", "dense_staged.cu", "sparse.cu", "sparse_staged.cu", "sparse_persist.cu", "select.cu", "tokens.cu", "prefill.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found; the FlashLoop CUDA library cannot be built")


def _newest_source_mtime() -> float:
    paths = [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [os.path.join(INCLUDE, "flashloop.h")]
    return max(os.path.getmtime(p) for p in paths)


def build(force: bool = False, ptxas_verbose: bool = False) -> str:
    """Compile every translation unit and link the shared library; returns its path."""
    if not force and os.path.exists(LIB_PATH) and os.path.getmtime(LIB_PATH) >= _newest_source_mtime():
        return LIB_PATH
    obj_dir = os.path.join(PKG, "_build")
    os.makedirs(obj_dir, exist_ok=True)
    objs = []
    common = [nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC",
              "-I", INCLUDE, "-I", CSRC, "--expt-relaxed-constexpr"]
    if ptxas_verbose:
        common += ["-Xptxas", "-v"]
    cmds = []
    for src in SOURCES:
        obj = os.path.join(obj_dir, src.replace(".cu", ".o"))
        cmds.append(common + ["-c", os.path.join(CSRC, src), "-o", obj])
        objs.append(obj)
    # translation units compile independently: one nvcc per unit, in parallel
    with ThreadPoolExecutor(max_workers=max(1, min(len(cmds), os.cpu_count() or 1))) as pool:
        for res in pool.map(lambda c: subprocess.run(c, capture_output=True, text=True), cmds):
            sys.stdout.write(res.stdout)
            sys.stderr.write(res.stderr)
            if res.returncode != 0:
                raise subprocess.CalledProcessError(res.returncode, res.args, res.stdout, res.stderr)
    tmp = LIB_PATH + ".tmp"
    subprocess.run([nvcc(), *ARCH, "-shared", "-Xcompiler", "-fPIC", *objs, "-o", tmp], check=True)
    os.replace(tmp, LIB_PATH)
    return LIB_PATH


if __name__ == "__main__":
    build(force=True, ptxas_verbose="--verbose-ptxas" in sys.argv)
    print(LIB_PATH)
