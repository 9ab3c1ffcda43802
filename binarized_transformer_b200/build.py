"""Compile the CUDA sources into in-tree shared libraries for sm_100a.

libbwta.so            the product: kernels + the C ABI of include/bwta.h
libbwta_microbench.so instruction-rate / bandwidth microbenchmarks used to
                      state the roofline of the bit GEMM
Objects go to _build/ (not committed); the .so files sit next to this file so
that they travel with the source tree.
"""
from __future__ import annotations

import concurrent.futures as cf
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(HERE, "libbwta.so")
MB_LIB = os.path.join(HERE, "libbwta_microbench.so")

NVCC = os.environ.get("NVCC", "nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
                "-I", os.path.join(ROOT, "include")]

LIB_SOURCES = ["pack.cu", "gemm.cu", "decode.cu", "gemm_tc.cu", "attn.cu", "billm.cu", "billm_tc.cu",
               "abi.cu"]
MB_SOURCES = ["microbench.cu"]
HEADERS = ["common.cuh", "tma.cuh", "quant.cuh", "tcgen05.cuh"]


def _mtime(p):
    return os.path.getmtime(p) if os.path.exists(p) else -1.0


def _deps_mtime():
    paths = [os.path.join(CSRC, h) for h in HEADERS] + [os.path.join(ROOT, "include", "bwta.h")]
    return max(_mtime(p) for p in paths)


def _compile(src, obj, verbose):
    cmd = [NVCC] + FLAGS + ["-c", os.path.join(CSRC, src), "-o", obj]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
    return r.stderr


def _link(objs, out):
    tmp = out + ".tmp"
    cmd = [NVCC] + ARCH + ["-shared", "-o", tmp] + objs
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed for {out}:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, out)


def _build_lib(sources, out, force, verbose):
    os.makedirs(BUILD, exist_ok=True)
    dep = _deps_mtime()
    objs, todo = [], []
    for s in sources:
        obj = os.path.join(BUILD, s.replace(".cu", ".o"))
        objs.append(obj)
        if force or _mtime(obj) < max(_mtime(os.path.join(CSRC, s)), dep):
            todo.append((s, obj))
    if todo:
        with cf.ThreadPoolExecutor(max_workers=min(8, len(todo))) as ex:
            logs = list(ex.map(lambda t: _compile(t[0], t[1], verbose), todo))
        if verbose:
            for (s, _), log in zip(todo, logs):
                print(f"== {s}\n{log}")
    if force or todo or _mtime(out) < max(_mtime(o) for o in objs):
        _link(objs, out)
    return out


def build(force: bool = False, verbose: bool = False) -> None:
    _build_lib(LIB_SOURCES, LIB, force, verbose)
    _build_lib(MB_SOURCES, MB_LIB, force, verbose)


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
    print(MB_LIB)
