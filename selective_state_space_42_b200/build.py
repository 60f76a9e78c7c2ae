"""Builds libselscan.so in-tree with nvcc for sm_100a.

    python -m selective_state_space_42_b200.build        # or build() from Python

Each CUDA source compiles to its own object (in parallel, under ``_build/``
next to this file), and the objects link into the shared library, which lands
next to this file so that the binding finds it and the built file travels
with the source tree.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_PATH = os.path.join(HERE, "libselscan.so")
OBJ_DIR = os.path.join(HERE, "_build")
SOURCES = ["api.cu", "scan.cu", "scan_tma.cu", "scan_wide.cu", "scan_bwd.cu", "scan_bwd2.cu", "ssd.cu", "ssd_tc.cu",
           "state_update.cu", "noalloc.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"),
                 "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _headers() -> list:
    hs = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]
    hs += [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE)]
    hs.append(os.path.abspath(__file__))
    return hs


def _newer(deps, out: str) -> bool:
    if not os.path.exists(out):
        return True
    mt = os.path.getmtime(out)
    return any(os.path.getmtime(d) > mt for d in deps)


def _flags(extra) -> list:
    return [*ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC",
            "-Xcompiler", "-fvisibility=hidden", "--expt-relaxed-constexpr",
            "-I", INCLUDE, "-I", CSRC, *extra]


def build(force: bool = False, verbose: bool = False, extra=(), out: str = LIB_PATH,
          obj_dir: str = OBJ_DIR, jobs: int = 0) -> str:
    """Compiles the sources that changed (all of them with ``force``) and links
    ``out``. ``extra`` flags go to every compile; a different ``obj_dir``
    keeps the objects of a differently configured build apart."""
    os.makedirs(obj_dir, exist_ok=True)
    headers = _headers()
    flags = _flags(extra)
    objs, todo = [], []
    for s in SOURCES:
        src = os.path.join(CSRC, s)
        obj = os.path.join(obj_dir, s[:-3] + ".o")
        objs.append(obj)
        if force or _newer([src, *headers], obj):
            todo.append((src, obj))

    def compile_one(item):
        src, obj = item
        tmp = obj + f".tmp{os.getpid()}"
        cmd = [nvcc(), *flags, "-c", "-o", tmp, src]
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.run(cmd, check=True)
        os.replace(tmp, obj)

    if todo:
        n = jobs or min(len(todo), os.cpu_count() or 1)
        with ThreadPoolExecutor(max_workers=n) as ex:
            for f in [ex.submit(compile_one, t) for t in todo]:
                f.result()
    if todo or force or _newer(objs, out):
        tmp = out + f".tmp{os.getpid()}"
        cmd = [nvcc(), *ARCH, "-shared", "-o", tmp, *objs, "-lcudart"]
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.run(cmd, check=True)
        os.replace(tmp, out)
    return out


if __name__ == "__main__":
    args = sys.argv[1:]
    build(force=True, verbose=True,
          extra=["-Xptxas", "-v"] if "--ptxas-v" in args else [])
    print(LIB_PATH)
