"""Builds libeta.so (the ETA C-ABI library) in-tree for sm_100a with nvcc.

    python -m long_context_decoding_eta_b200.build [--verbose] [--checked]

Objects are compiled in parallel into `_build/` next to this file and linked
into `long_context_decoding_eta_b200/libeta.so`.  Rebuilds only what changed.
`--checked` builds the range-checked debugging variant instead (-DETA_CHECKED,
objects in `_build_checked/`, library `libeta_checked.so`), which the binding
loads when the environment sets ETA_CHECKED=1.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libeta.so")
BUILD_CHECKED = os.path.join(HERE, "_build_checked")
LIB_CHECKED = os.path.join(HERE, "libeta_checked.so")
INCLUDE = os.path.join(ROOT, "include")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
CUFLAGS = ["-O3", "-std=c++17", "-lineinfo", "--expt-relaxed-constexpr",
           "-Xcompiler", "-fPIC", "-I", INCLUDE]


def _sources():
    cu = sorted(f for f in os.listdir(CSRC) if f.endswith(".cu"))
    cpp = sorted(f for f in os.listdir(CSRC) if f.endswith(".cpp"))
    return cu, cpp


def _headers_mtime():
    hs = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]
    hs.append(os.path.join(INCLUDE, "eta.h"))
    return max(os.path.getmtime(h) for h in hs)


def _compile(src: str, verbose: bool, checked: bool = False):
    path = os.path.join(CSRC, src)
    obj = os.path.join(BUILD_CHECKED if checked else BUILD, src + ".o")
    if (os.path.exists(obj) and os.path.getmtime(obj) >= os.path.getmtime(path)
            and os.path.getmtime(obj) >= _headers_mtime()):
        return obj, ""
    extra = ["-DETA_CHECKED"] if checked else []
    cmd = [NVCC, *ARCH, *CUFLAGS, *extra, "-c", path, "-o", obj]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    p = subprocess.run(cmd, capture_output=True, text=True)
    if p.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{p.stdout}\n{p.stderr}")
    return obj, p.stdout + p.stderr


def build(verbose: bool = False, checked: bool = False) -> str:
    """Builds libeta.so, or libeta_checked.so with checked=True; returns its path."""
    lib_path = LIB_CHECKED if checked else LIB
    os.makedirs(BUILD_CHECKED if checked else BUILD, exist_ok=True)
    cu, cpp = _sources()
    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        futs = [ex.submit(_compile, s, verbose, checked) for s in cu + cpp]
        objs = []
        for f in futs:
            obj, log = f.result()
            objs.append(obj)
            if verbose and log:
                print(log)
    newest = max(os.path.getmtime(o) for o in objs)
    if not os.path.exists(lib_path) or os.path.getmtime(lib_path) < newest:
        cmd = [NVCC, *ARCH, "-shared", "-o", lib_path, *objs, "-lcudart"]
        p = subprocess.run(cmd, capture_output=True, text=True)
        if p.returncode != 0:
            raise RuntimeError(f"link failed:\n{p.stdout}\n{p.stderr}")
    return lib_path


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--checked", action="store_true")
    a = ap.parse_args()
    print(build(a.verbose, a.checked))
    sys.exit(0)
