"""Builds libkvsparse.so in-tree with nvcc for sm_100a.

    python -m weighted_coreset_softmax_b200.build [--force]

Each translation unit compiles to _build/<name>.o (in parallel); the shared
library links the CUDA runtime statically, so loading it needs only the driver.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libkvsparse.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC",
         "-Xptxas", "-warn-spills", "-I", INCLUDE, "-I", CSRC]


def _nvcc():
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _newest(paths):
    return max(os.path.getmtime(p) for p in paths)


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False) -> str:
    sources = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    headers = sorted(glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
                     + glob.glob(os.path.join(INCLUDE, "*.h")))
    os.makedirs(BUILD, exist_ok=True)
    nvcc = _nvcc()
    hdr_time = _newest(headers) if headers else 0.0

    def deps_of(obj):
        """Headers the object was built from (nvcc's -MD file), or None."""
        dep = obj[:-2] + ".d"
        if not os.path.exists(dep):
            return None
        with open(dep) as f:
            text = f.read().replace("\\\n", " ")
        parts = text.split(":", 1)
        if len(parts) != 2:
            return None
        # the repository's own headers only (system headers belong to the image)
        return [t for t in parts[1].split() if t.endswith((".h", ".cuh")) and (
            os.path.realpath(t).startswith(os.path.realpath(CSRC)) or
            os.path.realpath(t).startswith(os.path.realpath(INCLUDE)))]

    def compile_one(src):
        obj = os.path.join(BUILD, os.path.basename(src)[:-3] + ".o")
        if not force and os.path.exists(obj):
            deps = deps_of(obj)
            newest = max([os.path.getmtime(src)] + ([os.path.getmtime(d) for d in deps if os.path.exists(d)]
                                                    if deps is not None else [hdr_time]))
            if os.path.getmtime(obj) >= newest:
                return obj, ""
        cmd = [nvcc, *ARCH, *FLAGS, "-MD", "-MF", obj[:-2] + ".d", "-c", src, "-o", obj]
        if ptxas_info:
            cmd[1:1] = ["-Xptxas", "-v"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
        return obj, r.stdout + r.stderr

    with cf.ThreadPoolExecutor(max_workers=max(1, min(len(sources), os.cpu_count() or 4))) as ex:
        results = list(ex.map(compile_one, sources))
    objs = [o for o, _ in results]
    logs = "".join(l for _, l in results)
    if verbose and logs:
        print(logs)
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < _newest(objs):
        cmd = [nvcc, *ARCH, "-shared", "-cudart", "static", "-o", LIB, *objs]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose=True, ptxas_info=a.ptxas_info))
    sys.exit(0)
