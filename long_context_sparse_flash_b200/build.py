"""Build libhs2.so (and its checked variant) in-tree with nvcc for sm_100a.

    python -m long_context_sparse_flash_b200.build [--force] [--jobs N]

Every .cu file under csrc/ is compiled to an object with
``-gencode arch=compute_100a,code=sm_100a -O3 -lineinfo`` and linked into
``libhs2.so``; the same sources compiled with ``-DHS2_CHECKED`` (device-side
input checks that report through the workspace error word) give
``libhs2_checked.so``.
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
CSRC = os.path.join(PKG, "csrc")
ROOT = os.path.dirname(PKG)
BUILD = os.path.join(ROOT, "_build")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
              "-Xptxas", "-warn-spills"]

LIBS = {"libhs2.so": [], "libhs2_checked.so": ["-DHS2_CHECKED"]}


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return _sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(ROOT, "include", "*.h"))


def _stale(target: str) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in _deps())


def _compile(src: str, obj: str, defs) -> None:
    cmd = [nvcc(), *ARCH, *NVCC_FLAGS, *defs, "-I", os.path.join(ROOT, "include"), "-c", src, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError(f"nvcc failed on {os.path.basename(src)}")
    if r.stderr.strip():
        sys.stderr.write(r.stderr)


def build(force: bool = False, jobs: int = 0) -> dict:
    os.makedirs(BUILD, exist_ok=True)
    out = {}
    todo = []
    for lib, defs in LIBS.items():
        target = os.path.join(PKG, lib)
        out[lib] = target
        if force or _stale(target):
            todo.append((lib, defs, target))
    if not todo:
        return out
    jobs = jobs or min(8, os.cpu_count() or 1)
    with cf.ThreadPoolExecutor(jobs) as ex:
        futs = []
        objs = {}
        for lib, defs, target in todo:
            tag = lib.replace(".so", "")
            objs[lib] = []
            for src in _sources():
                obj = os.path.join(BUILD, f"{tag}_{os.path.basename(src)}.o")
                objs[lib].append(obj)
                futs.append(ex.submit(_compile, src, obj, defs))
        for f in futs:
            f.result()
    for lib, defs, target in todo:
        tmp = target + f".tmp{os.getpid()}"
        cmd = [nvcc(), *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs[lib]]
        subprocess.run(cmd, check=True)
        os.replace(tmp, target)
    return out


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--jobs", type=int, default=0)
    a = ap.parse_args()
    for k, v in build(a.force, a.jobs).items():
        print(k, v)
