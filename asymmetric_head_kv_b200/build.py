"""Builds libdiffqkv.so in-tree with nvcc for sm_100a (B200).

Usage: ``python -m asymmetric_head_kv_b200.build`` (or ``build()`` from Python).
Each .cu file under csrc/ compiles to an object in _build/ (in parallel) and
they link into asymmetric_head_kv_b200/libdiffqkv.so.  Recompiles only what
changed (source or any header newer than its object).
"""
from __future__ import annotations

import concurrent.futures
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libdiffqkv.so")
LIB_CHECKED = os.path.join(PKG, "libdiffqkv_checked.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH + [
    "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
    "-I" + os.path.join(ROOT, "include"), "-Xptxas", "-warn-spills",
]


def _nvcc() -> str:
    p = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(p):
        raise RuntimeError("nvcc not found")
    return p


def _headers():
    return glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(ROOT, "include", "*.h"))


def _compile(src: str, obj: str, extra) -> str:
    cmd = [_nvcc()] + NVCC_FLAGS + list(extra) + ["-c", src, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {os.path.basename(src)}:\n{r.stdout}\n{r.stderr}")
    return r.stderr


def _build_one(lib: str, objdir: str, force: bool, verbose: bool, extra_flags) -> str:
    os.makedirs(objdir, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    hdr_mtime = max([os.path.getmtime(h) for h in _headers()] + [os.path.getmtime(__file__)])
    jobs = []
    objs = []
    for s in srcs:
        o = os.path.join(objdir, os.path.basename(s)[:-3] + ".o")
        objs.append(o)
        if force or not os.path.exists(o) or os.path.getmtime(o) < max(os.path.getmtime(s), hdr_mtime):
            jobs.append((s, o))
    if jobs:
        with concurrent.futures.ThreadPoolExecutor(max_workers=min(len(jobs), os.cpu_count() or 4)) as ex:
            for (s, _), log in zip(jobs, ex.map(lambda j: _compile(j[0], j[1], extra_flags), jobs)):
                if verbose and log.strip():
                    print(f"[{os.path.basename(s)}]\n{log}", file=sys.stderr)
    if jobs or not os.path.exists(lib):
        tmp = lib + f".tmp{os.getpid()}"
        cmd = [_nvcc()] + ARCH + ["-shared", "-o", tmp] + objs + ["-lcudart"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
        os.replace(tmp, lib)
    return lib


def build(force: bool = False, verbose: bool = False, extra_flags=(), checked: bool = True) -> str:
    """Builds libdiffqkv.so and, unless checked=False, libdiffqkv_checked.so: the same sources with
    -DDIFFQKV_BOUNDS_CHECK (device-side index checks; selected at run time by DIFFQKV_BOUNDS_CHECK=1)."""
    lib = _build_one(LIB, BUILD, force, verbose, extra_flags)
    if checked:
        _build_one(LIB_CHECKED, BUILD + "_checked", force, verbose, tuple(extra_flags) + ("-DDIFFQKV_BOUNDS_CHECK",))
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
