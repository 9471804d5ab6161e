"""Builds the in-tree shared libraries with nvcc for sm_100a.

* ``libdcu.so``    -- the DCU kernels and the C ABI of ``include/dcu.h``.
* ``libdcugen.so`` -- the device side of the seeded input generator.

Run ``python -m dynamic_layer_wise_b200.build`` (or ``__graft_entry__.build()``).
Objects go to ``_build/``; a source is recompiled when it or any header is
newer than its object.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(ROOT, "_build")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
         "-Xcompiler", "-Wall", "-Xcompiler", "-Wno-unknown-pragmas"]
GEN_SOURCES = ["gen.cu"]


def nvcc() -> str:
    p = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(p):
        raise RuntimeError("nvcc not found")
    return p


def _headers() -> list[str]:
    return (glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
            + glob.glob(os.path.join(ROOT, "include", "*.h")))


def _stale(obj: str, src: str, deps: list[str]) -> bool:
    if not os.path.exists(obj):
        return True
    t = os.path.getmtime(obj)
    return any(os.path.getmtime(p) > t for p in [src] + deps)


def _compile(src: str, extra: list[str]) -> str:
    obj = os.path.join(BUILD, os.path.basename(src) + ".o")
    if _stale(obj, src, _headers()):
        cmd = [nvcc(), *ARCH, *FLAGS, *extra, "-c", src, "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    return obj


def _link(objs: list[str], out: str) -> None:
    if os.path.exists(out) and all(os.path.getmtime(o) <= os.path.getmtime(out) for o in objs):
        return
    cmd = [nvcc(), *ARCH, "-shared", "-o", out + ".tmp", *objs]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed for {out}:\n{r.stdout}\n{r.stderr}")
    os.replace(out + ".tmp", out)


def build_all(verbose: bool = False, extra: list[str] | None = None) -> dict:
    os.makedirs(BUILD, exist_ok=True)
    extra = extra or []
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    dcu_srcs = [s for s in srcs if os.path.basename(s) not in GEN_SOURCES]
    gen_srcs = [s for s in srcs if os.path.basename(s) in GEN_SOURCES]
    with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 4)) as ex:
        objs = list(ex.map(lambda s: _compile(s, extra), dcu_srcs + gen_srcs))
    dcu_objs, gen_objs = objs[:len(dcu_srcs)], objs[len(dcu_srcs):]
    out = {"dcu": os.path.join(PKG, "libdcu.so"), "gen": os.path.join(PKG, "libdcugen.so")}
    _link(dcu_objs, out["dcu"])
    _link(gen_objs, out["gen"])
    if verbose:
        print("built", out)
    return out


if __name__ == "__main__":
    build_all(verbose=True, extra=sys.argv[1:])
