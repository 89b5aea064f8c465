"""Build the qlinear shared library (sm_100a) in-tree with nvcc.

    python -m group_wise_affine_qlinear_b200.build [--verbose-ptxas] [--bounds-check]

The library is two CUDA translation units (csrc/ql_api.cu, which includes
every kernel header, and csrc/ql_noalloc.cu), linked with the static CUDA runtime so it loads without a GPU driver
present; the driver is only needed when a call is made.

--bounds-check builds libqlinear_bounds.so with QL_BOUNDS_CHECK: the kernels' computed global indices
are checked against their extents, and a bad one records QL_ERR_BOUNDS in the device status word
instead of being accessed.  It stands in for a memory checker.  Run any caller against it by setting
QL_LIBRARY to its path.
"""
from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRCS = [os.path.join(HERE, "csrc", f) for f in ("ql_api.cu", "ql_noalloc.cu")]
OUT = os.path.join(HERE, "libqlinear.so")
OUT_BOUNDS = os.path.join(HERE, "libqlinear_bounds.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources() -> list[str]:
    d = os.path.join(HERE, "csrc")
    return sorted(os.path.join(d, f) for f in os.listdir(d) if f.endswith((".cu", ".cuh")))


def up_to_date(out: str = OUT) -> bool:
    if not os.path.exists(out):
        return False
    t = os.path.getmtime(out)
    deps = sources() + [os.path.join(ROOT, "include", "qlinear.h"), os.path.abspath(__file__)]
    return all(os.path.getmtime(s) <= t for s in deps)


def build(force: bool = False, verbose_ptxas: bool = False, extra: list[str] | None = None,
          bounds_check: bool = False) -> str:
    out = OUT_BOUNDS if bounds_check else OUT
    if not force and up_to_date(out):
        return out
    cmd = [nvcc_path(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
           "-Xcompiler", "-fvisibility=hidden", "--cudart", "static",
           "-I", os.path.join(ROOT, "include"), *SRCS, "-o", out + ".tmp"]
    if bounds_check:
        cmd.insert(1, "-DQL_BOUNDS_CHECK")
    if verbose_ptxas:
        cmd.insert(1, "-Xptxas=-v")
    if extra:
        cmd[1:1] = extra
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("nvcc failed building libqlinear.so")
    if verbose_ptxas:
        sys.stderr.write(r.stderr)
    os.replace(out + ".tmp", out)
    return out


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--verbose-ptxas", action="store_true")
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--bounds-check", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force or a.verbose_ptxas, verbose_ptxas=a.verbose_ptxas, bounds_check=a.bounds_check))
