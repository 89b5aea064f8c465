"""Build the qlinear shared library (sm_100a) in-tree with nvcc.

    python -m group_wise_affine_qlinear_b200.build [--verbose-ptxas]

The library is two CUDA translation units (csrc/ql_api.cu, which includes
every kernel header, and csrc/ql_noalloc.cu), linked with the static CUDA runtime so it loads without a GPU driver
present; the driver is only needed when a call is made.
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
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources() -> list[str]:
    d = os.path.join(HERE, "csrc")
    return sorted(os.path.join(d, f) for f in os.listdir(d) if f.endswith((".cu", ".cuh")))


def up_to_date() -> bool:
    if not os.path.exists(OUT):
        return False
    t = os.path.getmtime(OUT)
    deps = sources() + [os.path.join(ROOT, "include", "qlinear.h"), os.path.abspath(__file__)]
    return all(os.path.getmtime(s) <= t for s in deps)


def build(force: bool = False, verbose_ptxas: bool = False, extra: list[str] | None = None) -> str:
    if not force and up_to_date():
        return OUT
    cmd = [nvcc_path(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
           "-Xcompiler", "-fvisibility=hidden", "--cudart", "static",
           "-I", os.path.join(ROOT, "include"), *SRCS, "-o", OUT + ".tmp"]
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
    os.replace(OUT + ".tmp", OUT)
    return OUT


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--verbose-ptxas", action="store_true")
    ap.add_argument("--force", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force or a.verbose_ptxas, verbose_ptxas=a.verbose_ptxas))
