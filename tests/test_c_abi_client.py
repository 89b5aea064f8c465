"""The boundary is a C ABI: a C99 program compiles against include/qlinear.h, links libqlinear.so and
gets the documented argument errors without a GPU."""
import os
import shutil
import subprocess

import pytest

from group_wise_affine_qlinear_b200 import build as qb

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _cuda_include():
    for d in (os.environ.get("CUDA_HOME", ""), "/usr/local/cuda"):
        if d and os.path.exists(os.path.join(d, "include", "cuda_runtime_api.h")):
            return os.path.join(d, "include")
    return None


def test_c_client_compiles_links_and_runs(tmp_path):
    cc = shutil.which("gcc") or shutil.which("cc")
    inc = _cuda_include()
    if cc is None or inc is None:
        pytest.skip("no C compiler or CUDA headers")
    lib = qb.build()
    exe = tmp_path / "abi_client"
    cmd = [cc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), "-I", inc,
           os.path.join(ROOT, "tests", "c", "abi_client.c"), "-o", str(exe), lib, f"-Wl,-rpath,{os.path.dirname(lib)}"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "c abi client ok" in r.stdout
