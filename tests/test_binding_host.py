"""The Python binding on a host without a GPU: every entry refuses host tensors with an error (there is no
CPU fallback), and a missing library is a loud error, not a silent substitute."""
import os
import subprocess
import sys

import pytest
import torch

import group_wise_affine_qlinear_b200 as ql

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _w4(N=64, K=256):
    return (torch.zeros((N, K // 8), dtype=torch.int32), torch.zeros((N, K // 64), dtype=torch.float16),
            torch.zeros((N, K // 64), dtype=torch.float16))


def test_host_tensors_are_refused():
    x = torch.zeros((4, 256), dtype=torch.bfloat16)
    c, s, b = _w4()
    c8 = torch.zeros((64, 64), dtype=torch.int32)
    for call in (lambda: ql.forward(x, c, s, b),
                 lambda: ql.forward8(x, c8, s, b),
                 lambda: ql.swiglu(x, (c, s, b), (c, s, b)),
                 lambda: ql.dequant(c, s, b),
                 lambda: ql.dequant8(c8, s, b),
                 lambda: ql.pack(torch.zeros((64, 256))),
                 lambda: ql.pack8(torch.zeros((64, 256))),
                 lambda: ql.reduce_partials(torch.zeros((2, 4, 8)))):
        with pytest.raises(ValueError, match="CUDA tensor"):
            call()


def test_missing_library_is_a_loud_error():
    env = dict(os.environ, QL_LIBRARY=os.path.join(ROOT, "no_such_dir", "libqlinear.so"))
    code = "import group_wise_affine_qlinear_b200 as ql; ql.lib()"
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode != 0
    assert "missing" in r.stderr
