"""The dispatcher's per-shape choice on a B200, read from qlinear_last_dispatch after real calls.

The table is the one the CPU test reads through the workspace sizes (measured fastest configurations
of the text projection, the QKV projection and the MLP down projection); here the calls run, so the
record also shows the launch shape and the reason.  Values are zeros: parity of every path and split
is covered by the parity files.
"""
import pytest
import torch

import group_wise_affine_qlinear_b200 as ql

from .test_abi_host import DISPATCH_TABLE

pytestmark = pytest.mark.gpu

_NAMES = {ql.PATH_TC_SKINNY: "tc_skinny", ql.PATH_TC_FUSED: "tc_fused"}
_WEIGHTS = {}


def _weights(K, N):
    if (K, N) not in _WEIGHTS:
        _WEIGHTS.clear()
        _WEIGHTS[(K, N)] = (torch.zeros((N, K // 8), dtype=torch.int32, device="cuda"),
                            torch.zeros((N, K // 64), dtype=torch.float16, device="cuda"),
                            torch.zeros((N, K // 64), dtype=torch.float16, device="cuda"))
    return _WEIGHTS[(K, N)]


@pytest.mark.parametrize("M,K,N,path,split", DISPATCH_TABLE)
def test_dispatcher_choice(M, K, N, path, split):
    c, s, b = _weights(K, N)
    x = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    y = ql.forward(x, c, s, b)
    d = ql.last_dispatch()
    assert d.startswith(f"path={_NAMES[path]} "), d
    assert "why=auto" in d, d
    if path == ql.PATH_TC_FUSED:
        assert f"splitk={split} " in d, d
    else:
        assert f"nt={16 if M <= 16 else 32 if M <= 32 else 64} " in d, d
    assert not torch.any(y != 0)
    assert ql.device_status() == 0
