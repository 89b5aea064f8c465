"""Failure detection without a fault: a bounded wait inside a kernel gives up after the library's
limit, reports QL_ERR_DEVICE_TIMEOUT through the device status word, and leaves the context usable.
The wait is on a barrier that nothing completes (qlinear_selftest_bounded_wait); no trap, assert,
bad address or endless loop is involved."""
import time

import numpy as np
import pytest
import torch

import group_wise_affine_qlinear_b200 as ql
from oracle import qlinear_oracle as O

from ._helpers import bf16_bits, random_layer, to_dev_bf16, to_dev_codes, to_dev_f16

pytestmark = pytest.mark.gpu


def test_bounded_wait_expires_reports_and_recovers():
    if not torch.cuda.is_available():
        pytest.fail("CUDA GPU required for -m gpu tests")
    assert ql.device_status() == 0
    t0 = time.perf_counter()
    ql.selftest_bounded_wait()
    status = ql.device_status()            # synchronizes the stream, then reads and clears
    elapsed = time.perf_counter() - t0
    assert status == 6, status             # QL_ERR_DEVICE_TIMEOUT
    assert 0.5 < elapsed < 60.0, elapsed   # the limit is one second
    assert ql.device_status() == 0
    # the context still runs the layer
    rng = np.random.default_rng(99)
    x, codes, s, b = random_layer(rng, 64, 512, 136)
    y = ql.forward(to_dev_bf16(x), to_dev_codes(codes), to_dev_f16(s), to_dev_f16(b))
    t = O.tolerance(O.decode_bf16(bf16_bits(y)), O.forward_ref(x, codes, s, b))
    assert t["ok"], t
    assert ql.device_status() == 0


# ---------------------------------------------------------------- expiring waits inside the real pipelines

def _checked_library():
    from group_wise_affine_qlinear_b200 import build as qb
    return ql.load_library(qb.build(bounds_check=True))


@pytest.mark.parametrize("path,bit", [(ql.PATH_TC_FUSED, 1), (ql.PATH_TC_SKINNY, 2)])
def test_pipeline_unwinds_when_its_code_producer_is_held_back(path, bit):
    """The checked build holds back the code producer of one tensor-core kernel, so no code load (and
    hence no MMA on codes) is ever in flight: every other role's bounded wait must expire within the
    shortened limit, the call must report QL_ERR_DEVICE_TIMEOUT, and the CTAs must have freed their
    tensor memory and abandoned nothing, which the next, normal call on the same library shows by
    matching the oracle."""
    import ctypes

    Lc = _checked_library()
    rng = np.random.default_rng(40 + bit)
    M, K, N = 16, 1024, 264
    x, codes, s, b = random_layer(rng, M, K, N)
    xd, cd, sd, bd = to_dev_bf16(x), to_dev_codes(codes), to_dev_f16(s), to_dev_f16(b)
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    ws_bytes = Lc.qlinear_workspace_size_config(M, K, N, 64, path, 0)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device="cuda")
    st = torch.cuda.current_stream().cuda_stream

    def call():
        return Lc.qlinear_forward_config(xd.data_ptr(), cd.data_ptr(), sd.data_ptr(), bd.data_ptr(), y.data_ptr(),
                                         1, M, K, N, 64, path, 0, ws.data_ptr(), ws.numel(), ctypes.c_void_p(st))

    assert Lc.qlinear_get_device_status(ctypes.c_void_p(st)) == 0
    limit_ns = 20_000_000                                     # 20 ms
    assert Lc.qlinear_test_stall(bit, limit_ns) == 0
    try:
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        assert call() == 0
        status = Lc.qlinear_get_device_status(ctypes.c_void_p(st))
        elapsed = time.perf_counter() - t0
    finally:
        assert Lc.qlinear_test_stall(0, 1_000_000_000) == 0
    assert status == 6, status                                # QL_ERR_DEVICE_TIMEOUT
    assert elapsed < 0.9, elapsed                             # the shortened limit, not the default second
    torch.cuda.synchronize()
    assert Lc.qlinear_get_device_status(ctypes.c_void_p(st)) == 0
    for _ in range(2):                                        # the next calls run normally
        y.fill_(float("nan"))
        assert call() == 0
        assert Lc.qlinear_get_device_status(ctypes.c_void_p(st)) == 0
        t = O.tolerance(O.decode_bf16(bf16_bits(y)), O.forward_ref(x, codes, s, b))
        assert t["ok"], t
