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
