"""The layer inside a CUDA graph: a captured call replays to the bytes of a direct call.

Serving loops capture decode-sized layers once and replay them; the capture must hold every launch of the
call (the prepass, the main kernel and the ordered sum, chained by programmatic dependent launch) with the
call's buffers, and the library must do nothing at call time that a capture cannot record.
"""
import numpy as np
import pytest
import torch

import group_wise_affine_qlinear_b200 as ql
from oracle import qlinear_oracle as O

from ._helpers import (FUSED_TILE_TOKENS, bf16_bits, random_layer, random_layer8, sample_rows, to_dev_bf16,
                       to_dev_codes, to_dev_f16)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,K,N,path,split", [
    (1, 8192, 1032, ql.PATH_AUTO, 0),            # weight streaming
    (24, 4160, 264, ql.PATH_TC_SKINNY, 0),       # weight streaming, scales and biases not TMA-aligned
    (300, 2048, 776, ql.PATH_AUTO, 0),           # fused, the dispatcher's split
    (200, 8192, 1024, ql.PATH_TC_FUSED, 4),      # fused split-K: four launches
])
def test_graph_replay_matches_direct_call(M, K, N, path, split):
    if not torch.cuda.is_available():
        pytest.fail("CUDA GPU required for -m gpu tests")
    rng = np.random.default_rng(M * 13 + K)
    x, codes, s, b = random_layer(rng, M, K, N)
    xd, cd, sd, bd = to_dev_bf16(x), to_dev_codes(codes), to_dev_f16(s), to_dev_f16(b)
    ws = torch.empty(max(ql.workspace_size(M, K, N, path, split), 16), dtype=torch.uint8, device="cuda")
    y_direct = ql.forward(xd, cd, sd, bd, workspace=ws, path=path, split_k=split)
    torch.cuda.synchronize()
    ref = bf16_bits(y_direct)

    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        ql.forward(xd, cd, sd, bd, out=y, workspace=ws, path=path, split_k=split)
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        ql.forward(xd, cd, sd, bd, out=y, workspace=ws, path=path, split_k=split)
    for _ in range(3):
        y.fill_(float("nan"))
        ws.fill_(0xFF)                                  # nothing of a previous replay may be reused
        g.replay()
        torch.cuda.synchronize()
        assert np.array_equal(bf16_bits(y), ref)
    assert ql.device_status() == 0
    rows = sample_rows(M, n_random=8, seed=M, tile=FUSED_TILE_TOKENS)
    t = O.tolerance(O.decode_bf16(ref[rows]), O.forward_rows(x, codes, s, b, rows))
    assert t["ok"], t
    del g


def _capture(fn):
    """fn() once on a side stream, then captured; returns the graph."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fn()
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


@pytest.mark.parametrize("M,K,N,path", [(8, 4096, 520, ql.PATH_AUTO), (300, 2048, 776, ql.PATH_AUTO)])
def test_graph_replay_8bit_codes(M, K, N, path):
    rng = np.random.default_rng(M * 17 + K)
    x, codes, s, b = random_layer8(rng, M, K, N)
    xd, cd, sd, bd = to_dev_bf16(x), to_dev_codes(codes), to_dev_f16(s), to_dev_f16(b)
    ws = torch.empty(max(ql.workspace_size(M, K, N, path, 0, bits=8), 16), dtype=torch.uint8, device="cuda")
    ref = bf16_bits(ql.forward8(xd, cd, sd, bd, workspace=ws, path=path))
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    g = _capture(lambda: ql.forward8(xd, cd, sd, bd, out=y, workspace=ws, path=path))
    for _ in range(2):
        y.fill_(float("nan"))
        ws.fill_(0xFF)
        g.replay()
        torch.cuda.synchronize()
        assert np.array_equal(bf16_bits(y), ref)
    assert ql.device_status() == 0
    del g


def test_graph_replay_swiglu_pair():
    rng = np.random.default_rng(77)
    M, K, I = 300, 1024, 264
    x, gc, gs, gb = random_layer(rng, M, K, I)
    _, uc, us, ub = random_layer(rng, 1, K, I)
    xd = to_dev_bf16(x)
    gate = (to_dev_codes(gc), to_dev_f16(gs), to_dev_f16(gb))
    up = (to_dev_codes(uc), to_dev_f16(us), to_dev_f16(ub))
    ws = torch.empty(max(ql.swiglu_workspace_size(M, K, I), 16), dtype=torch.uint8, device="cuda")
    ref = bf16_bits(ql.swiglu(xd, gate, up, workspace=ws))
    h = torch.empty((M, I), dtype=torch.bfloat16, device="cuda")
    g = _capture(lambda: ql.swiglu(xd, gate, up, out=h, workspace=ws))
    for _ in range(2):
        h.fill_(float("nan"))
        ws.fill_(0xFF)
        g.replay()
        torch.cuda.synchronize()
        assert np.array_equal(bf16_bits(h), ref)
    assert ql.device_status() == 0
    del g
