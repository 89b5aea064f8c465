"""The row-parallel exchange with two ranks on CPU (gloo): every rank receives all partials in rank
order, and their ordered sum is the whole layer.  The per-rank partials come from the oracle here;
on GPUs the same gather feeds qlinear_reduce_partials."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from group_wise_affine_qlinear_b200 import tp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    from oracle import qlinear_oracle as O
    from tests._helpers import random_layer
    from datetime import timedelta
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=timedelta(seconds=60))
    try:
        rng = np.random.default_rng(74)                       # the same layer on every rank
        x, codes, s, b = random_layer(rng, 6, 512, 32)
        t = lambda a: torch.from_numpy(np.ascontiguousarray(a))  # noqa: E731

        def partial(r):
            sh = tp.row_shard(t(codes.view(np.int32)), t(s), t(b), r, world)
            xr = tp.input_shard(t(x.view(np.int16)), r, world).numpy().view(np.uint16)
            c, sc, bi = sh
            return torch.from_numpy(O.forward_ref(xr, c.numpy().view(np.uint32), sc.numpy(), bi.numpy())
                                    .astype(np.float32))

        mine = partial(rank)
        got = tp.gather_partials(mine)
        assert got.shape == (world, 6, 32)
        for r in range(world):
            assert torch.equal(got[r], partial(r)), r        # rank order
        y = O.forward_ref(x, codes, s, b)
        tot = got.double().sum(0).numpy()
        assert np.max(np.abs(tot - y)) <= 1e-5 * np.sqrt(np.mean(y * y))
    finally:
        dist.destroy_process_group()


def test_row_parallel_gather_two_ranks():
    mp.spawn(_rank_main, args=(2, _free_port()), nprocs=2, join=True)


def _rank_leaves(rank, world, port, result_dir):
    from datetime import timedelta
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=timedelta(seconds=10))
    if rank == 1:
        return                                  # leaves between steps: never joins the gather
    outcome = "returned"
    try:
        tp.gather_partials(torch.zeros(4, 8))
    except Exception as exc:                    # noqa: BLE001
        outcome = "raised " + type(exc).__name__
    with open(os.path.join(result_dir, "rank0"), "w") as f:
        f.write(outcome)


def test_row_parallel_gather_fails_when_a_rank_leaves(tmp_path):
    """A rank that leaves before the exchange ends the other rank's gather with an error (no hang)."""
    mp.spawn(_rank_leaves, args=(2, _free_port(), str(tmp_path)), nprocs=2, join=True)
    assert (tmp_path / "rank0").read_text().startswith("raised ")
