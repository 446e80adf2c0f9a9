"""Data-parallel path of bench.py on the CPU: 2 gloo ranks.

Each rank holds half of the batch; the weight gradient is a sum over the
batch, so summing the ranks' gradients with bench.allreduce_weight_grads must
give the full-batch gradient (computed here by the oracle), and
bench.max_over_ranks must return the slowest rank's value.
"""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import oracle
from wtconv_inputs import Case, make_inputs

CASE = Case("dp_small", 4, 3, 16, 16, 3, 2, "f32", 77, "normal", "normal")
PARAMS = ("base_w", "base_b", "base_scale", "wt_w", "wt_scale")


def _grads(inp, b0, b1):
    orc = oracle.default()
    p = {k: inp[k].double().numpy() for k in PARAMS}
    return orc.backward_weight(inp["x"][b0:b1].double().numpy(), inp["dy"][b0:b1].double().numpy(), p["base_w"],
                               p["base_b"], p["base_scale"], p["wt_w"], p["wt_scale"], CASE.L)


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        inp = make_inputs(CASE)
        half = CASE.B // world
        local = {k: torch.from_numpy(v).float() for k, v in _grads(inp, rank * half, (rank + 1) * half).items()}
        flat = torch.empty(sum(v.numel() for v in local.values()))
        bench.allreduce_weight_grads(local, flat, dist)
        full = _grads(inp, 0, CASE.B)
        errs = {k: float(np.max(np.abs(local[k].double().numpy() - full[k])) / np.max(np.abs(full[k]))) for k in PARAMS}
        slowest = bench.max_over_ranks(float(rank + 1), dist, torch.device("cpu"))
        out[rank] = (errs, slowest)
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_rank_gradient_sum_and_max():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, join=True, start_method="spawn")
    assert len(out) == world
    for rank in range(world):
        errs, slowest = out[rank]
        assert slowest == float(world)
        for k, e in errs.items():
            assert e <= 1e-6, (rank, k, e)
