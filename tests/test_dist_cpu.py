"""Multi-rank host logic of bench.py on CPU (gloo, world size 2).

The layer shards by batch: every rank runs its own sequences and no data-path
collective exists (weak scaling).  The only collectives are the barrier around the
timed region and the max over ranks of its duration; these tests run them on gloo.
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from selective_state_space_53_b200.inputs import SEEDS, config_inputs


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = 10.0 + 5.0 * rank                     # rank 1 is the slow one
        ms = bench.max_over_ranks(local_ms, world, device="cpu")
        seed = bench.rank_seed(SEEDS["p1_layer"], rank)
        inp = config_inputs("p1_layer", seed=seed, b=1, L=8)
        x0 = float(inp.x.reshape(-1)[0])
        t = torch.tensor([x0], dtype=torch.float64)
        gathered = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(gathered, t)
        dist.barrier()
        out[rank] = (ms, seed, [float(g.item()) for g in gathered])
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_time_and_independent_batches():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    ms0, seed0, xs0 = out[0]
    ms1, seed1, xs1 = out[1]
    assert ms0 == ms1 == 15.0                             # every rank reports the slowest rank
    assert seed0 != seed1                                 # each rank draws its own batch
    assert xs0 == xs1 and xs0[0] != xs0[1]


def test_job_throughput_counts_all_ranks():
    v1 = bench.job_throughput(8196, 10, 1, 5.0)
    v4 = bench.job_throughput(8196, 10, 4, 5.0)
    assert v4 == pytest.approx(4 * v1)
    assert v1 == pytest.approx(8196 * 10 / 5e-3)
