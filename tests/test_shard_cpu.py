"""Sequence sharding on CPU: two gloo ranks, each with one range of the same sequences.

The orchestration of ``selective_state_space_53_b200.shard.sharded_scan`` (summarise, all-gather
the summaries, fold the earlier ranges onto the initial state, scan the own range) runs over
operations built on the fp64 oracle; the concatenated outputs and the last rank's final state
must equal one oracle run over the whole sequences.  This pins the range algebra (the fold)
against the sequential recurrence and checks the exchange and its order.
"""

import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from selective_state_space_53_b200.inputs import make_inputs, make_state
from selective_state_space_53_b200.shard import all_gather_summaries, sharded_scan
from shard_oracle_ops import OracleOps, range_inputs
from oracle import oracle as orc

SHAPE = dict(b=2, L=90, H=4, P=8, N=8, R=2, G=2)
CUTS = [0, 37, 90]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _draw():
    inp = make_inputs(dtype="f32", seed=700, extras=True, **SHAPE)
    st = make_state(SHAPE["b"], SHAPE["H"], SHAPE["P"], SHAPE["N"], SHAPE["R"], seed=701)
    return inp, st


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        inp, st = _draw()
        mine = range_inputs(inp, CUTS[rank], CUTS[rank + 1])
        y, (h, cB, cx) = sharded_scan(OracleOps(), None, mine, st, rank, all_gather_summaries)
        out[rank] = (y, h, cB, cx)
    finally:
        dist.destroy_process_group()


def test_two_rank_sequence_sharding_equals_one_scan():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    inp, st = _draw()
    yr, hr, cBr, cxr = orc.scan_inputs(inp, h0=st[0], carry_B0=st[1], carry_x0=st[2])
    y = np.concatenate([out[0][0], out[1][0]], axis=1)
    np.testing.assert_allclose(y, yr, rtol=0, atol=1e-11 * np.abs(yr).max())
    np.testing.assert_allclose(out[1][1], hr, rtol=0, atol=1e-11 * np.abs(hr).max())
    np.testing.assert_array_equal(out[1][2], cBr)
    np.testing.assert_array_equal(out[1][3], cxr)
    # rank 0's own final state is the state after its range
    y0, h0, _, _ = orc.scan_inputs(range_inputs(inp, 0, CUTS[1]), h0=st[0], carry_B0=st[1], carry_x0=st[2])
    np.testing.assert_allclose(out[0][1], h0, rtol=0, atol=1e-12 * np.abs(h0).max())


def test_fold_of_many_ranges_equals_one_scan():
    # single process: five ranges of uneven length, summaries folded one range at a time
    inp, st = _draw()
    ops = OracleOps()
    cuts = [0, 1, 13, 14, 60, 90]
    summaries = [ops.summarise(None, range_inputs(inp, a, b)) for a, b in zip(cuts[:-1], cuts[1:])]
    every = {k: torch.stack([s[k] for s in summaries]) for k in summaries[0]}
    yr, hr, _, _ = orc.scan_inputs(inp, h0=st[0], carry_B0=st[1], carry_x0=st[2])
    for k in range(len(cuts) - 1):
        before = None if k == 0 else {n: v[:k] for n, v in every.items()}
        state = ops.fold(None, st, before, inp)
        y, _ = ops.scan(None, range_inputs(inp, cuts[k], cuts[k + 1]), state)
        np.testing.assert_allclose(y, yr[:, cuts[k]:cuts[k + 1]], rtol=0, atol=1e-11 * np.abs(yr).max())
