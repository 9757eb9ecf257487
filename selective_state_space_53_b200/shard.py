"""Sequence sharding: one batch of sequences split into consecutive token ranges, one range
per rank.

Each rank summarises its range (m3_scan_summary), the summaries are exchanged, every rank
folds the summaries of the ranges before its own onto the sequences' initial state
(m3_state_fold) and runs m3_scan_fwd over its range from the state it gets.  The scan is
associative over ranges (IBM Mamba page, hardware-aware scan), so the outputs equal one scan
over the whole sequences.  The exchange is one all-gather of the summaries (a few MiB per
rank), the only collective of the sharded path.

This module holds the orchestration only: argument marshalling, the exchange and the order
of the calls.  The arithmetic runs in libm3's kernels (``LibOps``); ``sharded_scan`` takes the
operations as an argument so that the same orchestration also runs over other operations (the
CPU tests pass ones built on the fp64 oracle).
"""

from __future__ import annotations

from . import m3

SUMMARY_KEYS = ("Z", "logdec", "angle", "bp_first", "carry_B", "carry_x")


class LibOps:
    """The three steps of a sharded scan on libm3 (device tensors, the current stream)."""

    def summarise(self, dims, dev):
        import torch
        b, H, N, P, R = dims.b, dims.H, dims.N, dims.P, dims.R
        d = dev["x"].device
        out = {
            "Z": torch.empty((b, H, N, P), dtype=torch.float32, device=d),
            "logdec": torch.empty((b, H), dtype=torch.float32, device=d),
            "angle": torch.empty((b, H, N // 2), dtype=torch.float64, device=d),
            "bp_first": torch.empty((b, H), dtype=torch.float32, device=d),
            "carry_B": torch.empty((b, H, R, N), dtype=torch.float32, device=d),
            "carry_x": torch.empty((b, H, P), dtype=torch.float32, device=d),
        }
        ws = torch.empty(max(m3.m3_scan_summary_workspace_size(dims), 16), dtype=torch.uint8, device=d)
        m3.m3_scan_summary(dims, dev["x"], dev["dt"], dev["A"], dev["lam"], dev["B"], dev["theta"], dev["bias_B"],
                           dev["W_x"], *[out[k] for k in SUMMARY_KEYS], ws)
        return out

    def fold(self, dims, state_tensors, before, dev):
        """Fold the stacked summaries `before` (leading axis: ranges in order) onto the state
        (h, carry_B, carry_x tensors, updated in place)."""
        n = 0 if before is None else int(before["logdec"].shape[0])
        st = m3.State.wrap(m3.make_dims(dims.b, 1, dims.H, dims.P, dims.N, dims.R, dims.G, dims.dtype),
                           *state_tensors)
        if n:
            m3.m3_state_fold(dims, n, *[before[k].contiguous() for k in SUMMARY_KEYS], dev["bias_B"], dev["W_x"], st)
        st.free()
        return state_tensors

    def scan(self, dims, dev, state_tensors):
        st = m3.State.wrap(dims, *state_tensors)
        y = m3.scan(dims, dev, st)
        st.free()
        return y, state_tensors


def all_gather_summaries(summary, group=None):
    """Every rank's summary, stacked along a new leading axis in rank order (torch.distributed)."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    out = {}
    for k in SUMMARY_KEYS:
        t = summary[k].contiguous()
        parts = [torch.empty_like(t) for _ in range(world)]
        dist.all_gather(parts, t, group=group)
        out[k] = torch.stack(parts)
    return out


def sharded_scan(ops, dims, dev, state_tensors, rank, exchange):
    """Scan this rank's range of every sequence.

    dims / dev: this rank's range (dims.L its length, dev its operands); state_tensors: the
    state entering range 0 (the sequences' initial state), overwritten with the state entering
    this range and then with the state after it; exchange(summary) returns the stacked
    summaries of all ranges in order.  Returns (y of this range, state_tensors)."""
    summary = ops.summarise(dims, dev)
    every = exchange(summary)
    before = None if rank == 0 else {k: v[:rank] for k, v in every.items()}
    state_tensors = ops.fold(dims, state_tensors, before, dev)
    return ops.scan(dims, dev, state_tensors)
