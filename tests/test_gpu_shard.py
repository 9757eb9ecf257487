"""Sequence sharding on the GPU: m3_scan_summary, m3_state_fold and m3_scan_fwd over consecutive
ranges of the same sequences, against one fp64 oracle run over the whole sequences.

The ranks of a sharded run are emulated in one process, one after another: every range is
summarised first (the summaries are independent), then each range folds the summaries before
it onto the initial state and scans from there.  No kernel waits on another range's kernel.
"""

import numpy as np
import pytest
import torch

from oracle import oracle as orc
from selective_state_space_53_b200 import m3
from selective_state_space_53_b200.inputs import make_inputs, make_state
from selective_state_space_53_b200.shard import LibOps
from shard_oracle_ops import range_inputs

pytestmark = pytest.mark.gpu

TOL = 2e-2


def rel_err(got, ref):
    return float(np.abs(np.asarray(got, np.float64) - ref).max() / max(np.abs(ref).max(), 1e-300))


@pytest.mark.parametrize("shape,cuts", [
    (dict(b=2, L=700, H=3, P=128, N=128, R=4, G=1), [0, 300, 333, 700]),
    (dict(b=1, L=3000, H=2, P=64, N=64, R=2, G=1), [0, 1000, 2999, 3000]),
    (dict(b=2, L=600, H=4, P=128, N=64, R=2, G=2), [0, 64, 600]),
], ids=["P128N128R4", "P64N64R2", "P128N64R2"])
def test_sharded_ranges_equal_one_scan(shape, cuts):
    inp = make_inputs(dtype="bf16", seed=710, extras=True, **shape)
    st = make_state(shape["b"], shape["H"], shape["P"], shape["N"], shape["R"], seed=711, scale=0.5)
    ops = LibOps()
    parts = [range_inputs(inp, a, b) for a, b in zip(cuts[:-1], cuts[1:])]
    devs = [m3.to_device(p) for p in parts]
    dims = [m3.dims_of(p) for p in parts]
    summaries = [ops.summarise(d, dv) for d, dv in zip(dims, devs)]
    every = {k: torch.stack([s[k] for s in summaries]) for k in summaries[0]}
    ys, last = [], None
    for k, (d, dv) in enumerate(zip(dims, devs)):
        state = tuple(torch.from_numpy(np.ascontiguousarray(a)).cuda() for a in st)
        before = None if k == 0 else {n: v[:k] for n, v in every.items()}
        ops.fold(d, state, before, dv)
        y, last = ops.scan(d, dv, state)
        ys.append(y.float())
    torch.cuda.synchronize()
    assert m3.m3_check() == 0
    y = torch.cat(ys, dim=1).cpu().numpy()
    yr, hr, cBr, cxr = orc.scan_inputs(inp, h0=st[0], carry_B0=st[1], carry_x0=st[2])
    ey, eh = rel_err(y, yr), rel_err(last[0].cpu().numpy(), hr)
    print(f"sharded {cuts}: y max rel {ey:.2e}, state max rel {eh:.2e}")
    assert ey < TOL and eh < TOL, (ey, eh)
    np.testing.assert_array_equal(last[1].cpu().numpy(), cBr.astype(np.float32))
    np.testing.assert_array_equal(last[2].cpu().numpy(), cxr.astype(np.float32))


def test_summary_rejects_unsupported_dims():
    d = m3.make_dims(1, 10, 2, 16, 16, 1, 1, "f32")
    with pytest.raises(m3.M3Error) as e:
        m3.m3_scan_summary_workspace_size(d)
    assert e.value.code == -8
