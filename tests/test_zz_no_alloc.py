"""m3_scan_fwd_noalloc, the prefill entry point for callers that cannot allocate.

Some callers cannot give the library a workspace: a serving process that handed all of
its device memory to an allocator it does not control, or a plain C host program with no
device allocator (where a cudaMalloc mid-request could also synchronise the device).
m3_scan_fwd_noalloc takes its scratch from a fixed array inside libm3 instead.  These
tests call it through the C ABI and compare it with m3_scan_fwd (which takes a
caller-allocated workspace) on the same inputs, twice in a row, within the bf16
tolerance the parity tests use.  The file is collected last on purpose.
"""

import numpy as np
import pytest
import torch

from oracle import oracle as orc
from selective_state_space_53_b200 import m3
from selective_state_space_53_b200.inputs import make_inputs, make_state

pytestmark = pytest.mark.gpu

TOL = 2e-2  # bf16 inputs, fp32 state: the parity tests' bound


def rel_err(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.abs(got - ref).max() / max(np.abs(ref).max(), 1e-30))


def _run(inp, init, noalloc):
    dims = m3.dims_of(inp)
    dev = m3.to_device(inp)
    st, (th, tb, tx) = m3.state_tensors(dims, h=init[0], carry_B=init[1], carry_x=init[2])
    y = torch.empty_like(dev["x"])
    ops = [dev[k] for k in m3._OPERANDS]
    if noalloc:
        m3.m3_scan_fwd_noalloc(dims, *ops, st, y)
    else:
        n = m3.m3_scan_workspace_size(dims)
        ws = torch.empty(max(n, 16), dtype=torch.uint8, device="cuda")
        m3.m3_scan_fwd(dims, *ops, st, y, workspace=ws)
    torch.cuda.synchronize()
    return y.float().cpu().numpy(), th.cpu().numpy(), tb.cpu().numpy(), tx.cpu().numpy()


@pytest.mark.parametrize("shape", [
    dict(b=1, L=2000, H=2, P=64, N=64, R=2, G=1),      # many segments: scratch in use
    dict(b=4, L=2048, H=24, P=64, N=64, R=2, G=1),     # the page-1 layer
    dict(b=2, L=999, H=2, P=128, N=128, R=4, G=2),     # 1.5B-scale heads, ragged tail
])
def test_noalloc_matches_workspace_entry_point_twice(shape):
    assert torch.cuda.is_available()
    inp = make_inputs(dtype="bf16", seed=301, extras=True, **shape)
    init = make_state(shape["b"], shape["H"], shape["P"], shape["N"], shape["R"], seed=302, scale=0.5)
    assert m3.m3_scan_workspace_size(m3.dims_of(inp)) > 0
    ref = _run(inp, init, noalloc=False)
    for _ in range(2):  # the shared scratch keeps the previous call's contents
        got = _run(inp, init, noalloc=True)
        assert rel_err(got[0], ref[0]) < TOL
        assert rel_err(got[1], ref[1]) < TOL
        np.testing.assert_array_equal(got[2], ref[2])
        np.testing.assert_array_equal(got[3], ref[3])
    assert m3.m3_check() == 0


def test_noalloc_near_the_scratch_limit():
    # 74 (batch, head) sequences at d_state = headdim = 128 make the segment planner ask for
    # its largest scratch on a 148-SM part (about 14 MiB of the 16 MiB array), so the high
    # end of the array is in use; checked against the oracle on sampled heads and against
    # m3_scan_fwd on everything, on two calls in a row
    shape = dict(b=2, L=4096, H=37, P=128, N=128, R=4, G=1)
    inp = make_inputs(dtype="bf16", seed=303, extras=True, **shape)
    init = make_state(shape["b"], shape["H"], shape["P"], shape["N"], shape["R"], seed=304, scale=0.5)
    need = m3.m3_scan_workspace_size(m3.dims_of(inp))
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    if sms == 148:
        assert need > 12 * 2**20, need
    ref = _run(inp, init, noalloc=False)
    pairs = [(0, 0), (0, 36), (1, 18)]
    yr, hr, _, _ = orc.scan_inputs(inp, sel=pairs, h0=init[0], carry_B0=init[1], carry_x0=init[2])
    for _ in range(2):
        got = _run(inp, init, noalloc=True)
        assert rel_err(got[0], ref[0]) < TOL
        assert rel_err(got[1], ref[1]) < TOL
        y = np.stack([got[0][bi, :, hi] for bi, hi in pairs])
        h = np.stack([got[1][bi, hi] for bi, hi in pairs])
        assert rel_err(y, np.stack([yr[bi, :, hi] for bi, hi in pairs])) < TOL
        assert rel_err(h, np.stack([hr[bi, hi] for bi, hi in pairs])) < TOL
    assert m3.m3_check() == 0
