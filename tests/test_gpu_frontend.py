"""The block's front-end on the GPU: m3_frontend alone, and m3_scan_fwd with
M3_FLAG_RAW_INPUTS (raw B, C, dt, A, lam) -- fused into the load stage of the headdim-128 kernel,
run as m3_frontend before the other kernels -- against the oracle's front-end composed with the
oracle's scan."""

import numpy as np
import pytest
import torch

from oracle import oracle as orc
from selective_state_space_53_b200 import m3
from selective_state_space_53_b200.inputs import make_raw_inputs, make_state

pytestmark = pytest.mark.gpu


def rel_err(got, ref):
    ref = np.asarray(ref, np.float64)
    return float(np.abs(np.asarray(got, np.float64) - ref).max() / max(np.abs(ref).max(), 1e-300))


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_frontend_kernel_matches_oracle(dtype):
    inp = make_raw_inputs(2, 33, 4, 16, 128, 2, 2, dtype, seed=960)
    dims = m3.dims_of(inp)
    dev = m3.to_device(inp)
    out = {k: torch.empty_like(dev[k]) for k in ("B", "C", "dt", "A", "lam")}
    m3.m3_frontend(dims, dev["B"], dev["C"], dev["dt"], dev["A"], dev["lam"], out["B"], out["C"], out["dt"],
                   out["A"], out["lam"])
    torch.cuda.synchronize()
    ref = orc.frontend(inp)
    tol = {"B": 8e-3 if dtype == "bf16" else 1e-5, "C": 8e-3 if dtype == "bf16" else 1e-5,
           "dt": 1e-5, "A": 1e-5, "lam": 1e-5}
    for k, t in tol.items():
        assert rel_err(out[k].float().cpu().numpy(), getattr(ref, k)) < t, k


@pytest.mark.parametrize("shape", [
    dict(b=2, L=300, H=4, P=128, N=128, R=4, G=1),   # warp-specialised kernel: front-end fused
    dict(b=1, L=3000, H=2, P=128, N=64, R=2, G=1),   # fused, segmented (state pass too)
    dict(b=1, L=200, H=2, P=64, N=64, R=2, G=1),     # headdim-64 tensor-core kernel: m3_frontend first
    dict(b=1, L=40, H=2, P=32, N=16, R=2, G=2),      # sequential kernel: m3_frontend first
    dict(b=1, L=600, H=2, P=128, N=128, R=3, G=1),   # fused, rank 3 padded to tile rank 4
], ids=["P128", "P128seg", "P64", "seq", "P128R3"])
def test_scan_with_raw_inputs_matches_oracle(shape):
    inp = make_raw_inputs(dtype="bf16", seed=961, extras=True, **shape)
    st = make_state(shape["b"], shape["H"], shape["P"], shape["N"], shape["R"], seed=962, scale=0.5)
    dims = m3.dims_of(inp, flags=m3.M3_FLAG_RAW_INPUTS)
    dev = m3.to_device(inp)
    s, (th, tb, tx) = m3.state_tensors(dims, h=st[0], carry_B=st[1], carry_x=st[2])
    y = m3.scan(dims, dev, s)
    torch.cuda.synchronize()
    assert m3.m3_check() == 0
    ref_in = orc.frontend(inp)
    yr, hr, cBr, _ = orc.scan_inputs(ref_in, h0=st[0], carry_B0=st[1], carry_x0=st[2])
    ey, eh = rel_err(y.float().cpu().numpy(), yr), rel_err(th.cpu().numpy(), hr)
    assert ey < 2e-2 and eh < 2e-2, (ey, eh)
    # the carry holds the last token's normalised B (the B the core used)
    assert rel_err(tb.cpu().numpy(), cBr) < 8e-3
