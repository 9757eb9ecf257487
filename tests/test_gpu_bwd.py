"""GPU backward pass (m3_scan_bwd through the C ABI) against the fp64 oracle's reverse-mode
gradient (m3o_scan_bwd, itself pinned by central finite differences of the forward recurrence).

Metric: max|got - ref| / max|ref| per gradient tensor; bounds 2e-2 for bf16 x/B/C/dy (the
gradients dx, dB, dC are stored in bf16) and 1e-4 for fp32 operands, the bounds of the forward
pass (the recomputed forward states and the sums over tokens run in fp32, in an order set by
atomics).
"""

import numpy as np
import pytest
import torch

from oracle import oracle as orc
from selective_state_space_53_b200 import m3
from selective_state_space_53_b200.inputs import make_inputs, make_state, round_to_bf16

pytestmark = pytest.mark.gpu

TOL = {"bf16": 2e-2, "f32": 1e-4}


def rel_err(got, ref):
    ref = np.asarray(ref, np.float64)
    return float(np.abs(np.asarray(got, np.float64) - ref).max() / max(np.abs(ref).max(), 1e-300))


def check_bwd(inp, state=None, with_dh=True, flags=0, seed=900):
    dims = m3.dims_of(inp, flags=flags)
    dev = m3.to_device(inp)
    d = inp.dims
    rng = np.random.default_rng(seed)
    dy = rng.standard_normal((d["b"], d["L"], d["H"], d["P"])).astype(np.float32)
    if d["dtype"] == "bf16":
        dy = round_to_bf16(dy)
    dhf = rng.standard_normal((d["b"], d["H"], d["N"], d["P"])).astype(np.float32) if with_dh else None
    st, keep = m3.state_tensors(dims, h=None if state is None else state[0],
                                carry_B=None if state is None else state[1],
                                carry_x=None if state is None else state[2])
    tdy = torch.from_numpy(dy).to(dev["x"].dtype).cuda()
    tdh = None if dhf is None else torch.from_numpy(dhf).cuda()
    got = m3.scan_backward(dims, dev, st, tdy, tdh)
    torch.cuda.synchronize()
    assert m3.m3_check() == 0
    kw = {} if state is None else dict(h0=state[0], carry_B0=state[1], carry_x0=state[2])
    ref = orc.scan_bwd(d, inp.x, inp.dt, inp.A, inp.lam, inp.B, inp.C, inp.theta, inp.bias_B, inp.bias_C, inp.W_x,
                       inp.W_o, inp.D, dy=dy, dh_final=dhf, angle_direct=bool(flags & m3.M3_FLAG_ANGLE_DIRECT), **kw)
    tol = TOL[d["dtype"]]
    errs = {}
    for k in m3.GRAD_KEYS:
        if ref[k] is None:
            continue
        errs[k] = rel_err(got[k].float().cpu().numpy(), ref[k])
    print("bwd errors: " + ", ".join(f"{k} {v:.1e}" for k, v in errs.items()))
    bad = {k: v for k, v in errs.items() if not v < tol}
    assert not bad, bad


@pytest.mark.parametrize("shape", [
    dict(b=2, L=37, H=4, P=16, N=16, R=1, G=1),
    dict(b=1, L=50, H=4, P=32, N=16, R=2, G=2),
    dict(b=2, L=20, H=2, P=64, N=64, R=2, G=1),
    dict(b=1, L=130, H=2, P=128, N=128, R=4, G=1),
], ids=lambda s: "L{L}P{P}N{N}R{R}G{G}".format(**s))
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_bwd_matches_oracle(shape, dtype):
    inp = make_inputs(dtype=dtype, seed=901, extras=True, **shape)
    st = make_state(shape["b"], shape["H"], shape["P"], shape["N"], shape["R"], seed=902, scale=0.5)
    check_bwd(inp, state=st)


def test_bwd_direct_angle_no_final_cotangent():
    inp = make_inputs(dtype="f32", seed=903, extras=True, b=2, L=33, H=2, P=16, N=8, R=2, G=1)
    check_bwd(inp, with_dh=False, flags=m3.M3_FLAG_ANGLE_DIRECT)


def test_bwd_page1_layer_shape_sampled():
    # the page-1 layer's head shape over a full-length sequence (one batch row, 4 heads)
    inp = make_inputs(dtype="bf16", seed=904, extras=True, b=1, L=2048, H=4, P=64, N=64, R=2, G=1)
    check_bwd(inp)


def _head_subset(inp, sel):
    """The draw restricted to heads `sel` (G = 1: B, C and theta are shared by every head)."""
    import copy
    sub = copy.copy(inp)
    sub.dims = dict(inp.dims, H=len(sel))
    for k in ("x", "dt", "A", "lam"):
        setattr(sub, k, np.ascontiguousarray(getattr(inp, k)[:, :, sel]))
    for k in ("bias_B", "bias_C", "W_x", "W_o", "D"):
        a = getattr(inp, k)
        setattr(sub, k, None if a is None else np.ascontiguousarray(a[sel]))
    return sub


@pytest.mark.parametrize("cfg", ["p1_layer", "l15b_2k"])
def test_bwd_full_config_sampled_heads(cfg):
    """The backward at a layer workload's full size on the GPU, with cotangents on two sampled heads
    only: their per-head gradients and the shared B, C, theta gradients (the other heads add
    nothing) against the oracle run on those heads."""
    from selective_state_space_53_b200.inputs import CONFIGS, SEEDS
    c = dict(CONFIGS[cfg])
    inp = make_inputs(seed=SEEDS[cfg] + 7, extras=True, **{k: c[k] for k in ("b", "L", "H", "P", "N", "R", "G", "dtype")})
    d = inp.dims
    rng = np.random.default_rng(905)
    sel = sorted(int(h) for h in rng.choice(d["H"], 2, replace=False))
    dy = np.zeros((d["b"], d["L"], d["H"], d["P"]), np.float32)
    dy[:, :, sel] = round_to_bf16(rng.standard_normal((d["b"], d["L"], 2, d["P"])).astype(np.float32))
    dhf = np.zeros((d["b"], d["H"], d["N"], d["P"]), np.float32)
    dhf[:, sel] = rng.standard_normal((d["b"], 2, d["N"], d["P"])).astype(np.float32)
    dims = m3.dims_of(inp)
    dev = m3.to_device(inp)
    st, keep = m3.state_tensors(dims)
    got = m3.scan_backward(dims, dev, st, torch.from_numpy(dy).to(torch.bfloat16).cuda(), torch.from_numpy(dhf).cuda())
    torch.cuda.synchronize()
    assert m3.m3_check() == 0
    sub = _head_subset(inp, sel)
    ref = orc.scan_bwd(sub.dims, sub.x, sub.dt, sub.A, sub.lam, sub.B, sub.C, sub.theta, sub.bias_B, sub.bias_C,
                       sub.W_x, sub.W_o, sub.D, dy=dy[:, :, sel], dh_final=dhf[:, sel])
    per_head_tok = ("dx", "ddt", "dA", "dlam")
    per_head = ("dbias_B", "dbias_C", "dW_x", "dW_o", "dD")
    per_seq_head = ("dh0", "dcarry_B", "dcarry_x")
    errs = {}
    for k in m3.GRAD_KEYS:
        g = got[k].float().cpu().numpy()
        if k in per_head_tok:
            g = g[:, :, sel]
        elif k in per_head:
            g = g[sel]
        elif k in per_seq_head:
            g = g[:, sel]
        errs[k] = rel_err(g, ref[k])
    print(f"{cfg} bwd (heads {sel}): " + ", ".join(f"{k} {v:.1e}" for k, v in errs.items()))
    bad = {k: v for k, v in errs.items() if not v < TOL["bf16"]}
    assert not bad, bad
