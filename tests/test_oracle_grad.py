"""Pins of the oracle's backward pass (m3o_scan_bwd) by central finite differences of the
oracle's forward recurrence (CPU, fp64).

The loss is sum(dy * y) + sum(dh_final * h_final) with random cotangents; for every operand
and the initial state, each element's analytic gradient must equal (loss(v + e) - loss(v - e))
/ 2e.  The forward pass follows the Mamba-3 paper note (docsaid.org), sections その1 (trapezoid
rule), その2 (rotation of state pairs) and その3 (MIMO branches), so these pins check the chain
rule through every term of that recurrence, the direct-angle variant included.
"""

import numpy as np
import pytest

from oracle import oracle as orc
from selective_state_space_53_b200.inputs import make_inputs, make_state

OPERANDS = ("x", "dt", "A", "lam", "B", "C", "theta", "bias_B", "bias_C", "W_x", "W_o", "D")


def _loss(vals, state, dims, dy, dhf, angle_direct):
    y, h, _, _ = orc.scan(dims, *[vals[k] for k in OPERANDS], h0=state[0], carry_B0=state[1], carry_x0=state[2],
                          angle_direct=angle_direct)
    return float((dy * y).sum() + (dhf * h).sum())


@pytest.mark.parametrize("shape,direct", [
    (dict(b=2, L=5, H=2, P=3, N=4, R=2, G=1), False),
    (dict(b=1, L=4, H=4, P=2, N=6, R=3, G=2), False),
    (dict(b=1, L=4, H=2, P=2, N=4, R=1, G=1), True),
], ids=["R2G1", "R3G2", "direct"])
def test_gradients_match_central_differences(shape, direct):
    inp = make_inputs(dtype="f32", seed=800, extras=True, **shape)
    vals = {k: (None if getattr(inp, k) is None else getattr(inp, k).astype(np.float64).copy()) for k in OPERANDS}
    st = [a.astype(np.float64) for a in make_state(shape["b"], shape["H"], shape["P"], shape["N"], shape["R"], seed=801)]
    rng = np.random.default_rng(802)
    b, L, H, P, N = shape["b"], shape["L"], shape["H"], shape["P"], shape["N"]
    dy = rng.standard_normal((b, L, H, P))
    dhf = rng.standard_normal((b, H, N, P))
    grads = orc.scan_bwd(inp.dims, *[vals[k] for k in OPERANDS], h0=st[0], carry_B0=st[1], carry_x0=st[2],
                         dy=dy, dh_final=dhf, angle_direct=direct)
    eps = 1e-6
    targets = [(k, vals, "d" + k) for k in OPERANDS] + [
        (i, st, g) for i, g in enumerate(("dh0", "dcarry_B", "dcarry_x"))]
    for key, holder, gk in targets:
        arr = holder[key]
        got = grads[gk]
        num = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            old = arr[idx]
            arr[idx] = old + eps
            lp = _loss(vals, st, inp.dims, dy, dhf, direct)
            arr[idx] = old - eps
            lm = _loss(vals, st, inp.dims, dy, dhf, direct)
            arr[idx] = old
            num[idx] = (lp - lm) / (2 * eps)
        scale = max(np.abs(num).max(), 1e-3)
        np.testing.assert_allclose(got, num, rtol=0, atol=2e-6 * scale, err_msg=gk)


def test_gradient_without_cotangents_is_zero():
    inp = make_inputs(dtype="f32", seed=803, b=1, L=3, H=1, P=2, N=2, R=1)
    g = orc.scan_bwd(inp.dims, inp.x, inp.dt, inp.A, inp.lam, inp.B, inp.C, inp.theta, inp.bias_B, inp.bias_C,
                     inp.W_x, inp.W_o, inp.D)
    for k, v in g.items():
        if v is not None:
            assert not np.any(v), k
