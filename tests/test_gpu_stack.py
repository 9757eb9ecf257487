"""GPU parity of the core inside the 12-layer stack (b8 L4096, the page-1 language-model shape).

Every layer's core (m3_scan_fwd with M3_FLAG_RAW_INPUTS through the C ABI: the core applies the
block's front-end itself) is compared with the fp64 oracle composed with the oracle's front-end
on sampled (batch, head) sequences of that layer, on the raw operands the stack produced for it:
the inputs of deeper layers come from the residual stream of the model, not from the seeded
generator.
Tolerance as for every bf16 case: max relative error 2e-2 per output tensor.
"""

import numpy as np
import pytest
import torch

from oracle import oracle as orc
from selective_state_space_53_b200 import m3
from selective_state_space_53_b200.inputs import CONFIGS, Inputs
from selective_state_space_53_b200.stack import Mamba3Stack, StackShape

pytestmark = pytest.mark.gpu

TOL = 2e-2


def rel_err(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.abs(ref).max()
    return float(np.abs(got - ref).max() / (den if den > 0 else 1.0))


def pair_inputs(dev, bi, hi, shape, L):
    """The operands of one (batch, head) sequence as a b = 1, H = 1 draw (G = 1: B, C, theta
    are shared by the heads of the group)."""
    def host(t):
        return None if t is None else t.float().cpu().numpy()
    g = hi // (shape.H // shape.G)
    return Inputs(
        dims=dict(b=1, L=L, H=1, P=shape.P, N=shape.N, R=shape.R, G=1, dtype="bf16"),
        x=host(dev["x"][bi:bi + 1, :, hi:hi + 1]),
        dt=host(dev["dt"][bi:bi + 1, :, hi:hi + 1]),
        A=host(dev["A"][bi:bi + 1, :, hi:hi + 1]),
        lam=host(dev["lam"][bi:bi + 1, :, hi:hi + 1]),
        theta=host(dev["theta"][bi:bi + 1, :, g:g + 1]),
        B=host(dev["B"][bi:bi + 1, :, g:g + 1]),
        C=host(dev["C"][bi:bi + 1, :, g:g + 1]),
        bias_B=host(dev["bias_B"][hi:hi + 1]), bias_C=host(dev["bias_C"][hi:hi + 1]),
        W_x=host(dev["W_x"][hi:hi + 1]), W_o=host(dev["W_o"][hi:hi + 1]), D=host(dev["D"][hi:hi + 1]),
        extra={"raw": True})


def test_twelve_layer_stack_core_parity():
    cfg = CONFIGS["p1_stack"]
    shape = StackShape(layers=cfg["layers"], H=cfg["H"], P=cfg["P"], N=cfg["N"], R=cfg["R"], G=cfg["G"])
    b, L = cfg["b"], cfg["L"]
    stack = Mamba3Stack(shape, seed=1002)
    gen = torch.Generator(device="cpu").manual_seed(2002)
    u = torch.randn(b, L, shape.d_model, generator=gen).to(torch.bfloat16).cuda()
    errs = []
    rng = np.random.default_rng(3002)

    def check(li, dev, y):
        pairs = [(int(rng.integers(b)), int(rng.integers(shape.H))) for _ in range(2)]
        for bi, hi in pairs:
            inp = orc.frontend(pair_inputs(dev, bi, hi, shape, L))
            yr, _, _, _ = orc.scan_inputs(inp)
            got = y[bi:bi + 1, :, hi:hi + 1].float().cpu().numpy()
            errs.append((li, bi, hi, rel_err(got, yr)))

    out = stack.forward(u, check=check)
    torch.cuda.synchronize()
    assert m3.m3_check() == 0
    assert torch.isfinite(out.float()).all()
    worst = max(errs, key=lambda e: e[3])
    print(f"stack: {len(errs)} sampled sequences, worst y max rel err {worst[3]:.2e} at layer {worst[0]}")
    assert worst[3] < TOL, worst
