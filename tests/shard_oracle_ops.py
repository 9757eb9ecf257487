"""Range summaries and their fold computed with the fp64 oracle and numpy (test infrastructure).

The same three operations as ``selective_state_space_53_b200.shard.LibOps`` (summarise a range,
fold summaries onto a state, scan a range from a state), on host arrays: the CPU tests run the
sharded orchestration over them, and the fold below restates the range algebra that the GPU
fold kernel implements (a range maps the state entering it to e^{logdec} Rot(angle)(h +
bp_first u) + Z; Mamba-3 paper note, sections その1-その3; IBM Mamba page, associative scan).
"""

import numpy as np
import torch

from oracle import oracle as orc


def range_inputs(inp, lo, hi):
    """The draw restricted to tokens lo..hi-1 of every sequence."""
    import copy
    sub = copy.copy(inp)
    for k in ("x", "dt", "A", "lam", "B", "C", "theta"):
        setattr(sub, k, np.ascontiguousarray(getattr(inp, k)[:, lo:hi]))
    sub.dims = dict(inp.dims, L=hi - lo)
    return sub


class OracleOps:
    def summarise(self, dims, inp):
        d = inp.dims
        H, G = d["H"], d["G"]
        _, Z, cB, cx = orc.scan_inputs(inp)
        dt = inp.dt.astype(np.float64)
        logdec = (dt * inp.A.astype(np.float64)).sum(axis=1)                      # (b, H)
        gidx = np.arange(H) // (H // G)
        th = inp.theta.astype(np.float64)[:, :, gidx, :]                           # (b, L, H, N/2)
        ang = (dt[..., None] * th).sum(axis=1)
        ang = ang - 2 * np.pi * np.rint(ang / (2 * np.pi))
        bp = (1.0 - inp.lam[:, 0].astype(np.float64)) * dt[:, 0]
        out = dict(Z=Z, logdec=logdec, angle=ang, bp_first=bp, carry_B=cB, carry_x=cx)
        return {k: torch.from_numpy(np.ascontiguousarray(v, dtype=np.float64)) for k, v in out.items()}

    def fold(self, dims, state, before, inp):
        h, cB, cx = (np.array(a, dtype=np.float64) for a in state)
        if before is None:
            return h, cB, cx
        R = inp.dims["R"]
        bias = np.zeros((inp.dims["H"], R, inp.dims["N"])) if inp.bias_B is None else inp.bias_B.astype(np.float64)
        wx = np.ones((inp.dims["H"], R, inp.dims["P"])) if inp.W_x is None else inp.W_x.astype(np.float64)
        for q in range(before["logdec"].shape[0]):
            s = {k: v[q].numpy() for k, v in before.items()}
            Bb = cB + bias[None]                                                   # (b, H, R, N)
            X = wx[None] * cx[:, :, None, :]                                       # (b, H, R, P)
            u = np.einsum("bhrn,bhrp->bhnp", Bb, X)
            hp = h + s["bp_first"][..., None, None] * u
            c = np.cos(s["angle"])[..., None]
            sn = np.sin(s["angle"])[..., None]
            rot = np.empty_like(hp)
            rot[:, :, 0::2] = c * hp[:, :, 0::2] - sn * hp[:, :, 1::2]
            rot[:, :, 1::2] = sn * hp[:, :, 0::2] + c * hp[:, :, 1::2]
            h = np.exp(s["logdec"])[..., None, None] * rot + s["Z"]
            cB, cx = s["carry_B"], s["carry_x"]
        return h, cB, cx

    def scan(self, dims, inp, state):
        y, h, cB, cx = orc.scan_inputs(inp, h0=state[0], carry_B0=state[1], carry_x0=state[2])
        return y, (h, cB, cx)
