"""GPU output norm (m3_output_norm through the C ABI) against the oracle's output norm."""

import numpy as np
import pytest
import torch

from oracle import oracle as orc
from selective_state_space_53_b200 import m3
from selective_state_space_53_b200.inputs import round_to_bf16

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype,gate,weight,P", [
    ("bf16", True, True, 128), ("bf16", False, False, 64), ("f32", True, True, 16), ("f32", False, True, 256),
])
def test_output_norm_matches_oracle(dtype, gate, weight, P):
    b, L, H = 2, 37, 3
    rng = np.random.default_rng(950)
    y = (3.0 * rng.standard_normal((b, L, H, P))).astype(np.float32)
    z = rng.standard_normal((b, L, H, P)).astype(np.float32) if gate else None
    if dtype == "bf16":
        y = round_to_bf16(y)
        z = None if z is None else round_to_bf16(z)
    w = (1.0 + 0.1 * rng.standard_normal((H, P))).astype(np.float32) if weight else None
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    ty = torch.from_numpy(y).to(tdt).cuda()
    tz = None if z is None else torch.from_numpy(z).to(tdt).cuda()
    tw = None if w is None else torch.from_numpy(w).cuda()
    out = torch.empty_like(ty)
    dims = m3.make_dims(b, L, H, P, 16, 1, 1, dtype)
    m3.m3_output_norm(dims, ty, tz, tw, 1e-6, out)
    torch.cuda.synchronize()
    ref = orc.output_norm(y, z, w, eps=1e-6)
    err = float(np.abs(out.float().cpu().numpy() - ref).max() / np.abs(ref).max())
    assert err < (1e-2 if dtype == "bf16" else 1e-5), err
