"""Pins of the oracle's front-end (BCNorm of B and C, softplus, -exp, sigmoid; Cartesia blog and
docsaid note, section アーキテクチャ; section その1 for the step parameterisation): closed values
of the activations, unit RMS of normalised rows and their scale invariance."""

import math

import numpy as np

from oracle import oracle as orc
from selective_state_space_53_b200.inputs import make_raw_inputs


def test_activations_closed_values():
    inp = make_raw_inputs(1, 3, 1, 8, 8, 1, 1, "f32", seed=1)
    inp.dt[:] = np.array([0.0, -30.0, 30.0]).reshape(1, 3, 1)
    inp.A[:] = np.array([0.0, 1.0, -1.0]).reshape(1, 3, 1)
    inp.lam[:] = np.array([0.0, 40.0, -40.0]).reshape(1, 3, 1)
    f = orc.frontend(inp)
    np.testing.assert_allclose(f.dt.ravel(), [math.log(2.0), math.exp(-30.0), 30.0], rtol=1e-12)
    np.testing.assert_allclose(f.A.ravel(), [-1.0, -math.e, -1.0 / math.e], rtol=1e-15)
    np.testing.assert_allclose(f.lam.ravel(), [0.5, 1.0, 0.0], atol=1e-16)


def test_bcnorm_rows_unit_rms_and_scale_free():
    inp = make_raw_inputs(2, 5, 2, 8, 16, 2, 1, "f32", seed=2)
    f = orc.frontend(inp)
    for M in (f.B, f.C):
        rms = np.sqrt(np.mean(M * M, axis=-1))
        np.testing.assert_allclose(rms, 1.0, atol=1e-5)  # eps 1e-6 against rows of RMS >= 0.25
    g = orc.frontend(inp)
    inp.B = inp.B * 3.0
    np.testing.assert_allclose(orc.frontend(inp).B, g.B, rtol=1e-4)  # up to eps / mean(B^2) >= 1.6e-5
