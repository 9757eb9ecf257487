"""Pins of the oracle's output norm (the hybrid model's norm before the output projection;
Mamba-3 paper note, docsaid.org, section アーキテクチャ): a hand-computed row, the RMS of a
normalised row, scale invariance, the gate's closed form and the per-channel weight."""

import math

import numpy as np

from oracle import oracle as orc


def test_hand_computed_row():
    y = np.array([3.0, 4.0]).reshape(1, 1, 1, 2)
    out = orc.output_norm(y, eps=0.0)
    r = math.sqrt((9 + 16) / 2)
    np.testing.assert_allclose(out.ravel(), [3 / r, 4 / r], rtol=1e-15)


def test_normalised_rows_have_unit_rms_and_ignore_scale():
    rng = np.random.default_rng(1)
    y = rng.standard_normal((2, 3, 4, 16))
    out = orc.output_norm(y, eps=0.0)
    np.testing.assert_allclose(np.sqrt(np.mean(out ** 2, axis=-1)), 1.0, rtol=1e-14)
    np.testing.assert_allclose(orc.output_norm(7.5 * y, eps=0.0), out, rtol=1e-13)


def test_gate_is_silu():
    y = np.ones((1, 1, 1, 2))
    z = np.array([0.0, 2.0]).reshape(1, 1, 1, 2)
    v = np.array([0.0, 2.0 / (1.0 + math.exp(-2.0))])
    out = orc.output_norm(y, z, eps=0.0)
    np.testing.assert_allclose(out.ravel(), v / math.sqrt(np.mean(v ** 2)), rtol=1e-14)


def test_weight_scales_channels_per_head():
    rng = np.random.default_rng(2)
    y = rng.standard_normal((1, 2, 3, 4))
    w = rng.standard_normal((3, 4))
    np.testing.assert_allclose(orc.output_norm(y, weight=w), orc.output_norm(y) * w[None, None], rtol=1e-14)
