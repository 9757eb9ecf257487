"""Seeded synthetic inputs for the Mamba-3 SSM layer core.

This module draws random tensors and casts them to their storage dtype.  It holds
none of the SSM's arithmetic: the oracle (test infrastructure) and the CUDA path
both receive what it returns, and neither is imported here.

Distributions follow the workload description of the layer (Mamba-3, "Mamba-3:
Improved Sequence Modeling using State Space Principles", docsaid.org paper note,
section "その1 離散化" for Delta/A/lambda, "アーキテクチャ" for the B/C
normalisation and bias; the page-1 article "Mamba3をゼロから実装して..." section
"モデルの初期化方法" for the 0.02 B/C bias):

* x ~ N(0, 1)                              shape (b, L, H, P)
* dt = softplus(N(-2, 0.5))                shape (b, L, H)
* A = -exp(U(0, 1))                        shape (b, L, H)
* lam = sigmoid(N(0, 1))                   shape (b, L, H)
* theta ~ U(-pi, pi)                       shape (b, L, G, N/2)
* B, C ~ N(0, 1), RMS-normalised over N    shape (b, L, G, R, N)
* bias_B = bias_C = 0.02                   shape (H, R, N)
* W_x = 1 + 0.1 N(0, 1), W_o = (1 + 0.1 N(0, 1)) / R   shape (H, R, P)
* D: absent unless ``extras=True``

Draw order is fixed (x, dt, A, lam, theta, B, C, W_x, W_o, then the optional
extras) and every draw is made in float64 before the cast, so a given seed gives
the same values whatever the storage dtype.  bf16 tensors are returned as float32
arrays whose values are exactly representable in bf16 (round to nearest even).
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field, asdict

import numpy as np

# Workloads of the layer, by name.  Sizes only; no arithmetic of the method.
CONFIGS = {
    # tiny single-layer SISO scan, fp32
    "tiny_f32": dict(b=1, L=256, H=4, P=16, N=16, R=1, G=1, dtype="f32"),
    # page-1-shaped layer: d_model 768 -> d_inner 1536 = 24 heads x 64, d_state 64, MIMO rank 2
    "p1_layer": dict(b=4, L=2048, H=24, P=64, N=64, R=2, G=1, dtype="bf16"),
    # 12-layer stack of the page-1 layer shape, batch 8, seqlen 4096
    "p1_stack": dict(b=8, L=4096, H=24, P=64, N=64, R=2, G=1, dtype="bf16", layers=12),
    # 1.5B-scale layer: 32 heads x 128, d_state 128, MIMO rank 4 (seqlen sweep 2K/8K/32K)
    "l15b_2k": dict(b=2, L=2048, H=32, P=128, N=128, R=4, G=1, dtype="bf16"),
    "l15b_8k": dict(b=2, L=8192, H=32, P=128, N=128, R=4, G=1, dtype="bf16"),
    "l15b_32k": dict(b=2, L=32768, H=32, P=128, N=128, R=4, G=1, dtype="bf16"),
    # decode on the 1.5B-scale layer: batch sweep, 1024 one-token steps
    "decode_b1": dict(b=1, L=1024, H=32, P=128, N=128, R=4, G=1, dtype="bf16"),
    "decode_b16": dict(b=16, L=1024, H=32, P=128, N=128, R=4, G=1, dtype="bf16"),
    "decode_b128": dict(b=128, L=1024, H=32, P=128, N=128, R=4, G=1, dtype="bf16"),
    "decode_b512": dict(b=512, L=1024, H=32, P=128, N=128, R=4, G=1, dtype="bf16"),
    # decode on the page-1 layer (N = P = 64, R = 2) at batch 128
    "decode_p1_b128": dict(b=128, L=1024, H=24, P=64, N=64, R=2, G=1, dtype="bf16"),
}

# seed = 1000 + index of the workload family in the list above's families
SEEDS = {"tiny_f32": 1000, "p1_layer": 1001, "p1_stack": 1002,
         "l15b_2k": 1003, "l15b_8k": 1003, "l15b_32k": 1003,
         "decode_b1": 1004, "decode_b16": 1004, "decode_b128": 1004, "decode_b512": 1004, "decode_p1_b128": 1001}

_CHUNK = 1 << 22  # draws are made in blocks of this many values to bound host memory


def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returns float32."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32)


def _cast(a64: np.ndarray, dtype: str) -> np.ndarray:
    a32 = a64.astype(np.float32)
    return round_to_bf16(a32) if dtype == "bf16" else a32


def _normal(rng, shape, dtype, loc=0.0, scale=1.0):
    """N(loc, scale) drawn in float64 blocks, cast per block to the storage dtype."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.float32)
    for i in range(0, n, _CHUNK):
        m = min(_CHUNK, n - i)
        out[i:i + m] = _cast(loc + scale * rng.standard_normal(m), dtype)
    return out.reshape(shape)


def _softplus(z):
    return np.logaddexp(0.0, z)


def _sigmoid(z):
    return 0.5 * (1.0 + np.tanh(0.5 * z))


def _rms_normalise(v, eps=1e-6):
    # BCNorm of the block (applied before the core): x / sqrt(mean(x^2) + eps) over N
    return v / np.sqrt(np.mean(v * v, axis=-1, keepdims=True) + eps)


@dataclass
class Inputs:
    """One seeded draw.  Arrays are float32 holding storage-dtype-exact values."""
    dims: dict
    x: np.ndarray
    dt: np.ndarray
    A: np.ndarray
    lam: np.ndarray
    theta: np.ndarray
    B: np.ndarray
    C: np.ndarray
    bias_B: np.ndarray | None
    bias_C: np.ndarray | None
    W_x: np.ndarray | None
    W_o: np.ndarray | None
    D: np.ndarray | None
    seed: int = 0
    extra: dict = field(default_factory=dict)

    def arrays(self):
        return {k: getattr(self, k) for k in
                ("x", "dt", "A", "lam", "theta", "B", "C", "bias_B", "bias_C", "W_x", "W_o", "D")}


def make_inputs(b, L, H, P, N, R, G=1, dtype="bf16", seed=0, *, extras=False,
                bias=0.02, with_weights=True, **_ignored) -> Inputs:
    """Draw one batch of layer inputs.

    extras=True also randomises bias_B, bias_C (0.02 + 0.1 N(0,1)) and draws
    D ~ N(0, 1) per head; tests use it to exercise those operands.
    with_weights=False returns W_x = W_o = None (the SISO reading: ones).
    """
    if N % 2:
        raise ValueError("d_state N must be even (complex pairs)")
    rng = np.random.default_rng(seed)
    x = _normal(rng, (b, L, H, P), dtype)
    dt = _softplus(-2.0 + 0.5 * rng.standard_normal((b, L, H))).astype(np.float32)
    A = (-np.exp(rng.uniform(0.0, 1.0, (b, L, H)))).astype(np.float32)
    lam = _sigmoid(rng.standard_normal((b, L, H))).astype(np.float32)
    theta = rng.uniform(-math.pi, math.pi, (b, L, G, N // 2)).astype(np.float32)
    B = _cast(_rms_normalise(rng.standard_normal((b, L, G, R, N))), dtype)
    C = _cast(_rms_normalise(rng.standard_normal((b, L, G, R, N))), dtype)
    if with_weights:
        W_x = (1.0 + 0.1 * rng.standard_normal((H, R, P))).astype(np.float32)
        W_o = ((1.0 + 0.1 * rng.standard_normal((H, R, P))) / R).astype(np.float32)
    else:
        W_x = W_o = None
    if extras:
        bias_B = (bias + 0.1 * rng.standard_normal((H, R, N))).astype(np.float32)
        bias_C = (bias + 0.1 * rng.standard_normal((H, R, N))).astype(np.float32)
        D = rng.standard_normal(H).astype(np.float32)
    else:
        bias_B = np.full((H, R, N), bias, dtype=np.float32)
        bias_C = np.full((H, R, N), bias, dtype=np.float32)
        D = None
    dims = dict(b=b, L=L, H=H, P=P, N=N, R=R, G=G, dtype=dtype)
    return Inputs(dims, x, dt, A, lam, theta, B, C, bias_B, bias_C, W_x, W_o, D, seed=seed)


def make_raw_inputs(b, L, H, P, N, R, G=1, dtype="bf16", seed=0, *, extras=False, bias=0.02) -> Inputs:
    """Draw the layer's raw projections (for M3_FLAG_RAW_INPUTS, where the core applies the
    front-end itself): dt_raw ~ N(-2, 0.5), A_raw ~ U(0, 1), lam_raw ~ N(0, 1) (the arguments of
    softplus, -exp and sigmoid in the recipe above), and B_raw, C_raw ~ N(0, 1) scaled per
    (token, group, branch) row by U(0.25, 4) so that the row norms vary, cast to the storage
    dtype.  x, theta, biases and weights as in make_inputs.  The returned draw holds the raw
    values in dt, A, lam, B, C and extra["raw"] = True."""
    if N % 2:
        raise ValueError("d_state N must be even (complex pairs)")
    rng = np.random.default_rng(seed)
    x = _normal(rng, (b, L, H, P), dtype)
    dt = (-2.0 + 0.5 * rng.standard_normal((b, L, H))).astype(np.float32)
    A = rng.uniform(0.0, 1.0, (b, L, H)).astype(np.float32)
    lam = rng.standard_normal((b, L, H)).astype(np.float32)
    theta = rng.uniform(-math.pi, math.pi, (b, L, G, N // 2)).astype(np.float32)
    Bs = rng.uniform(0.25, 4.0, (b, L, G, R, 1))
    B = _cast(Bs * rng.standard_normal((b, L, G, R, N)), dtype)
    Cs = rng.uniform(0.25, 4.0, (b, L, G, R, 1))
    C = _cast(Cs * rng.standard_normal((b, L, G, R, N)), dtype)
    W_x = (1.0 + 0.1 * rng.standard_normal((H, R, P))).astype(np.float32)
    W_o = ((1.0 + 0.1 * rng.standard_normal((H, R, P))) / R).astype(np.float32)
    if extras:
        bias_B = (bias + 0.1 * rng.standard_normal((H, R, N))).astype(np.float32)
        bias_C = (bias + 0.1 * rng.standard_normal((H, R, N))).astype(np.float32)
        D = rng.standard_normal(H).astype(np.float32)
    else:
        bias_B = np.full((H, R, N), bias, dtype=np.float32)
        bias_C = np.full((H, R, N), bias, dtype=np.float32)
        D = None
    dims = dict(b=b, L=L, H=H, P=P, N=N, R=R, G=G, dtype=dtype)
    return Inputs(dims, x, dt, A, lam, theta, B, C, bias_B, bias_C, W_x, W_o, D, seed=seed, extra={"raw": True})


def make_state(b, H, P, N, R, seed, scale=1.0):
    """A seeded non-zero initial state (h, carry_B, carry_x) for continuation tests."""
    rng = np.random.default_rng(seed)
    h = (scale * rng.standard_normal((b, H, N, P))).astype(np.float32)
    carry_B = rng.standard_normal((b, H, R, N)).astype(np.float32)
    carry_x = rng.standard_normal((b, H, P)).astype(np.float32)
    return h, carry_B, carry_x


def config_inputs(name: str, **overrides) -> Inputs:
    cfg = dict(CONFIGS[name])
    cfg.update(overrides)
    seed = cfg.pop("seed", SEEDS.get(name, 0))
    cfg.pop("layers", None)
    return make_inputs(seed=seed, **cfg)
