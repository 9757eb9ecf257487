"""Pins of the fp64 oracle against facts that do not come from the oracle itself.

Every test here runs on the CPU.  Sources (Mamba-3 paper note, docsaid.org):
  * section その2, worked example (listing and printed output): a rotating 2-D
    state solves parity; a non-negative decay only shrinks (values in
    tests/golden/parity_example.txt);
  * section その2, statements 1 and 2: complex SSM == real SSM of doubled size ==
    data-dependent RoPE on B and C;
  * section その1: lam = 1 gives back the exponential-Euler (Mamba-2) rule; the
    previous-token term acts as a width-2 convolution of the input;
  * section その3: MIMO rank R is a sum of rank-one (SISO) updates;
  * IBM page on Mamba, SSD section: matrix form and chunking of the scan.
"""

import math
import os

import numpy as np
import pytest

from oracle import forms
from oracle import oracle as orc
from selective_state_space_53_b200.inputs import make_inputs, make_state

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "parity_example.txt")


def _golden():
    vals = {}
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        k, *v = line.split()
        vals[k] = v
    return vals


def _toy(L, theta_vals, log_alpha, x=None, N=2, P=1, lam=0.5, dt=1.0):
    """b=1, H=1, R=1, G=1 arrays for hand-built examples."""
    b, H, R, G = 1, 1, 1, 1
    arr = dict(
        x=np.zeros((b, L, H, P)) if x is None else np.asarray(x, float).reshape(b, L, H, P),
        dt=np.full((b, L, H), dt),
        A=(np.asarray(log_alpha, float) / dt).reshape(b, L, H) * np.ones((b, L, H)),
        lam=np.full((b, L, H), lam),
        theta=(np.asarray(theta_vals, float) / dt).reshape(b, L, G, -1) * np.ones((b, L, G, N // 2)),
        B=np.zeros((b, L, G, R, N)), C=np.zeros((b, L, G, R, N)),
    )
    dims = dict(b=b, L=L, H=H, P=P, N=N, R=R, G=G)
    return dims, arr


def _scan(dims, arr, **kw):
    return orc.scan(dims, arr["x"], arr["dt"], arr["A"], arr["lam"], arr["B"], arr["C"], arr["theta"],
                    arr.get("bias_B"), arr.get("bias_C"), arr.get("W_x"), arr.get("W_o"), arr.get("D"), **kw)


# ---------------------------------------------------------------- printed example

def test_parity_example_matches_printed_output():
    g = _golden()
    bits = np.random.default_rng(int(g["seed"][0])).integers(0, 2, size=int(g["n_bits"][0]))
    assert bits.sum() % 2 == int(g["parity"][0])
    L = len(bits)
    dims, arr = _toy(L, theta_vals=math.pi * bits, log_alpha=np.zeros(L))
    h0 = np.array([1.0, 0.0]).reshape(1, 1, 2, 1)
    _, h, _, _ = _scan(dims, arr, h0=h0)
    want = np.array([float(v) for v in g["rotating_state_final"]])
    np.testing.assert_allclose(h[0, 0, :, 0], want, atol=1e-6)
    assert (0 if h[0, 0, 0, 0] > 0 else 1) == int(g["parity"][0])


def test_decay_example_matches_printed_output():
    g = _golden()
    bits = np.random.default_rng(int(g["seed"][0])).integers(0, 2, size=int(g["n_bits"][0]))
    n = int(g["decay_steps"][0])
    alpha = np.where(bits[:n] == 1, 0.5, 0.9)
    dims, arr = _toy(n, theta_vals=np.zeros(n), log_alpha=np.log(alpha))
    h0 = np.array([1.0, 0.0]).reshape(1, 1, 2, 1)
    _, h, _, _ = _scan(dims, arr, h0=h0)
    assert round(float(h[0, 0, 0, 0]), 6) == float(g["decay_final_rounded_6"][0])
    assert h[0, 0, 1, 0] == 0.0
    assert float(h[0, 0, 0, 0]) > 0.0  # never flips sign


def test_rotation_convention_quarter_turn():
    # The listing's rot(theta) is [[c, -s], [s, c]]: a quarter turn maps [1, 0] to [0, 1].
    dims, arr = _toy(1, theta_vals=[math.pi / 2], log_alpha=[0.0])
    _, h, _, _ = _scan(dims, arr, h0=np.array([1.0, 0.0]).reshape(1, 1, 2, 1))
    np.testing.assert_allclose(h[0, 0, :, 0], [0.0, 1.0], atol=1e-15)


# ---------------------------------------------------------------- closed forms

def test_impulse_response_closed_form():
    # x only at s = 0, theta = 0: h_t = (prod_{k=1..t} alpha_k)(gamma_0 + beta'_1) u_0, t >= 1
    rng = np.random.default_rng(5)
    L = 9
    la = -rng.uniform(0.05, 0.5, L)
    dt = rng.uniform(0.1, 0.6, L)
    lam = rng.uniform(0.0, 1.0, L)
    x = np.zeros(L)
    x[0] = 1.7
    dims, arr = _toy(L, theta_vals=np.zeros(L), log_alpha=np.zeros(L), x=x)
    arr["dt"] = dt.reshape(1, L, 1)
    arr["A"] = (la / dt).reshape(1, L, 1)
    arr["lam"] = lam.reshape(1, L, 1)
    arr["B"][0, :, 0, 0, 0] = 1.0
    for t in range(1, L + 1):
        d = dict(dims, L=t)
        sub = {k: v[:, :t] for k, v in arr.items()}
        _, h, _, _ = _scan(d, sub)
        gam0, bp1 = lam[0] * dt[0], (1.0 - lam[1]) * dt[1] if t > 1 else 0.0
        want = (gam0 if t == 1 else np.exp(la[1:t].sum()) * (gam0 + bp1)) * 1.7
        assert abs(h[0, 0, 0, 0] - want) < 1e-14 * max(1.0, abs(want))


def test_steady_state_closed_form_with_rotation():
    # Constant alpha, lam, dt, angle phi and constant input u: the state tends to the
    # fixed point h* = (I - alpha Rot)^{-1} (alpha Rot beta' + gamma) u.
    L = 600
    alpha, lam, dt, phi = 0.9, 0.3, 0.7, 0.4
    dims, arr = _toy(L, theta_vals=np.full(L, phi), log_alpha=np.full(L, math.log(alpha)),
                     x=np.ones(L), lam=lam, dt=dt)
    arr["B"][0, :, 0, 0, :] = [0.6, -0.8]
    _, h, _, _ = _scan(dims, arr)
    u = np.array([0.6, -0.8])
    c, s = math.cos(phi), math.sin(phi)
    Rm = np.array([[c, -s], [s, c]])
    bp, gm = (1 - lam) * dt, lam * dt
    want = np.linalg.solve(np.eye(2) - alpha * Rm, (alpha * bp * Rm + gm * np.eye(2)) @ u)
    np.testing.assert_allclose(h[0, 0, :, 0], want, rtol=1e-12, atol=1e-12)
    # theta = 0 reduces to the scalar fixed point (alpha beta' + gamma) u / (1 - alpha)
    arr["theta"][:] = 0.0
    _, h, _, _ = _scan(dims, arr)
    np.testing.assert_allclose(h[0, 0, :, 0], (alpha * bp + gm) * u / (1 - alpha), rtol=1e-12)


def test_skip_term_only():
    inp = make_inputs(1, 7, 3, 8, 4, 2, 1, "f32", seed=11, extras=True)
    a = inp.arrays()
    a["C"] = np.zeros_like(a["C"])
    a["bias_C"] = np.zeros_like(a["bias_C"])
    y, _, _, _ = orc.scan(inp.dims, **{k: a[k] for k in a})
    want = a["D"].astype(np.float64)[None, None, :, None] * inp.x.astype(np.float64)
    np.testing.assert_allclose(y, want, rtol=0, atol=1e-15)


# ---------------------------------------------------------------- independent forms

SHAPES = [
    dict(b=1, L=13, H=2, P=3, N=4, R=1, G=1),
    dict(b=2, L=11, H=4, P=5, N=6, R=2, G=2),
    dict(b=1, L=10, H=2, P=4, N=8, R=4, G=1),
]


def _rand(shape, seed, state=False):
    inp = make_inputs(shape["b"], shape["L"], shape["H"], shape["P"], shape["N"], shape["R"],
                      shape["G"], "f32", seed=seed, extras=True)
    st = None
    if state:
        st = make_state(shape["b"], shape["H"], shape["P"], shape["N"], shape["R"], seed + 1)
    return inp, st


def _oracle(inp, st):
    if st is None:
        return orc.scan_inputs(inp)
    return orc.scan_inputs(inp, h0=st[0], carry_B0=st[1], carry_x0=st[2])


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("with_state", [False, True])
def test_complex_form_agrees(shape, with_state):
    inp, st = _rand(shape, 21, with_state)
    y, h, _, _ = _oracle(inp, st)
    kw = {} if st is None else dict(h0=st[0], cB0=st[1], cx0=st[2])
    yc, hc = forms.complex_form(inp.dims, inp.arrays(), **kw)
    np.testing.assert_allclose(y, yc, rtol=0, atol=1e-12 * np.abs(yc).max())
    np.testing.assert_allclose(h, hc, rtol=0, atol=1e-12 * np.abs(hc).max())


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("with_state", [False, True])
def test_rope_form_agrees(shape, with_state):
    inp, st = _rand(shape, 22, with_state)
    y, h, _, _ = _oracle(inp, st)
    kw = {} if st is None else dict(h0=st[0], cB0=st[1], cx0=st[2])
    yr, hr = forms.rope_form(inp.dims, inp.arrays(), **kw)
    np.testing.assert_allclose(y, yr, rtol=0, atol=1e-12 * np.abs(yr).max())
    np.testing.assert_allclose(h, hr, rtol=0, atol=1e-12 * np.abs(hr).max())


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("with_state", [False, True])
def test_masked_matrix_form_agrees(shape, with_state):
    inp, st = _rand(shape, 23, with_state)
    y, _, _, _ = _oracle(inp, st)
    kw = {} if st is None else dict(h0=st[0], cB0=st[1], cx0=st[2])
    ym = forms.masked_matrix_form(inp.dims, inp.arrays(), **kw)
    np.testing.assert_allclose(y, ym, rtol=0, atol=1e-12 * np.abs(ym).max())


@pytest.mark.parametrize("Q", [1, 2, 3, 4, 5, 7, 8, 11, 13])
def test_chunked_form_agrees_for_every_chunk(Q):
    shape = dict(b=1, L=13, H=2, P=3, N=4, R=2, G=1)
    inp, st = _rand(shape, 24, True)
    y, h, _, _ = _oracle(inp, st)
    yq, hq = forms.chunked_form(inp.dims, inp.arrays(), Q, h0=st[0], cB0=st[1], cx0=st[2])
    np.testing.assert_allclose(y, yq, rtol=0, atol=1e-12 * np.abs(yq).max())
    np.testing.assert_allclose(h, hq, rtol=0, atol=1e-12 * np.abs(hq).max())


def test_lambda_one_is_exponential_euler():
    inp, _ = _rand(dict(b=1, L=12, H=2, P=3, N=4, R=2, G=1), 25)
    inp.lam[:] = 1.0
    y, _, _, _ = orc.scan_inputs(inp)
    ye = forms.euler_form(inp.dims, inp.arrays())
    np.testing.assert_allclose(y, ye, rtol=0, atol=1e-12 * np.abs(ye).max())


def test_zero_angle_is_real_trapezoid():
    # theta = 0: the page's trapezoid recurrence with a real scalar alpha, written out.
    inp, _ = _rand(dict(b=1, L=9, H=1, P=2, N=4, R=1, G=1), 26)
    inp.theta[:] = 0.0
    a = {k: (None if v is None else v.astype(np.float64)) for k, v in inp.arrays().items()}
    y, _, _, _ = orc.scan_inputs(inp)
    Bb = a["B"][0, :, 0, 0] + a["bias_B"][0, 0]
    Cb = a["C"][0, :, 0, 0] + a["bias_C"][0, 0]
    xs = a["W_x"][0, 0] * a["x"][0, :, 0]
    h = np.zeros((4, 2))
    prev = np.zeros((4, 2))
    for t in range(9):
        dt, A, lam = (float(a[k][0, t, 0]) for k in ("dt", "A", "lam"))
        al = math.exp(dt * A)
        cur = np.outer(Bb[t], xs[t])
        h = al * h + (1 - lam) * dt * al * prev + lam * dt * cur
        yt = a["W_o"][0, 0] * (Cb[t] @ h) + a["D"][0] * a["x"][0, t, 0]
        np.testing.assert_allclose(y[0, t, 0], yt, rtol=1e-13, atol=1e-13)
        prev = cur


def test_previous_token_term_is_width2_convolution():
    # theta = 0: the trapezoid rule equals the exponential-Euler rule driven by a
    # width-2 convolution of the SSM input, u'_t = (gamma_t u_t + alpha_t beta'_t u_{t-1}) / dt_t.
    inp, _ = _rand(dict(b=1, L=9, H=1, P=1, N=4, R=1, G=1), 27)
    inp.theta[:] = 0.0
    a = {k: (None if v is None else v.astype(np.float64)) for k, v in inp.arrays().items()}
    a["bias_B"] = None
    a["W_x"] = a["W_o"] = a["D"] = None
    y, _, _, _ = orc.scan(inp.dims, **a)
    dt, al, lam = a["dt"][0, :, 0].astype(float), np.exp(a["dt"][0, :, 0] * a["A"][0, :, 0]), a["lam"][0, :, 0]
    u = a["B"][0, :, 0, 0].astype(float) * a["x"][0, :, 0, 0][:, None]          # (L, N), P = 1
    uprev = np.vstack([np.zeros((1, 4)), u[:-1]])
    conv = (lam * dt)[:, None] * u + (al * (1 - lam) * dt)[:, None] * uprev
    e = dict(a)
    e["B"] = (conv / dt[:, None]).reshape(a["B"].shape)
    e["x"] = np.ones_like(a["x"])
    ye = forms.euler_form(inp.dims, e)
    np.testing.assert_allclose(y, ye, rtol=0, atol=1e-13 * np.abs(ye).max())


def test_mimo_is_sum_of_siso_updates():
    # Rank-R update = sum over input branches j of rank-one updates; readouts r
    # each see the whole state, so y = sum_{j,r} W_o[r] * SISO(B_j, C_r, W_x[j] x) + D x.
    shape = dict(b=1, L=10, H=2, P=3, N=4, R=3, G=1)
    inp, _ = _rand(shape, 28)
    y, _, _, _ = orc.scan_inputs(inp)
    R = shape["R"]
    total = inp.D[None, None, :, None] * inp.x.astype(float)
    for j in range(R):
        for r in range(R):
            d1 = dict(inp.dims, R=1)
            yj, _, _, _ = orc.scan(d1, inp.x, inp.dt, inp.A, inp.lam, inp.B[:, :, :, j:j + 1],
                                   inp.C[:, :, :, r:r + 1], inp.theta, inp.bias_B[:, j:j + 1],
                                   inp.bias_C[:, r:r + 1], inp.W_x[:, j:j + 1], inp.W_o[:, r:r + 1])
            total += yj
    np.testing.assert_allclose(y, total, rtol=0, atol=1e-12 * np.abs(y).max())


def test_siso_reduction_without_weights():
    # R = 1 with no W_x / W_o: y_t = Cb_t^T h_t and u_t = Bb_t x_t^T (single-input single-output)
    inp, _ = _rand(dict(b=1, L=8, H=1, P=2, N=2, R=1, G=1), 29)
    a = inp.arrays()
    a["W_x"] = a["W_o"] = a["D"] = None
    y, _, _, _ = orc.scan(inp.dims, **a)
    yc, _ = forms.complex_form(inp.dims, a)
    np.testing.assert_allclose(y, yc, rtol=0, atol=1e-13)


# ---------------------------------------------------------------- invariants

def test_linear_in_x():
    inp, _ = _rand(dict(b=1, L=9, H=2, P=3, N=4, R=2, G=1), 30)
    y1, _, _, _ = orc.scan_inputs(inp)
    x1 = inp.x.copy()
    inp2, _ = _rand(dict(b=1, L=9, H=2, P=3, N=4, R=2, G=1), 31)
    inp.x = inp2.x.copy()
    y2, _, _, _ = orc.scan_inputs(inp)
    inp.x = 2.5 * x1.astype(np.float64) - 0.75 * inp2.x.astype(np.float64)
    y3, _, _, _ = orc.scan_inputs(inp)
    np.testing.assert_allclose(y3, 2.5 * y1 - 0.75 * y2, rtol=0, atol=1e-12 * np.abs(y3).max())


@pytest.mark.parametrize("split", [1, 5, 12])
def test_prefill_then_decode_equals_longer_prefill(split):
    shape = dict(b=2, L=13, H=2, P=3, N=4, R=2, G=1)
    inp, st = _rand(shape, 32, True)
    y, h, cB, cx = orc.scan_inputs(inp, h0=st[0], carry_B0=st[1], carry_x0=st[2])
    a = inp.arrays()
    seq = lambda k, s: a[k][:, s] if a[k] is not None and k in ("x", "dt", "A", "lam", "B", "C", "theta") else a[k]
    d1 = dict(inp.dims, L=split)
    ya, ha, cBa, cxa = orc.scan(d1, **{k: seq(k, slice(0, split)) for k in a},
                                h0=st[0], carry_B0=st[1], carry_x0=st[2])
    ys = [ya]
    for t in range(split, shape["L"]):
        dt1 = dict(inp.dims, L=1)
        yt, ha, cBa, cxa = orc.scan(dt1, **{k: seq(k, slice(t, t + 1)) for k in a},
                                    h0=ha, carry_B0=cBa, carry_x0=cxa)
        ys.append(yt)
    np.testing.assert_allclose(np.concatenate(ys, axis=1), y, rtol=0, atol=1e-12 * np.abs(y).max())
    np.testing.assert_allclose(ha, h, rtol=0, atol=1e-12 * np.abs(h).max())
    np.testing.assert_array_equal(cBa, cB)
    np.testing.assert_array_equal(cxa, cx)


def test_selected_pairs_match_full_run():
    inp, st = _rand(dict(b=2, L=7, H=3, P=2, N=4, R=2, G=1), 33, True)
    y, h, _, _ = orc.scan_inputs(inp, h0=st[0], carry_B0=st[1], carry_x0=st[2])
    sel = [(1, 2), (0, 1)]
    ys, hs, _, _ = orc.scan_inputs(inp, sel=sel, h0=st[0], carry_B0=st[1], carry_x0=st[2])
    for bi, hi in sel:
        np.testing.assert_array_equal(ys[bi, :, hi], y[bi, :, hi])
        np.testing.assert_array_equal(hs[bi, hi], h[bi, hi])
    assert np.all(ys[0, :, 0] == 0.0)


def test_empty_sequence_keeps_state():
    inp, st = _rand(dict(b=1, L=0, H=2, P=2, N=4, R=1, G=1), 34, True)
    y, h, cB, cx = orc.scan_inputs(inp, h0=st[0], carry_B0=st[1], carry_x0=st[2])
    assert y.shape == (1, 0, 2, 2)
    np.testing.assert_array_equal(h, st[0])
    np.testing.assert_array_equal(cB, st[1])
    np.testing.assert_array_equal(cx, st[2])


def test_bad_dims_rejected():
    inp, _ = _rand(dict(b=1, L=3, H=2, P=2, N=4, R=1, G=1), 35)
    with pytest.raises(RuntimeError):
        orc.scan(dict(inp.dims, G=3), inp.x, inp.dt, inp.A, inp.lam,
                 np.zeros((1, 3, 3, 1, 4)), np.zeros((1, 3, 3, 1, 4)), np.zeros((1, 3, 3, 2)))


# ------------------------------------------------------------------ direct-angle variant

def test_direct_angle_equals_prescaled_theta():
    # With one head per group, the direct-angle variant fed theta' = dt * theta is the
    # default recurrence fed theta: the rotation of each step is the same angle.
    inp = make_inputs(b=2, L=40, H=3, P=8, N=8, R=2, G=3, dtype="f32", seed=77, extras=True)
    y0, h0, _, _ = orc.scan_inputs(inp)
    direct = make_inputs(b=2, L=40, H=3, P=8, N=8, R=2, G=3, dtype="f32", seed=77, extras=True)
    direct.theta = inp.dt.astype(np.float64)[..., None] * inp.theta.astype(np.float64)
    y1, h1, _, _ = orc.scan_inputs(direct, angle_direct=True)
    np.testing.assert_array_equal(y1, y0)
    np.testing.assert_array_equal(h1, h0)
    # and the flag matters: the same theta as a direct angle gives another result
    y2, _, _, _ = orc.scan_inputs(inp, angle_direct=True)
    assert np.abs(y2 - y0).max() > 1e-3 * np.abs(y0).max()
