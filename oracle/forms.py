"""Independent fp64 forms of the Mamba-3 SSM core, used to pin the oracle.

TEST INFRASTRUCTURE ONLY (tests/ import it; nothing on the product path does).
Each function computes the same layer output as ``oracle.scan`` by a different
route that the pages state or imply, so that a mistake in the sequential C
recurrence (a dropped term, a wrong sign or index, a transposed operand) shows
up as a disagreement.  All are written for tiny inputs: plain numpy, per
(batch, head) Python loops.

Sources, Mamba-3 paper note (docsaid.org):
  * section その1: exponential-Euler rule h_t = e^{dt A} h_{t-1} + dt B_t x_t and
    the trapezoid generalisation with alpha, beta, gamma; lam = 1 gives back
    the Euler rule;
  * section その2, statement 1: a complex SSM equals a real SSM of doubled size
    (complex_form below runs it in complex arithmetic);
  * section その2, statement 2: absorbing the cumulative rotation into B and C is
    a data-dependent RoPE (rope_form);
  * section その3: MIMO rank-R update, same state size.
  * IBM page on Mamba, Mamba-2 / SSD section: the scan has a matrix
    (attention-like) form and can be split into chunks (masked_matrix_form,
    chunked_form).
"""

from __future__ import annotations

import numpy as np


def _get(inp, name, shape, default):
    a = inp.get(name)
    if a is None:
        return np.full(shape, default, dtype=np.float64)
    return np.asarray(a, dtype=np.float64)


def _unpack(dims, arrays):
    b, L, H, P, N, R, G = (int(dims[k]) for k in ("b", "L", "H", "P", "N", "R", "G"))
    f = {k: (None if arrays.get(k) is None else np.asarray(arrays[k], dtype=np.float64))
         for k in ("x", "dt", "A", "lam", "B", "C", "theta")}
    f["bias_B"] = _get(arrays, "bias_B", (H, R, N), 0.0)
    f["bias_C"] = _get(arrays, "bias_C", (H, R, N), 0.0)
    f["W_x"] = _get(arrays, "W_x", (H, R, P), 1.0)
    f["W_o"] = _get(arrays, "W_o", (H, R, P), 1.0)
    f["D"] = _get(arrays, "D", (H,), 0.0)
    return (b, L, H, P, N, R, G), f


def _head_inputs(f, dims7, bi, hi, h0, cB0, cx0):
    """Per-token quantities of one (batch, head): biased B/C, branches X, coefficients."""
    b, L, H, P, N, R, G = dims7
    g = hi // (H // G)
    Bb = f["B"][bi, :, g] + f["bias_B"][hi][None]            # (L, R, N)
    Cb = f["C"][bi, :, g] + f["bias_C"][hi][None]            # (L, R, N)
    X = f["W_x"][hi][None] * f["x"][bi, :, hi][:, None, :]   # (L, R, P)
    Bp = cB0[bi, hi] + f["bias_B"][hi]                       # (R, N) previous token
    Xp = f["W_x"][hi] * cx0[bi, hi][None, :]                 # (R, P)
    dt = f["dt"][bi, :, hi]
    a = dt * f["A"][bi, :, hi]                               # log alpha
    lam = f["lam"][bi, :, hi]
    phi = dt[:, None] * f["theta"][bi, :, g]                 # (L, N/2)
    return Bb, Cb, X, Bp, Xp, a, (1.0 - lam) * dt, lam * dt, phi


def _combine(f, hi, Y, x_bh):
    """y_t = sum_r W_o[h, r] * Y_{t, r} + D_h x_t."""
    return np.einsum("rp,lrp->lp", f["W_o"][hi], Y) + f["D"][hi] * x_bh


def _state_defaults(dims7, h0, cB0, cx0):
    b, L, H, P, N, R, G = dims7
    h0 = np.zeros((b, H, N, P)) if h0 is None else np.asarray(h0, dtype=np.float64)
    cB0 = np.zeros((b, H, R, N)) if cB0 is None else np.asarray(cB0, dtype=np.float64)
    cx0 = np.zeros((b, H, P)) if cx0 is None else np.asarray(cx0, dtype=np.float64)
    return h0, cB0, cx0


def complex_form(dims, arrays, h0=None, cB0=None, cx0=None):
    """The layer run as a complex-valued SSM with N/2 complex state rows.

    State rows (2k, 2k+1) are the real and imaginary parts of complex row k;
    the transition is the scalar e^{dt (A + i theta)}; readout is Re(conj(c) . z).
    Returns (y, h) with h converted back to the real (2k, 2k+1) layout.
    """
    dims7, f = _unpack(dims, arrays)
    b, L, H, P, N, R, G = dims7
    h0, cB0, cx0 = _state_defaults(dims7, h0, cB0, cx0)
    y = np.zeros((b, L, H, P))
    hout = np.zeros((b, H, N, P))
    for bi in range(b):
        for hi in range(H):
            Bb, Cb, X, Bp, Xp, a, bp, gm, phi = _head_inputs(f, dims7, bi, hi, h0, cB0, cx0)
            bz = Bb[..., 0::2] + 1j * Bb[..., 1::2]          # (L, R, N/2)
            cz = Cb[..., 0::2] + 1j * Cb[..., 1::2]
            bpz = Bp[:, 0::2] + 1j * Bp[:, 1::2]
            z = h0[bi, hi, 0::2] + 1j * h0[bi, hi, 1::2]     # (N/2, P)
            vprev = np.einsum("rk,rp->kp", bpz, Xp)
            Y = np.zeros((L, R, P))
            for t in range(L):
                v = np.einsum("rk,rp->kp", bz[t], X[t])
                lam_c = np.exp(a[t] + 1j * phi[t])[:, None]  # e^{dt (A + i theta)}
                z = lam_c * (z + bp[t] * vprev) + gm[t] * v
                Y[t] = np.real(np.einsum("rk,kp->rp", np.conj(cz[t]), z))
                vprev = v
            y[bi, :, hi] = _combine(f, hi, Y, f["x"][bi, :, hi])
            hout[bi, hi, 0::2] = z.real
            hout[bi, hi, 1::2] = z.imag
    return y, hout


def _rot_minus(v, ang):
    """Rotate adjacent pairs (2k, 2k+1) of the last axis of v by -ang[..., k]."""
    c, s = np.cos(ang), np.sin(ang)
    out = np.empty_like(v)
    out[..., 0::2] = c * v[..., 0::2] + s * v[..., 1::2]
    out[..., 1::2] = -s * v[..., 0::2] + c * v[..., 1::2]
    return out


def rope_form(dims, arrays, h0=None, cB0=None, cx0=None):
    """RoPE-absorbed real form: rotate B and C by the cumulative angle, then a
    real scalar-decay trapezoid scan.  Returns (y, h) with h rotated back."""
    dims7, f = _unpack(dims, arrays)
    b, L, H, P, N, R, G = dims7
    h0, cB0, cx0 = _state_defaults(dims7, h0, cB0, cx0)
    y = np.zeros((b, L, H, P))
    hout = np.zeros((b, H, N, P))
    for bi in range(b):
        for hi in range(H):
            Bb, Cb, X, Bp, Xp, a, bp, gm, phi = _head_inputs(f, dims7, bi, hi, h0, cB0, cx0)
            Phi = np.cumsum(phi, axis=0)                               # (L, N/2)
            Bt = _rot_minus(Bb, Phi[:, None, :])
            Ct = _rot_minus(Cb, Phi[:, None, :])
            ut = np.einsum("lrn,lrp->lnp", Bt, X)                      # rotated u_t
            uprev = np.einsum("rn,rp->np", Bp, Xp)                     # frame of step -1 (angle 0)
            ht = h0[bi, hi].copy()
            Y = np.zeros((L, R, P))
            for t in range(L):
                prev = uprev if t == 0 else ut[t - 1]
                ht = np.exp(a[t]) * (ht + bp[t] * prev) + gm[t] * ut[t]
                Y[t] = Ct[t] @ ht
            y[bi, :, hi] = _combine(f, hi, Y, f["x"][bi, :, hi])
            if L > 0:
                c, s = np.cos(Phi[-1])[:, None], np.sin(Phi[-1])[:, None]
                hr = np.empty_like(ht)
                hr[0::2] = c * ht[0::2] - s * ht[1::2]
                hr[1::2] = s * ht[0::2] + c * ht[1::2]
                hout[bi, hi] = hr
            else:
                hout[bi, hi] = ht
    return y, hout


def masked_matrix_form(dims, arrays, h0=None, cB0=None, cx0=None):
    """Materialised (L R) x (L R) masked matrix times X, plus the initial-state term.

    Y_{t,r} = sum_{s<=t} Lam[t,s] w[t,s] sum_{r'} (Ct_{t,r} . Bt_{s,r'}) X_{s,r'}
              + Lam[t,-1] Ct_{t,r} . hplus,
    Lam[t,s] = prod_{k=s+1..t} alpha_k,  w[t,s] = gamma_s + [s<t] beta'_{s+1},
    hplus = h_{-1} + beta'_0 u_{-1}.  Brute force, O(L^2); tiny inputs only.
    """
    dims7, f = _unpack(dims, arrays)
    b, L, H, P, N, R, G = dims7
    h0, cB0, cx0 = _state_defaults(dims7, h0, cB0, cx0)
    y = np.zeros((b, L, H, P))
    for bi in range(b):
        for hi in range(H):
            Bb, Cb, X, Bp, Xp, a, bp, gm, phi = _head_inputs(f, dims7, bi, hi, h0, cB0, cx0)
            Phi = np.cumsum(phi, axis=0)
            Bt = _rot_minus(Bb, Phi[:, None, :]).reshape(L * R, N)
            Ct = _rot_minus(Cb, Phi[:, None, :]).reshape(L * R, N)
            cum = np.concatenate([[0.0], np.cumsum(a)])               # cum[t+1] = sum_{k<=t} log alpha_k
            M = np.zeros((L, L))
            for t in range(L):
                for s in range(t + 1):
                    w = gm[s] + (bp[s + 1] if s < t else 0.0)
                    M[t, s] = np.exp(cum[t + 1] - cum[s + 1]) * w
            Mfull = np.kron(M, np.ones((R, R)))                        # row (t,r), col (s,r')
            S = (Ct @ Bt.T) * Mfull
            Y = S @ X.reshape(L * R, P)
            hplus = h0[bi, hi] + (bp[0] * np.einsum("rn,rp->np", Bp, Xp) if L > 0 else 0.0)
            decay0 = np.exp(cum[1:])                                   # Lam[t, -1]
            Y = Y + decay0.repeat(R)[:, None] * (Ct @ hplus)
            y[bi, :, hi] = _combine(f, hi, Y.reshape(L, R, P), f["x"][bi, :, hi])
    return y


def chunked_form(dims, arrays, Q, h0=None, cB0=None, cx0=None):
    """Chunked scan with chunk length Q: within a chunk the masked matrix form with
    chunk-local decay and angle; across chunks the carried state
    hplus = h_{c0-1} + beta'_{c0} u_{c0-1}, rotated into each chunk's local frame.
    Returns (y, h)."""
    dims7, f = _unpack(dims, arrays)
    b, L, H, P, N, R, G = dims7
    h0, cB0, cx0 = _state_defaults(dims7, h0, cB0, cx0)
    y = np.zeros((b, L, H, P))
    hout = np.zeros((b, H, N, P))
    for bi in range(b):
        for hi in range(H):
            Bb, Cb, X, Bp, Xp, a, bp, gm, phi = _head_inputs(f, dims7, bi, hi, h0, cB0, cx0)
            h = h0[bi, hi].copy()                       # true-frame state h_{c0-1}
            uprev = np.einsum("rn,rp->np", Bp, Xp)      # u_{c0-1}, true frame
            Y = np.zeros((L, R, P))
            for c0 in range(0, L, Q):
                c1 = min(L, c0 + Q)
                q = c1 - c0
                hplus = h + bp[c0] * uprev
                Phl = np.cumsum(phi[c0:c1], axis=0)     # chunk-local angles
                Bt = _rot_minus(Bb[c0:c1], Phl[:, None, :])
                Ct = _rot_minus(Cb[c0:c1], Phl[:, None, :])
                cum = np.concatenate([[0.0], np.cumsum(a[c0:c1])])
                M = np.zeros((q, q))
                for t in range(q):
                    for s in range(t + 1):
                        w = gm[c0 + s] + (bp[c0 + s + 1] if s < t else 0.0)
                        M[t, s] = np.exp(cum[t + 1] - cum[s + 1]) * w
                S = (Ct.reshape(q * R, N) @ Bt.reshape(q * R, N).T) * np.kron(M, np.ones((R, R)))
                Yc = S @ X[c0:c1].reshape(q * R, P)
                Yc += np.exp(cum[1:]).repeat(R)[:, None] * (Ct.reshape(q * R, N) @ hplus)
                Y[c0:c1] = Yc.reshape(q, R, P)
                # end-of-chunk state in the local frame, then rotated back to the true frame
                wend = np.array([np.exp(cum[q] - cum[s + 1]) * (gm[c0 + s] + (bp[c0 + s + 1] if s < q - 1 else 0.0))
                                 for s in range(q)])
                ht = np.exp(cum[q]) * hplus + np.einsum("s,srn,srp->np", wend, Bt, X[c0:c1])
                cth, sth = np.cos(Phl[-1])[:, None], np.sin(Phl[-1])[:, None]
                h = np.empty_like(ht)
                h[0::2] = cth * ht[0::2] - sth * ht[1::2]
                h[1::2] = sth * ht[0::2] + cth * ht[1::2]
                uprev = np.einsum("rn,rp->np", Bb[c1 - 1], X[c1 - 1])
            y[bi, :, hi] = _combine(f, hi, Y, f["x"][bi, :, hi])
            hout[bi, hi] = h
    return y, hout


def euler_form(dims, arrays, h0=None):
    """The exponential-Euler rule h_t = e^{dt A} Rot(phi) h_{t-1} + dt u_t (lam = 1 case)."""
    dims7, f = _unpack(dims, arrays)
    b, L, H, P, N, R, G = dims7
    h0, cB0, cx0 = _state_defaults(dims7, h0, None, None)
    y = np.zeros((b, L, H, P))
    for bi in range(b):
        for hi in range(H):
            Bb, Cb, X, Bp, Xp, a, bp, gm, phi = _head_inputs(f, dims7, bi, hi, h0, cB0, cx0)
            dt = f["dt"][bi, :, hi]
            h = h0[bi, hi].copy()
            Y = np.zeros((L, R, P))
            for t in range(L):
                c, s = np.cos(phi[t])[:, None], np.sin(phi[t])[:, None]
                hr = np.empty_like(h)
                hr[0::2] = c * h[0::2] - s * h[1::2]
                hr[1::2] = s * h[0::2] + c * h[1::2]
                h = np.exp(a[t]) * hr + dt[t] * np.einsum("rn,rp->np", Bb[t], X[t])
                Y[t] = Cb[t] @ h
            y[bi, :, hi] = _combine(f, hi, Y, f["x"][bi, :, hi])
    return y
