"""Python front-end of the fp64 oracle (test infrastructure only).

Only tests/, ``__graft_entry__.smoke()`` and the cpu_baseline / reference legs of
``bench.py`` may import this module.  It loads ``libm3oracle.so`` (built from
``m3_oracle.c`` next to it by ``build()``) and shares nothing with the CUDA path.

``scan`` runs the sequential recurrence documented at the top of m3_oracle.c
(Mamba-3 paper note on docsaid.org, sections その1 / その2 / その3).  Decode is the
same recurrence one token at a time: ``scan`` with L = 1 and the carried state.
"""

from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "m3_oracle.c")
_LIB = os.path.join(_HERE, "libm3oracle.so")
_lib = None


class _Dims(ctypes.Structure):
    _fields_ = [("b", ctypes.c_int64), ("L", ctypes.c_int64), ("H", ctypes.c_int32),
                ("P", ctypes.c_int32), ("N", ctypes.c_int32), ("R", ctypes.c_int32),
                ("G", ctypes.c_int32), ("angle_direct", ctypes.c_int32)]


GRAD_KEYS = ("dx", "ddt", "dA", "dlam", "dB", "dC", "dtheta", "dbias_B", "dbias_C", "dW_x", "dW_o", "dD",
             "dh0", "dcarry_B", "dcarry_x")


class _Grads(ctypes.Structure):
    _fields_ = [(k, ctypes.POINTER(ctypes.c_double)) for k in GRAD_KEYS]


def build(force: bool = False) -> str:
    """Compile m3_oracle.c with gcc (-O2, OpenMP) into libm3oracle.so."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        dp = ctypes.POINTER(ctypes.c_double)
        lib.m3o_scan.restype = ctypes.c_int
        lib.m3o_scan.argtypes = [ctypes.POINTER(_Dims)] + [dp] * 16 + [
            ctypes.POINTER(ctypes.c_int64), ctypes.c_int64, ctypes.c_int]
        lib.m3o_max_threads.restype = ctypes.c_int
        lib.m3o_scan_bwd.restype = ctypes.c_int
        lib.m3o_scan_bwd.argtypes = [ctypes.POINTER(_Dims)] + [dp] * 17 + [ctypes.POINTER(_Grads)]
        _lib = lib
    return _lib


def max_threads() -> int:
    return int(_load().m3o_max_threads())


def _f64(a):
    if a is None:
        return None
    return np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def scan(dims, x, dt, A, lam, B, C, theta, bias_B=None, bias_C=None, W_x=None, W_o=None,
         D=None, h0=None, carry_B0=None, carry_x0=None, sel=None, threads=0, angle_direct=False):
    """Sequential fp64 recurrence.

    dims: mapping with b, L, H, P, N, R, G.  Arrays in the layouts of m3_oracle.c
    (any float dtype; converted exactly to float64).  h0 / carry_*0 default to
    zeros (a fresh state).  sel: optional iterable of (batch, head) pairs; only
    those pairs are computed (others' y rows are zero and their state untouched).
    Returns (y, h, carry_B, carry_x) as float64 arrays.
    """
    lib = _load()
    b, L, H, P, N, R, G = (int(dims[k]) for k in ("b", "L", "H", "P", "N", "R", "G"))
    d = _Dims(b, L, H, P, N, R, G, 1 if angle_direct else 0)
    h = np.zeros((b, H, N, P)) if h0 is None else np.array(h0, dtype=np.float64, copy=True)
    cB = np.zeros((b, H, R, N)) if carry_B0 is None else np.array(carry_B0, dtype=np.float64, copy=True)
    cx = np.zeros((b, H, P)) if carry_x0 is None else np.array(carry_x0, dtype=np.float64, copy=True)
    y = np.zeros((b, L, H, P))
    arrs = [_f64(a) for a in (x, dt, A, lam, B, C, theta, bias_B, bias_C, W_x, W_o, D)]
    shapes = [(b, L, H, P), (b, L, H), (b, L, H), (b, L, H), (b, L, G, R, N), (b, L, G, R, N),
              (b, L, G, N // 2), (H, R, N), (H, R, N), (H, R, P), (H, R, P), (H,)]
    for a, s in zip(arrs, shapes):
        if a is not None and a.shape != s:
            raise ValueError(f"oracle: expected shape {s}, got {a.shape}")
    if sel is not None:
        ids = np.array([int(bi) * H + int(hi) for bi, hi in sel], dtype=np.int64)
        sel_p, nsel = ids.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), len(ids)
    else:
        ids, sel_p, nsel = None, None, 0
    rc = lib.m3o_scan(ctypes.byref(d), *[_ptr(a) for a in arrs], _ptr(h), _ptr(cB), _ptr(cx),
                      _ptr(y), sel_p, nsel, int(threads))
    if rc != 0:
        raise RuntimeError(f"m3o_scan failed with code {rc}")
    return y, h, cB, cx


def scan_inputs(inp, sel=None, threads=0, h0=None, carry_B0=None, carry_x0=None, angle_direct=False):
    """``scan`` on an ``Inputs`` draw from the shared seeded generator."""
    return scan(inp.dims, inp.x, inp.dt, inp.A, inp.lam, inp.B, inp.C, inp.theta, inp.bias_B,
                inp.bias_C, inp.W_x, inp.W_o, inp.D, h0=h0, carry_B0=carry_B0,
                carry_x0=carry_x0, sel=sel, threads=threads, angle_direct=angle_direct)


def scan_bwd(dims, x, dt, A, lam, B, C, theta, bias_B=None, bias_C=None, W_x=None, W_o=None, D=None,
             h0=None, carry_B0=None, carry_x0=None, dy=None, dh_final=None, angle_direct=False):
    """Reverse-mode gradient of ``scan`` (m3o_scan_bwd in m3_oracle.c): the gradients of
    sum(dy * y) + sum(dh_final * h_final) with respect to every operand and the initial state.
    Returns a dict keyed by GRAD_KEYS (float64; None for an operand passed as None)."""
    lib = _load()
    b, L, H, P, N, R, G = (int(dims[k]) for k in ("b", "L", "H", "P", "N", "R", "G"))
    d = _Dims(b, L, H, P, N, R, G, 1 if angle_direct else 0)
    h = np.zeros((b, H, N, P)) if h0 is None else _f64(h0)
    cB = np.zeros((b, H, R, N)) if carry_B0 is None else _f64(carry_B0)
    cx = np.zeros((b, H, P)) if carry_x0 is None else _f64(carry_x0)
    arrs = [_f64(a) for a in (x, dt, A, lam, B, C, theta, bias_B, bias_C, W_x, W_o, D)]
    shapes = {"dx": (b, L, H, P), "ddt": (b, L, H), "dA": (b, L, H), "dlam": (b, L, H), "dB": (b, L, G, R, N),
              "dC": (b, L, G, R, N), "dtheta": (b, L, G, N // 2), "dbias_B": (H, R, N), "dbias_C": (H, R, N),
              "dW_x": (H, R, P), "dW_o": (H, R, P), "dD": (H,), "dh0": (b, H, N, P), "dcarry_B": (b, H, R, N),
              "dcarry_x": (b, H, P)}
    out = {k: np.zeros(v) for k, v in shapes.items()}
    gr = _Grads(*[_ptr(out[k]) for k in GRAD_KEYS])
    rc = lib.m3o_scan_bwd(ctypes.byref(d), *[_ptr(a) for a in arrs], _ptr(h), _ptr(cB), _ptr(cx),
                          _ptr(_f64(dy)), _ptr(_f64(dh_final)), ctypes.byref(gr))
    if rc != 0:
        raise RuntimeError(f"m3o_scan_bwd failed with code {rc}")
    for k, a in (("dbias_B", bias_B), ("dbias_C", bias_C), ("dW_x", W_x), ("dW_o", W_o), ("dD", D)):
        if a is None:
            out[k] = None
    return out


def output_norm(y, z=None, weight=None, eps=1e-6):
    """The hybrid model's output norm (test infrastructure), in float64: per (batch, token,
    head) row of P values, v = y * silu(z) (v = y without a gate), then
    out = weight[h] * v / sqrt(mean_p v^2 + eps).  y, z: (b, L, H, P); weight: (H, P) or None
    (ones).  Mamba-3 paper note (docsaid.org), section アーキテクチャ: the norm before the output
    projection is removed in the pure Mamba-3 model and kept in the hybrid one."""
    v = np.asarray(y, dtype=np.float64)
    if z is not None:
        zz = np.asarray(z, dtype=np.float64)
        v = v * (zz / (1.0 + np.exp(-zz)))
    rms = np.sqrt(np.mean(v * v, axis=-1, keepdims=True) + eps)
    out = v / rms
    if weight is not None:
        out = out * np.asarray(weight, dtype=np.float64)[None, None]
    return out


BCNORM_EPS = 1e-6


def frontend(inp):
    """The block's front-end on a raw draw (test infrastructure), in float64: a copy of the
    draw whose B, C are RMS-normalised over N per (token, group, branch) row (B / sqrt(mean_N
    B^2 + 1e-6), no weight: the QK-norm-like BCNorm of the Cartesia blog and the docsaid note,
    section アーキテクチャ), dt = softplus(dt_raw), A = -exp(A_raw) and lam = sigmoid(lam_raw)
    (the parameterisation of the step, decay and trapezoid weight in section その1's
    discretisation).  The biases are added by the core after the norm."""
    import copy
    out = copy.copy(inp)
    B = np.asarray(inp.B, dtype=np.float64)
    C = np.asarray(inp.C, dtype=np.float64)
    out.B = B / np.sqrt(np.mean(B * B, axis=-1, keepdims=True) + BCNORM_EPS)
    out.C = C / np.sqrt(np.mean(C * C, axis=-1, keepdims=True) + BCNORM_EPS)
    d = np.asarray(inp.dt, dtype=np.float64)
    out.dt = np.logaddexp(0.0, d)
    out.A = -np.exp(np.asarray(inp.A, dtype=np.float64))
    out.lam = 1.0 / (1.0 + np.exp(-np.asarray(inp.lam, dtype=np.float64)))
    out.extra = dict(inp.extra, raw=False)
    return out
