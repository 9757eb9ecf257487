"""ctypes binding of libm3.so (include/m3.h), argument marshalling only.

Every function takes torch tensors (device memory for tensor operands) and
passes raw pointers, sizes and the current CUDA stream to the C ABI.  All
arithmetic runs in the library's CUDA kernels; there is no other code path.
Loading fails loudly (``M3Error``) when the library is missing.
"""

from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libm3.so")

M3_F32, M3_BF16 = 0, 1
M3_FLAG_SEQUENTIAL = 1
M3_FLAG_ANGLE_DIRECT = 2
M3_FLAG_RAW_INPUTS = 4

_STATUS = {0: "M3_OK", -1: "M3_ERR_DIMS", -2: "M3_ERR_DTYPE", -3: "M3_ERR_ALIGN",
           -4: "M3_ERR_NULL", -5: "M3_ERR_WORKSPACE", -6: "M3_ERR_CUDA", -7: "M3_ERR_TIMEOUT",
           -8: "M3_ERR_UNSUPPORTED", -9: "M3_ERR_STATE"}


class M3Error(RuntimeError):
    def __init__(self, code, what=""):
        self.code = code
        name = _STATUS.get(code, str(code))
        super().__init__(f"{what}: {name}" if what else name)


class Dims(ctypes.Structure):
    _fields_ = [("b", ctypes.c_int64), ("L", ctypes.c_int64), ("H", ctypes.c_int32),
                ("P", ctypes.c_int32), ("N", ctypes.c_int32), ("R", ctypes.c_int32),
                ("G", ctypes.c_int32), ("chunk", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("flags", ctypes.c_uint32)]


_lib = None

# Every symbol include/m3.h declares, with (restype, argtypes).
_VP, _SZ, _I = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
_DP = ctypes.POINTER(Dims)
SIGNATURES = {
    "m3_state_bytes": (_I, [_DP, ctypes.POINTER(_SZ)]),
    "m3_state_alloc": (_I, [_DP, _VP, ctypes.POINTER(_VP)]),
    "m3_state_wrap": (_I, [_DP, _VP, _VP, _VP, ctypes.POINTER(_VP)]),
    "m3_state_free": (_I, [_VP]),
    "m3_state_tensors": (_I, [_VP, ctypes.POINTER(_VP), ctypes.POINTER(_VP), ctypes.POINTER(_VP)]),
    "m3_state_copy_to_host": (_I, [_VP, _VP, _SZ, _VP]),
    "m3_state_copy_from_host": (_I, [_VP, _VP, _SZ, _VP]),
    "m3_scan_workspace_size": (_I, [_DP, ctypes.POINTER(_SZ)]),
    "m3_scan_fwd": (_I, [_DP] + [_VP] * 14 + [_VP, _SZ, _VP]),
    "m3_scan_fwd_noalloc": (_I, [_DP] + [_VP] * 14 + [_VP]),
    "m3_decode_step": (_I, [_DP] + [_VP] * 15),
    "m3_output_norm": (_I, [_DP, _VP, _VP, _VP, ctypes.c_float, _VP, _VP]),
    "m3_frontend": (_I, [_DP] + [_VP] * 10 + [_VP]),
    "m3_scan_bwd_workspace_size": (_I, [_DP, ctypes.POINTER(_SZ)]),
    "m3_scan_bwd": (_I, [_DP] + [_VP] * 12 + [_VP, _VP, _VP, _VP, _VP, _SZ, _VP]),
    "m3_scan_summary_workspace_size": (_I, [_DP, ctypes.POINTER(_SZ)]),
    "m3_scan_summary": (_I, [_DP] + [_VP] * 14 + [_VP, _SZ, _VP]),
    "m3_state_fold": (_I, [_DP, ctypes.c_int32] + [_VP] * 8 + [_VP, _VP]),
    "m3_check": (_I, [_VP]),
    "m3_selftest_wait": (_I, [ctypes.c_uint64, _VP]),
    "m3_status_str": (ctypes.c_char_p, [_I]),
    "m3_version": (ctypes.c_char_p, []),
    "m3_last_error": (ctypes.c_char_p, []),
}


def lib():
    """Load libm3.so once; raise M3Error if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise M3Error(-6, f"{LIB_PATH} not built (python -m selective_state_space_53_b200.build)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(code, what):
    if code != 0:
        if code == -6:
            what = f"{what} ({lib().m3_last_error().decode()})"
        raise M3Error(code, what)


def make_dims(b, L, H, P, N, R, G=1, dtype="bf16", chunk=32, flags=0) -> Dims:
    dt = {"bf16": M3_BF16, "f32": M3_F32}[dtype] if isinstance(dtype, str) else int(dtype)
    return Dims(int(b), int(L), int(H), int(P), int(N), int(R), int(G), int(chunk), dt, int(flags))


def _ptr(t):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


class State:
    """An m3_state handle.  ``State.wrap`` keeps torch tensors as the storage."""

    def __init__(self, handle, dims, keep=None):
        self.handle = handle
        self.dims = dims
        self._keep = keep

    @classmethod
    def alloc(cls, dims: Dims, stream=None):
        h = ctypes.c_void_p()
        _check(lib().m3_state_alloc(ctypes.byref(dims), _stream(stream), ctypes.byref(h)), "m3_state_alloc")
        return cls(h, dims)

    @classmethod
    def wrap(cls, dims: Dims, h, carry_B, carry_x):
        hd = ctypes.c_void_p()
        _check(lib().m3_state_wrap(ctypes.byref(dims), _ptr(h), _ptr(carry_B), _ptr(carry_x),
                                   ctypes.byref(hd)), "m3_state_wrap")
        return cls(hd, dims, keep=(h, carry_B, carry_x))

    def nbytes(self) -> int:
        n = ctypes.c_size_t()
        _check(lib().m3_state_bytes(ctypes.byref(self.dims), ctypes.byref(n)), "m3_state_bytes")
        return n.value

    def to_host(self, stream=None):
        import numpy as np
        buf = np.empty(self.nbytes() // 4, dtype=np.float32)
        _check(lib().m3_state_copy_to_host(self.handle, buf.ctypes.data_as(ctypes.c_void_p), buf.nbytes,
                                           _stream(stream)), "m3_state_copy_to_host")
        return buf

    def from_host(self, buf, stream=None):
        import numpy as np
        buf = np.ascontiguousarray(buf, dtype=np.float32)
        _check(lib().m3_state_copy_from_host(self.handle, buf.ctypes.data_as(ctypes.c_void_p), buf.nbytes,
                                             _stream(stream)), "m3_state_copy_from_host")

    def tensors(self):
        """(h, carry_B, carry_x) device pointers as ints."""
        a, b, c = ctypes.c_void_p(), ctypes.c_void_p(), ctypes.c_void_p()
        _check(lib().m3_state_tensors(self.handle, ctypes.byref(a), ctypes.byref(b), ctypes.byref(c)),
               "m3_state_tensors")
        return a.value, b.value, c.value

    def free(self):
        if self.handle is not None and self.handle.value:
            _check(lib().m3_state_free(self.handle), "m3_state_free")
        self.handle = None
        self._keep = None

    def __del__(self):
        try:
            if self.handle is not None and self.handle.value:
                lib().m3_state_free(self.handle)
        except Exception:
            pass


def m3_scan_workspace_size(dims: Dims) -> int:
    n = ctypes.c_size_t()
    _check(lib().m3_scan_workspace_size(ctypes.byref(dims), ctypes.byref(n)), "m3_scan_workspace_size")
    return n.value


def m3_scan_fwd(dims: Dims, x, dt, A, lam, B, C, theta, bias_B, bias_C, W_x, W_o, D, state: State, y,
                workspace=None, stream=None):
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().m3_scan_fwd(ctypes.byref(dims), _ptr(x), _ptr(dt), _ptr(A), _ptr(lam), _ptr(B), _ptr(C),
                             _ptr(theta), _ptr(bias_B), _ptr(bias_C), _ptr(W_x), _ptr(W_o), _ptr(D),
                             state.handle, _ptr(y), _ptr(workspace), ws_bytes, _stream(stream)),
           "m3_scan_fwd")


def m3_scan_fwd_noalloc(dims: Dims, x, dt, A, lam, B, C, theta, bias_B, bias_C, W_x, W_o, D, state: State, y,
                        stream=None):
    """m3_scan_fwd without a workspace: the library's fixed 16 MiB device scratch is used
    (for callers that cannot allocate; calls overlapping on the GPU race on it)."""
    _check(lib().m3_scan_fwd_noalloc(ctypes.byref(dims), _ptr(x), _ptr(dt), _ptr(A), _ptr(lam), _ptr(B), _ptr(C),
                                     _ptr(theta), _ptr(bias_B), _ptr(bias_C), _ptr(W_x), _ptr(W_o), _ptr(D),
                                     state.handle, _ptr(y), _stream(stream)), "m3_scan_fwd_noalloc")


def m3_decode_step(dims: Dims, x_t, dt_t, A_t, lam_t, B_t, C_t, theta_t, bias_B, bias_C, W_x, W_o, D,
                   state: State, y_t, stream=None):
    _check(lib().m3_decode_step(ctypes.byref(dims), _ptr(x_t), _ptr(dt_t), _ptr(A_t), _ptr(lam_t), _ptr(B_t),
                                _ptr(C_t), _ptr(theta_t), _ptr(bias_B), _ptr(bias_C), _ptr(W_x), _ptr(W_o),
                                _ptr(D), state.handle, _ptr(y_t), _stream(stream)), "m3_decode_step")


def m3_scan_summary_workspace_size(dims: Dims) -> int:
    n = ctypes.c_size_t()
    _check(lib().m3_scan_summary_workspace_size(ctypes.byref(dims), ctypes.byref(n)),
           "m3_scan_summary_workspace_size")
    return n.value


def m3_scan_summary(dims: Dims, x, dt, A, lam, B, theta, bias_B, W_x, Z, logdec, angle, bp_first, carry_B,
                    carry_x, workspace, stream=None):
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib().m3_scan_summary(ctypes.byref(dims), _ptr(x), _ptr(dt), _ptr(A), _ptr(lam), _ptr(B), _ptr(theta),
                                 _ptr(bias_B), _ptr(W_x), _ptr(Z), _ptr(logdec), _ptr(angle), _ptr(bp_first),
                                 _ptr(carry_B), _ptr(carry_x), _ptr(workspace), ws_bytes, _stream(stream)),
           "m3_scan_summary")


def m3_state_fold(dims: Dims, nranges: int, Z, logdec, angle, bp_first, carry_B, carry_x, bias_B, W_x,
                  state: State, stream=None):
    _check(lib().m3_state_fold(ctypes.byref(dims), int(nranges), _ptr(Z), _ptr(logdec), _ptr(angle),
                               _ptr(bp_first), _ptr(carry_B), _ptr(carry_x), _ptr(bias_B), _ptr(W_x),
                               state.handle, _stream(stream)), "m3_state_fold")


def m3_frontend(dims: Dims, B_raw, C_raw, dt_raw, A_raw, lam_raw, B, C, dt, A, lam, stream=None):
    _check(lib().m3_frontend(ctypes.byref(dims), _ptr(B_raw), _ptr(C_raw), _ptr(dt_raw), _ptr(A_raw), _ptr(lam_raw),
                             _ptr(B), _ptr(C), _ptr(dt), _ptr(A), _ptr(lam), _stream(stream)), "m3_frontend")


def m3_output_norm(dims: Dims, y, z, weight, eps, out, stream=None):
    _check(lib().m3_output_norm(ctypes.byref(dims), _ptr(y), _ptr(z), _ptr(weight), float(eps), _ptr(out),
                                _stream(stream)), "m3_output_norm")


GRAD_KEYS = ("dx", "ddt", "dA", "dlam", "dB", "dC", "dtheta", "dbias_B", "dbias_C", "dW_x", "dW_o", "dD",
             "dh0", "dcarry_B", "dcarry_x")


class Grads(ctypes.Structure):
    """m3_grads: device pointers of the gradients (None where not wanted)."""
    _fields_ = [(k, ctypes.c_void_p) for k in GRAD_KEYS]


def m3_scan_bwd_workspace_size(dims: Dims) -> int:
    n = ctypes.c_size_t()
    _check(lib().m3_scan_bwd_workspace_size(ctypes.byref(dims), ctypes.byref(n)), "m3_scan_bwd_workspace_size")
    return n.value


def m3_scan_bwd(dims: Dims, x, dt, A, lam, B, C, theta, bias_B, bias_C, W_x, W_o, D, state0: State, dy,
                dh_final, grads: dict, workspace=None, stream=None):
    g = Grads(*[(None if grads.get(k) is None else grads[k].data_ptr()) for k in GRAD_KEYS])
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().m3_scan_bwd(ctypes.byref(dims), _ptr(x), _ptr(dt), _ptr(A), _ptr(lam), _ptr(B), _ptr(C),
                             _ptr(theta), _ptr(bias_B), _ptr(bias_C), _ptr(W_x), _ptr(W_o), _ptr(D), state0.handle,
                             _ptr(dy), _ptr(dh_final), ctypes.byref(g), _ptr(workspace), ws_bytes, _stream(stream)),
           "m3_scan_bwd")


def scan_backward(dims: Dims, dev: dict, state0: State, dy, dh_final=None, stream=None):
    """m3_scan_bwd on a dict from ``to_device``: allocates the gradients (every one of them) and
    the workspace; returns the gradients keyed by GRAD_KEYS."""
    import torch
    d = dev["x"].device
    b, L, H, P, N, R, G = dims.b, dims.L, dims.H, dims.P, dims.N, dims.R, dims.G
    f32 = dict(dtype=torch.float32, device=d)
    out = {"dx": torch.empty_like(dev["x"]), "ddt": torch.empty((b, L, H), **f32), "dA": torch.empty((b, L, H), **f32),
           "dlam": torch.empty((b, L, H), **f32), "dB": torch.empty_like(dev["B"]), "dC": torch.empty_like(dev["C"]),
           "dtheta": torch.empty((b, L, G, N // 2), **f32), "dbias_B": torch.empty((H, R, N), **f32),
           "dbias_C": torch.empty((H, R, N), **f32), "dW_x": torch.empty((H, R, P), **f32),
           "dW_o": torch.empty((H, R, P), **f32), "dD": torch.empty((H,), **f32),
           "dh0": torch.empty((b, H, N, P), **f32), "dcarry_B": torch.empty((b, H, R, N), **f32),
           "dcarry_x": torch.empty((b, H, P), **f32)}
    n = m3_scan_bwd_workspace_size(dims)
    ws = torch.empty(max(n, 16), dtype=torch.uint8, device=d)
    m3_scan_bwd(dims, *[dev[k] for k in _OPERANDS], state0, dy, dh_final, out, workspace=ws, stream=stream)
    return out


def m3_check(stream=None) -> int:
    return int(lib().m3_check(_stream(stream)))


def m3_selftest_wait(limit_ns: int, stream=None):
    _check(lib().m3_selftest_wait(int(limit_ns), _stream(stream)), "m3_selftest_wait")


def m3_status_str(code: int) -> str:
    return lib().m3_status_str(int(code)).decode()


def m3_version() -> str:
    return lib().m3_version().decode()


# ---- marshalling helpers: seeded host draws -> device tensors

_OPERANDS = ("x", "dt", "A", "lam", "B", "C", "theta", "bias_B", "bias_C", "W_x", "W_o", "D")


def to_device(inp, device="cuda"):
    """Copy an ``inputs.Inputs`` draw to the device in its storage dtypes
    (x, B, C in the draw's dtype; everything else fp32).  Returns a dict."""
    import torch
    tdt = torch.bfloat16 if inp.dims["dtype"] == "bf16" else torch.float32
    out = {}
    for k in _OPERANDS:
        a = getattr(inp, k)
        if a is None:
            out[k] = None
            continue
        t = torch.from_numpy(a)
        if k in ("x", "B", "C"):
            t = t.to(tdt)
        out[k] = t.to(device).contiguous()
    return out


def dims_of(inp, L=None, flags=0, b=None) -> Dims:
    d = inp.dims
    return make_dims(d["b"] if b is None else b, d["L"] if L is None else L, d["H"], d["P"], d["N"], d["R"],
                     d["G"], d["dtype"], flags=flags)


def state_tensors(dims: Dims, device="cuda", h=None, carry_B=None, carry_x=None):
    """Torch-owned state buffers (zeros unless given) and their m3_state handle."""
    import torch
    b, H, N, P, R = dims.b, dims.H, dims.N, dims.P, dims.R
    th = torch.zeros((b, H, N, P), dtype=torch.float32, device=device) if h is None else \
        torch.as_tensor(h, dtype=torch.float32).to(device).contiguous()
    tb = torch.zeros((b, H, R, N), dtype=torch.float32, device=device) if carry_B is None else \
        torch.as_tensor(carry_B, dtype=torch.float32).to(device).contiguous()
    tx = torch.zeros((b, H, P), dtype=torch.float32, device=device) if carry_x is None else \
        torch.as_tensor(carry_x, dtype=torch.float32).to(device).contiguous()
    return State.wrap(dims, th, tb, tx), (th, tb, tx)


def scan(dims: Dims, dev: dict, state: State, y=None, workspace=None, stream=None):
    """m3_scan_fwd on a dict from ``to_device``; allocates y if not given."""
    import torch
    if y is None:
        y = torch.empty_like(dev["x"])
    if workspace is None:
        n = m3_scan_workspace_size(dims)
        workspace = torch.empty(n, dtype=torch.uint8, device=dev["x"].device) if n else None
    m3_scan_fwd(dims, *[dev[k] for k in _OPERANDS], state, y, workspace=workspace, stream=stream)
    return y


def decode(dims: Dims, tok: dict, state: State, y=None, stream=None):
    """m3_decode_step on one token's operands (dict with x (b,H,P), dt (b,H), ...)."""
    import torch
    if y is None:
        y = torch.empty_like(tok["x"])
    m3_decode_step(dims, *[tok[k] for k in _OPERANDS], state, y, stream=stream)
    return y
