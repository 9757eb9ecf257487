"""Host-side checks of the C ABI: the library loads without a GPU, exports every
symbol include/m3.h declares, and rejects bad arguments before launching anything."""

import ctypes
import os
import re

import pytest

from selective_state_space_53_b200 import build as m3build
from selective_state_space_53_b200 import m3

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    m3build.build()
    return m3.lib()


def _declared():
    src = open(os.path.join(ROOT, "include", "m3.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(m3_[a-z_0-9]+)\s*\(", src)))


def test_every_declared_symbol_is_exported(L):
    names = _declared()
    assert "m3_scan_fwd" in names and "m3_decode_step" in names and "m3_state_alloc" in names
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(m3.SIGNATURES), "binding and header disagree"


def test_status_strings(L):
    assert m3.m3_status_str(0) == "ok"
    assert "aligned" in m3.m3_status_str(-3)
    assert m3.m3_version().startswith("m3")


def _dims(**kw):
    d = dict(b=2, L=5, H=4, P=16, N=16, R=2, G=2, dtype="bf16")
    d.update(kw)
    return m3.make_dims(**d)


@pytest.mark.parametrize("kw,code", [
    (dict(N=15), -1), (dict(N=12), -1), (dict(P=12), -1), (dict(G=3), -1), (dict(R=0), -1),
    (dict(R=9), -1), (dict(P=512), -1), (dict(b=-1), -1), (dict(dtype=7), -2), (dict(flags=8), -1)])
def test_bad_dims_rejected_on_host(L, kw, code):
    d = _dims(**kw)
    n = ctypes.c_size_t()
    assert L.m3_state_bytes(ctypes.byref(d), ctypes.byref(n)) == code
    assert L.m3_scan_workspace_size(ctypes.byref(d), ctypes.byref(n)) == code
    st = ctypes.c_void_p()
    assert L.m3_state_alloc(ctypes.byref(d), None, ctypes.byref(st)) == code


def test_state_bytes(L):
    d = _dims()
    n = ctypes.c_size_t()
    assert L.m3_state_bytes(ctypes.byref(d), ctypes.byref(n)) == 0
    assert n.value == 4 * 2 * 4 * (16 * 16 + 2 * 16 + 16)


def _fake_state(L, d, base=1 << 20):
    st = ctypes.c_void_p()
    assert L.m3_state_wrap(ctypes.byref(d), ctypes.c_void_p(base), ctypes.c_void_p(base + 4096),
                           ctypes.c_void_p(base + 8192), ctypes.byref(st)) == 0
    return st


def test_null_and_alignment_rejected_before_launch(L):
    d = _dims()
    st = _fake_state(L, d)
    ok = ctypes.c_void_p(1 << 24)
    args = [ok] * 7 + [None] * 5
    # missing y
    assert L.m3_scan_fwd(ctypes.byref(d), *args, st, None, None, 0, None) == -4
    # missing x
    assert L.m3_scan_fwd(ctypes.byref(d), None, *args[1:], st, ok, None, 0, None) == -4
    # misaligned B
    bad = list(args)
    bad[4] = ctypes.c_void_p((1 << 24) + 2)
    assert L.m3_scan_fwd(ctypes.byref(d), *bad, st, ok, None, 0, None) == -3
    # misaligned optional W_x
    bad = list(args)
    bad[9] = ctypes.c_void_p((1 << 24) + 8)
    assert L.m3_scan_fwd(ctypes.byref(d), *bad, st, ok, None, 0, None) == -3
    # decode: missing theta
    bad = list(args)
    bad[6] = None
    assert L.m3_decode_step(ctypes.byref(d), *bad, st, ok, None) == -4
    # no state
    assert L.m3_scan_fwd(ctypes.byref(d), *args, None, ok, None, 0, None) == -4
    assert L.m3_state_free(st) == 0


def test_state_dims_mismatch_rejected(L):
    st = _fake_state(L, _dims())
    d2 = _dims(N=32)
    ok = ctypes.c_void_p(1 << 24)
    assert L.m3_scan_fwd(ctypes.byref(d2), *([ok] * 7 + [None] * 5), st, ok, None, 0, None) == -9
    assert L.m3_state_free(st) == 0


def test_empty_batch_or_length_is_noop(L):
    # L = 0 and b = 0 return before touching the device
    for kw in (dict(L=0), dict(b=0)):
        d = _dims(**kw)
        st = _fake_state(L, d)
        assert L.m3_scan_fwd(ctypes.byref(d), *([None] * 12), st, None, None, 0, None) == 0
        assert L.m3_state_free(st) == 0
    d = _dims(b=0)
    st = _fake_state(L, d)
    assert L.m3_decode_step(ctypes.byref(d), *([None] * 12), st, None, None) == 0
    assert L.m3_state_free(st) == 0


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(m3, "LIB_PATH", str(tmp_path / "absent.so"))
    monkeypatch.setattr(m3, "_lib", None)
    with pytest.raises(m3.M3Error):
        m3.lib()


def test_workspace_size_and_missing_workspace(L):
    # a long sequence with few (batch, head) pairs is split into segments that need scratch
    d = m3.make_dims(1, 4096, 2, 64, 64, 2, 1, "bf16")
    n = ctypes.c_size_t()
    assert L.m3_scan_workspace_size(ctypes.byref(d), ctypes.byref(n)) == 0
    assert n.value > 0
    st = _fake_state(L, d)
    ok = ctypes.c_void_p(1 << 24)
    assert L.m3_scan_fwd(ctypes.byref(d), *([ok] * 7 + [None] * 5), st, ok, None, 0, None) == -5
    assert L.m3_scan_fwd(ctypes.byref(d), *([ok] * 7 + [None] * 5), st, ok, ok, n.value - 1, None) == -5
    # the sequential kernel needs none
    d.flags = 1
    assert L.m3_scan_workspace_size(ctypes.byref(d), ctypes.byref(n)) == 0 and n.value == 0
    assert L.m3_state_free(st) == 0
