"""Mutation check of the oracle's pins (CPU).

A pin is only worth something if a plausible mistake in the oracle makes it fail.  Each
case below plants one such mistake in a copy of oracle/m3_oracle.c (a wrong sign, a
dropped term, a swapped coefficient, a wrong index), builds the copy in a temporary
directory, and runs the pin suites (tests/test_oracle_pins.py and the finite-difference pins of
the backward pass, tests/test_oracle_grad.py) against it in a child process; they must fail.
The unmodified copy must pass, so that a failure means the planted mistake was caught and not
that the harness is broken.

The mistakes follow the recurrence the oracle states (Mamba-3 paper note, docsaid.org:
section その1 for the trapezoid coefficients and the previous-token term, その2 for the
rotation of adjacent state pairs by dt * theta, その3 for the MIMO branches; the IBM page
on Mamba for the D skip term).
"""

import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PINS = [os.path.join(ROOT, "tests", "test_oracle_pins.py"), os.path.join(ROOT, "tests", "test_oracle_grad.py")]
BWD = "static int bwd_one("  # the backward pass follows the forward recurrence in the file

# (name, text in m3_oracle.c, replacement); the first occurrence of the text is replaced
MUTANTS = [
    ("rotation_sign", "h0[p] = alpha * (c * v0 - s * v1)", "h0[p] = alpha * (c * v0 + s * v1)"),
    ("beta_without_rotation",
     "const double v0 = h0[p] + bprime * q0[p];\n        const double v1 = h1[p] + bprime * q1[p];\n"
     "        h0[p] = alpha * (c * v0 - s * v1) + gamma * u0[p];\n"
     "        h1[p] = alpha * (s * v0 + c * v1) + gamma * u1[p];",
     "const double v0 = h0[p];\n        const double v1 = h1[p];\n"
     "        h0[p] = alpha * (c * v0 - s * v1) + gamma * u0[p] + alpha * bprime * q0[p];\n"
     "        h1[p] = alpha * (s * v0 + c * v1) + gamma * u1[p] + alpha * bprime * q1[p];"),
    ("bias_B_dropped", "Bb[r * N + n] = Bt[r * N + n] + bb;", "Bb[r * N + n] = Bt[r * N + n];"),
    ("bias_C_dropped", "Cb[r * N + n] = Ct[r * N + n] + bc;", "Cb[r * N + n] = Ct[r * N + n];"),
    ("gamma_beta_swapped",
     "const double bprime = (1.0 - lm) * delta;\n    const double gamma = lm * delta;",
     "const double bprime = lm * delta;\n    const double gamma = (1.0 - lm) * delta;"),
    ("carry_not_updated", "memcpy(cB, Bt, sizeof(double) * (size_t)R * N);", "/* carry of B kept */"),
    ("W_o_rank_reversed", "W_o[((int64_t)hi * R + r) * P + p]", "W_o[((int64_t)hi * R + (R - 1 - r)) * P + p]"),
    ("pairs_split_in_halves",
     "double* h0 = hs + (int64_t)(2 * k) * P;\n      double* h1 = hs + (int64_t)(2 * k + 1) * P;\n"
     "      const double* u0 = u + (int64_t)(2 * k) * P;\n      const double* u1 = u + (int64_t)(2 * k + 1) * P;\n"
     "      const double* q0 = up + (int64_t)(2 * k) * P;\n      const double* q1 = up + (int64_t)(2 * k + 1) * P;",
     "double* h0 = hs + (int64_t)(k) * P;\n      double* h1 = hs + (int64_t)(k + K) * P;\n"
     "      const double* u0 = u + (int64_t)(k) * P;\n      const double* u1 = u + (int64_t)(k + K) * P;\n"
     "      const double* q0 = up + (int64_t)(k) * P;\n      const double* q1 = up + (int64_t)(k + K) * P;"),
    ("group_index_modulo", "const int32_t g = hi / (H / G);", "const int32_t g = hi % G;"),
    ("angle_without_dt", "d->angle_direct ? th[k] : delta * th[k]", "d->angle_direct ? th[k] : th[k]"),
    ("decay_without_dt", "const double alpha = exp(delta * a);", "const double alpha = exp(a);"),
    ("skip_term_dropped", "yt[p] = s + dh * xt[p];", "yt[p] = s;"),
    # the backward pass (pinned by the finite-difference tests)
    ("bwd_rotation_transpose", "dz[i0] = c * dm0 + s * dm1;", "dz[i0] = c * dm0 - s * dm1;"),
    ("bwd_previous_input_dropped", "duN[i] = bprime * dz[i];", "duN[i] = 0.0 * dz[i];"),
    ("bwd_lambda_beta_term_dropped", "gr->dlam[tok * H + hi] += (dgamma - dbp) * delta;",
     "gr->dlam[tok * H + hi] += dgamma * delta;"),
]


def _run_pins(tmp_path, name, src_text):
    """Copy oracle/ with m3_oracle.c replaced by src_text, build it, run the pins on it."""
    work = tmp_path / name
    pkg = work / "oracle"
    shutil.copytree(os.path.join(ROOT, "oracle"), pkg,
                    ignore=shutil.ignore_patterns("*.so", "__pycache__", "*.tmp*"))
    (pkg / "m3_oracle.c").write_text(src_text)
    env = dict(os.environ)
    # the copy comes first on the path; the repository root provides everything else
    env["PYTHONPATH"] = os.pathsep.join([str(work), ROOT])
    cmd = [sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider", *PINS]
    return subprocess.run(cmd, cwd=str(work), env=env, capture_output=True, text=True, timeout=600)


@pytest.fixture(scope="module")
def source():
    with open(os.path.join(ROOT, "oracle", "m3_oracle.c")) as f:
        return f.read()


def test_unmodified_copy_passes_the_pins(tmp_path, source):
    r = _run_pins(tmp_path, "unmodified", source)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_fails_a_pin(tmp_path, source, name, old, new):
    # a forward mistake is planted in the forward recurrence (the first occurrence, before the
    # backward pass, which restates some of its lines); a backward one in the backward pass
    at = source.find(old)
    assert at >= 0, f"mutation site of {name} not found"
    assert (at > source.find(BWD)) == name.startswith("bwd_"), f"mutation site of {name} in the wrong pass"
    r = _run_pins(tmp_path, name, source[:at] + new + source[at + len(old):])
    assert r.returncode == 1, f"{name}: the pins did not catch it\n" + r.stdout[-2000:]
