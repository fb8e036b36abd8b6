"""Each plausible mistake planted in a copy of the oracle's C source must fail at least one pin.

The mutant is compiled into a temporary directory on the CPU and swapped in for the real oracle
library for the duration of one check; the real oracle is restored afterwards.
"""

import ctypes
import inspect
import os
import shutil
import subprocess

import pytest

import oracle
import tests.test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "ss_oracle.c")

MUTATIONS = [
    ("dropped D skip", "(Dk ? Dk[d] : 0.0) * ut", "0.0 * ut"),
    ("B read where C belongs", "bcoef * B[row * N + n] * ut", "bcoef * C[row * N + n] * ut"),
    ("C read where B belongs", "yt += C[row * N + n] * h[n]", "yt += B[row * N + n] * h[n]"),
    ("wrong sign in exp(Delta A)", "exp(dt * a)", "exp(-dt * a)"),
    ("dropped delta bias", "+ (biask ? biask[d] : 0.0)", "+ 0.0"),
    ("softplus skipped", "dt = oracle_softplus(dt);", "dt = dt;"),
    ("softplus sign", "log1p(exp(-fabs(x)))", "log1p(exp(fabs(x)))"),
    ("column map transposed", "return (t % H) * W + (t / H);", "return (t / W) * W + (t % W);"),
    ("reverse map off by one", "return L - 1 - t;", "return (L - t) % L;"),
    ("gate sign", "v / (1.0 + exp(-v))", "v / (1.0 + exp(v))"),
    ("readout before update", "h[n] = abar * h[n] + bcoef * B[row * N + n] * ut;\n"
     "                            yt += C[row * N + n] * h[n];",
     "yt += C[row * N + n] * h[n];\n"
     "                            h[n] = abar * h[n] + bcoef * B[row * N + n] * ut;"),
    ("exact ZOH coefficient without 1/A", "expm1(dt * a) / a", "expm1(dt * a)"),
    ("last_state layout transposed", "last_state[(((int64_t)k * batch + b) * D + d) * N + n]",
     "last_state[(((int64_t)k * batch + b) * N + n) * D + d]"),
    ("state not reset between directions", "for (int64_t n = 0; n < N; ++n)\n"
     "                        h[n] = initial_state", "if (k == 0) for (int64_t n = 0; n < N; ++n)\n"
     "                        h[n] = initial_state"),
    ("initial state of the wrong direction", "initial_state[(((int64_t)k * batch + b) * D + d) * N + n]",
     "initial_state[(((int64_t)0 * batch + b) * D + d) * N + n]"),
    ("initial state ignored", "h[n] = initial_state\n", "h[n] = 0 && initial_state\n"),
    ("conv taps in reverse order", "const int64_t s = t - (width - 1) + j;",
     "const int64_t s = t - j;"),
    ("conv along the spatial order", "u[(b * L + ss_oracle_position(dir, L, H, W, s)) * D + d]",
     "u[(b * L + s) * D + d]"),
    ("conv bias dropped", "double c = bias;", "double c = 0.0;"),
    ("no activation after the conv", "return oracle_silu(c);", "return c;"),
    ("D skip reads the unconvolved input", "(Dk ? Dk[d] : 0.0) * ut;",
     "(Dk ? Dk[d] : 0.0) * u[(b * L + p) * D + d];"),
    ("scan takes conv weights of direction 0", "uk, b, d, L, D, dirs[k], H, W, t,\n"
     "                                      conv_weight + ((int64_t)k * D + d) * conv_width,",
     "uk, b, d, L, D, dirs[k], H, W, t,\n"
     "                                      conv_weight + ((int64_t)0 * D + d) * conv_width,"),
    ("int8 scale of the first channel", "delta[row * D + d] * delta_scale[d]",
     "delta[row * D + d] * delta_scale[0]"),
    ("int8 scale applied after the bias", "double dt = draw + (biask ? biask[d] : 0.0);",
     "double dt = (delta_scale ? (delta[row * D + d] + (biask ? biask[d] : 0.0)) * "
     "delta_scale[d] : draw + (biask ? biask[d] : 0.0));"),
    ("parameters of the first direction for all", "const int64_t pk = params_per_direction ? (int64_t)k : 0;",
     "const int64_t pk = 0;"),
    ("every direction reads the first input", "u_per_direction ? u + (int64_t)k * batch",
     "u_per_direction ? u + (int64_t)0 * batch"),
]


def _pin_calls():
    calls = []
    for name, fn in inspect.getmembers(pins, inspect.isfunction):
        if not name.startswith("test_") or name == "test_golden_regression_fixture":
            continue
        marks = getattr(fn, "pytestmark", [])
        params = [m for m in marks if m.name == "parametrize"]
        if not params:
            calls.append((name, fn, {}))
            continue
        m = params[0]
        argnames = [a.strip() for a in m.args[0].split(",")] if isinstance(m.args[0], str) \
            else list(m.args[0])
        for vals in m.args[1]:
            if len(argnames) == 1:
                vals = (vals,)
            calls.append((name, fn, dict(zip(argnames, vals))))
    return calls


@pytest.mark.parametrize("label,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_mutant_fails_a_pin(tmp_path, label, old, new):
    src = open(SRC).read()
    assert src.count(old) >= 1, "mutation anchor not found: %s" % label
    mutant = tmp_path / "mutant.c"
    mutant.write_text(src.replace(old, new))
    so = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fopenmp", "-o", str(so),
                    str(mutant), "-lm"], check=True)
    real = oracle._load()
    lib = ctypes.CDLL(str(so))
    for fname in ("ss_oracle_scan", "ss_oracle_position", "ss_oracle_max_threads",
                  "ss_oracle_conv_silu"):
        getattr(lib, fname).restype = getattr(real, fname).restype
        getattr(lib, fname).argtypes = getattr(real, fname).argtypes
    failed = []
    try:
        oracle._lib = lib
        for name, fn, kw in _pin_calls():
            try:
                if "tmp_path" in inspect.signature(fn).parameters:
                    kw = dict(kw, tmp_path=tmp_path)
                fn(**kw)
            except (AssertionError, ValueError):
                failed.append(name)
    finally:
        oracle._lib = real
        shutil.rmtree(tmp_path, ignore_errors=True)
    assert failed, "no pin caught the planted mistake: %s" % label
