"""fp64 CPU oracle for the selective scan (S6) forward pass.

TEST INFRASTRUCTURE ONLY: tests/, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` are the only callers.  The product path (the CUDA library and its binding) never
imports this package, and this package imports nothing from the product.

The arithmetic lives in ``ss_oracle.c`` (plain C, double precision, a loop over batch, channel,
direction, time and state); this module only builds it with gcc, converts the inputs to float64
and calls it.  What each step computes, and the passage of the pages it follows, is written in
the header of ``ss_oracle.c``.

Readings of the pages that the oracle fixes (each is listed with its reason in the design notes):
  * Delta = softplus(delta_raw + bias) with no extra scale factor ("Understanding Mamba from
    zero" sec. 4.1 Algorithm 2; the tau factor of "Mamba-UNet" sec. 3 is not used).
  * Abar = exp(Delta*A) exactly (eq. 4), Bbar*u = Delta*B*u (the first-order form of eq. 4 that
    "Mamba-UNet" sec. 4 writes).  ``zoh_exact=True`` switches Bbar to eq. 4 exactly.
  * A is diagonal: one scalar per (channel, state) ("Understanding Mamba from zero" sec. 5).
  * The gate is silu(z) = z*sigmoid(z) (Step 6, phi = SiLU); the Vim block's sigma(z) is read
    as the same gate.
  * With several directions every direction adds its own Dskip*u (each is a full S6 scan).
  * The state starts at zero unless an initial state is given.
  * Delta may arrive as int8 codes q with one scale per channel: the raw value is q * scale[d]
    ("S4 -> Mamba" sec. 2.3; the pages give no scale convention).
  * A, Dskip and delta_bias may be given per direction ([K, D, N], [K, D], [K, D]): direction k
    then uses its own (VMamba's cross-scan and Vim's two directions are separate S6 modules).
  * With u given per direction ([K, batch, L, D]), direction k scans its own input; Sigma's
    CroMB ("S4 -> Mamba" sec. 4.1) is two such directions in forward order with the C of the
    other modality, summed.
  * With a convolution given, each direction convolves u along its own scan order (causal,
    depthwise, zero before the first step; the last tap takes the current step) and applies
    SiLU; the result replaces u in both the Bbar*u term and the D skip ("Understanding Mamba
    from zero" sec. 6.2 Step 2 and sec. 8; "Vision Mamba" sec. 2.2).
"""

from __future__ import annotations

import ctypes
import os
import subprocess
import sys
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ss_oracle.c")
_LIB = os.path.join(_HERE, "libss_oracle.so")
_lock = threading.Lock()
_lib = None

DIR_FORWARD, DIR_REVERSE, DIR_COLUMN, DIR_COLUMN_REVERSE = 0, 1, 2, 3


def build(force: bool = False) -> str:
    """Compile ss_oracle.c with gcc (-O2, OpenMP, no fast-math) into libss_oracle.so."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        cmd = ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fopenmp", "-fno-fast-math",
               "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            i64, i32, dp = ctypes.c_int64, ctypes.c_int32, ctypes.c_void_p
            lib.ss_oracle_scan.restype = ctypes.c_int
            lib.ss_oracle_scan.argtypes = [i64, i64, i64, i64, i32, dp, i64, i64,
                                           dp, dp, dp, dp, dp, dp, dp, dp,
                                           i32, i32, dp, dp, i32, dp, dp, dp, i64, i32, dp, i32]
            lib.ss_oracle_conv_silu.restype = ctypes.c_int
            lib.ss_oracle_conv_silu.argtypes = [i64, i64, i64, i32, dp, i64, i64, dp, dp, dp,
                                                i64, dp]
            lib.ss_oracle_position.restype = ctypes.c_int64
            lib.ss_oracle_position.argtypes = [i32, i64, i64, i64, i64]
            lib.ss_oracle_max_threads.restype = ctypes.c_int
            lib.ss_oracle_max_threads.argtypes = []
            _lib = lib
    return _lib


def max_threads() -> int:
    return int(_load().ss_oracle_max_threads())


def position(direction: int, L: int, t: int, H: int = 0, W: int = 0) -> int:
    """Spatial position visited at step t of a scan in ``direction`` (-1 if unknown)."""
    return int(_load().ss_oracle_position(direction, L, H, W, t))


def _f64(x):
    return None if x is None else np.ascontiguousarray(x, dtype=np.float64)


def _ptr(x):
    return None if x is None else x.ctypes.data_as(ctypes.c_void_p)


def _check_conv(conv_weight, conv_bias, K, D):
    if conv_weight.ndim != 3 or conv_weight.shape[:2] != (K, D) or conv_weight.shape[2] < 1:
        raise ValueError("conv_weight must be [K, D, width]")
    if conv_bias is not None and conv_bias.shape != (K, D):
        raise ValueError("conv_bias must be [K, D]")


def conv_silu(u, conv_weight, conv_bias=None, dirs=(DIR_FORWARD,), H=0, W=0):
    """The convolved and activated inputs alone: [K, batch, L, D], direction k's scan order."""
    u, conv_weight, conv_bias = _f64(u), _f64(conv_weight), _f64(conv_bias)
    dirs_arr = np.ascontiguousarray(np.asarray(dirs, dtype=np.int32).reshape(-1))
    K = int(dirs_arr.size)
    batch, L, D = u.shape
    _check_conv(conv_weight, conv_bias, K, D)
    out = np.empty((K, batch, L, D), dtype=np.float64)
    rc = _load().ss_oracle_conv_silu(batch, L, D, K, _ptr(dirs_arr), int(H), int(W), _ptr(u),
                                     _ptr(conv_weight), _ptr(conv_bias),
                                     int(conv_weight.shape[2]), _ptr(out))
    if rc != 0:
        raise ValueError("oracle rejected its arguments (code %d)" % rc)
    return out


def selective_scan(u, delta, A, B, C, Dskip=None, z=None, delta_bias=None, softplus=True,
                   dirs=(DIR_FORWARD,), H=0, W=0, zoh_exact=False, threads=None,
                   return_last_state=True, initial_state=None, conv_weight=None,
                   conv_bias=None, delta_scale=None):
    """Run the oracle.

    u, z: [batch, L, D] (u may be [K, batch, L, D]: direction k then reads u[k], as in the
    cross-modal scan); delta: [K, batch, L, D]; B, C: [K, batch, L, N]; A: [D, N], or
    [K, D, N] for parameters per direction (then Dskip and delta_bias are [K, D]);
    Dskip, delta_bias: [D] or None; initial_state: [K, batch, D, N] or None (zero);
    conv_weight: [K, D, width] or None (u is used as it is); conv_bias: [K, D] or None;
    delta_scale: [D] or None -- with it, delta holds int8 codes q and the raw value is
    q * delta_scale[d].
    Inputs may be any real dtype; they are upcast to float64 exactly.  Returns
    (out [batch, L, D], last_state [K, batch, D, N]) in float64.
    """
    u, delta, A, B, C = _f64(u), _f64(delta), _f64(A), _f64(B), _f64(C)
    Dskip, z, delta_bias = _f64(Dskip), _f64(z), _f64(delta_bias)
    initial_state = _f64(initial_state)
    conv_weight, conv_bias = _f64(conv_weight), _f64(conv_bias)
    delta_scale = _f64(delta_scale)
    dirs_arr = np.ascontiguousarray(np.asarray(dirs, dtype=np.int32).reshape(-1))
    K = int(dirs_arr.size)
    u_per_dir = u.ndim == 4
    if u.ndim not in (3, 4) or (u_per_dir and u.shape[0] != K):
        raise ValueError("u must be [batch, L, D] or [K, batch, L, D]")
    batch, L, D = u.shape[-3:]
    params_per_dir = A.ndim == 3
    if A.ndim not in (2, 3) or A.shape[-2] != D or (params_per_dir and A.shape[0] != K):
        raise ValueError("A must be [D, N] or [K, D, N]")
    N = A.shape[-1]
    if delta.shape != (K, batch, L, D):
        raise ValueError("delta must be [K, batch, L, D], got %r" % (delta.shape,))
    if B.shape != (K, batch, L, N) or C.shape != (K, batch, L, N):
        raise ValueError("B and C must be [K, batch, L, N]")
    if z is not None and z.shape != (batch, L, D):
        raise ValueError("z must be [batch, L, D]")
    pshape = (K, D) if params_per_dir else (D,)
    for v in (Dskip, delta_bias):
        if v is not None and v.shape != pshape:
            raise ValueError("Dskip and delta_bias must be %r" % (pshape,))
    if delta_scale is not None and delta_scale.shape != (D,):
        raise ValueError("delta_scale must be [D]")
    if initial_state is not None and initial_state.shape != (K, batch, D, N):
        raise ValueError("initial_state must be [K, batch, D, N]")
    if conv_weight is not None:
        _check_conv(conv_weight, conv_bias, K, D)
    elif conv_bias is not None:
        raise ValueError("conv_bias needs conv_weight")
    out = np.empty((batch, L, D), dtype=np.float64)
    last = np.empty((K, batch, D, N), dtype=np.float64) if return_last_state else None
    if threads is None:
        threads = max_threads()
    rc = _load().ss_oracle_scan(batch, L, D, N, K, _ptr(dirs_arr), int(H), int(W),
                                _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(Dskip),
                                _ptr(z), _ptr(delta_bias), int(bool(softplus)),
                                int(bool(zoh_exact)), _ptr(out), _ptr(last), int(threads),
                                _ptr(initial_state), _ptr(conv_weight), _ptr(conv_bias),
                                0 if conv_weight is None else int(conv_weight.shape[2]),
                                int(u_per_dir), _ptr(delta_scale), int(params_per_dir))
    if rc != 0:
        raise ValueError("oracle rejected its arguments (code %d)" % rc)
    return out, last


if __name__ == "__main__":  # pragma: no cover - manual build helper
    print(build(force="--force" in sys.argv))
