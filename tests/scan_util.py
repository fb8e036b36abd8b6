"""Helpers shared by the GPU parity tests: move seeded inputs to the device, run the CUDA path
through the binding, run the oracle on the same values, and measure the error."""

import numpy as np

import oracle
from selective_state_space_13_b200 import workloads as wl

TOL_F32 = 1e-4   # max relative error for fp32 inputs
TOL_BF16 = 2e-2  # max relative error for bf16 inputs with fp32 state


def rel_err(got, ref):
    """max_i |g_i - r_i| / (|r_i| + 1e-2 * rms(r)): relative error with a floor that keeps
    near-zero reference values from dominating."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if ref.size == 0:
        return 0.0
    if not np.all(np.isfinite(got)):
        return float("inf")
    rms = float(np.sqrt(np.mean(ref * ref)))
    return float(np.max(np.abs(got - ref) / (np.abs(ref) + 1e-2 * rms + 1e-30)))


def tol_for(w):
    return TOL_F32 if w.dtype == wl.F32 else TOL_BF16


to_torch = wl.to_torch
to_device = wl.to_device


def out_to_f64(t):
    import torch
    return t.detach().to(torch.float64).cpu().numpy()


def run_gpu(inp, dev_inputs=None, device="cuda:0", segments=0, flags=0, use_z=True, use_D=True,
            use_bias=True, softplus=None, initial_state=None, zoh_exact=False, use_conv_bias=True):
    import torch
    from selective_state_space_13_b200 import scan
    w = inp["workload"]
    t = dev_inputs if dev_inputs is not None else to_device(inp, device)
    h0 = None if initial_state is None else \
        torch.from_numpy(np.ascontiguousarray(initial_state, dtype=np.float32)).to(t["u"].device)
    out, last = scan.selective_scan_fwd(
        t["u"], t["delta"], t["A"], t["B"], t["C"], D=t["D"] if use_D else None,
        z=t["z"] if use_z else None, delta_bias=t["delta_bias"] if use_bias else None,
        softplus=w.softplus if softplus is None else softplus, dirs=w.dirs, H=w.H, W=w.W,
        return_last_state=True, segments=segments, flags=flags, initial_state=h0,
        zoh_exact=zoh_exact, conv_weight=t.get("conv_weight"),
        conv_bias=t.get("conv_bias") if use_conv_bias else None,
        delta_scale=t.get("delta_scale"))
    return out, last


def run_oracle(inp, channels=None, batches=None, use_z=True, use_D=True, use_bias=True,
               softplus=None, initial_state=None, zoh_exact=False, use_conv_bias=True):
    w = inp["workload"]
    f = wl.inputs_f64(inp, channels=channels, batches=batches)
    return oracle.selective_scan(f["u"], f["delta"], f["A"], f["B"], f["C"],
                                 Dskip=f["Dskip"] if use_D else None,
                                 z=f["z"] if use_z else None,
                                 delta_bias=f["delta_bias"] if use_bias else None,
                                 softplus=w.softplus if softplus is None else softplus,
                                 dirs=w.dirs, H=w.H, W=w.W, initial_state=initial_state,
                                 zoh_exact=zoh_exact, conv_weight=f["conv_weight"],
                                 conv_bias=f["conv_bias"] if use_conv_bias else None,
                                 delta_scale=f["delta_scale"])
