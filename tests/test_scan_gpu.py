"""Parity of the CUDA selective scan with the fp64 oracle (needs a B200).

Small cases are compared element by element: they span several channel tiles and time tiles,
ragged channel and time tails, every state count up to 16, one to four directions, split
sequences, the generic-A path, softplus off with Delta = 0 steps, and missing optional inputs.
The five full-size workloads run in the launch configuration the benchmark times and are
compared on sampled channels (every step of every sampled channel, which the oracle computes
independently per channel).  Bars: max relative error (floor 1e-2 * rms) <= 1e-4 for fp32
inputs, <= 2e-2 for bf16 inputs with fp32 state.
"""

import numpy as np
import pytest

import oracle

from selective_state_space_13_b200 import workloads as wl
from tests.scan_util import (TOL_BF16, TOL_F32, out_to_f64, rel_err, run_gpu, run_oracle,
                             to_device, tol_for)

pytestmark = pytest.mark.gpu


def _check(inp, device, tol=None, **kw):
    w = inp["workload"]
    opts = {k: kw.pop(k) for k in ("segments", "flags") if k in kw}
    out, last = run_gpu(inp, device=device, **opts, **kw)
    ref_out, ref_last = run_oracle(inp, **kw)
    tol = tol_for(w) if tol is None else tol
    e_out = rel_err(out_to_f64(out), ref_out)
    e_last = rel_err(out_to_f64(last), ref_last)
    assert e_out <= tol and e_last <= tol, (w.name, e_out, e_last)
    return e_out, e_last


def test_tiny_workload(cuda_device):
    _check(wl.make_inputs("tiny"), cuda_device)


# ----------------------------------------------------------------------------- zero and tiny steps
# The bf16 kernel keeps the normalised state k = h / w with w = Delta*u and normalises a step
# whose |w| is below 2^-64 by 2^-64 instead (which adds at most 2^-64*|B| to h).  These cases
# put such steps -- u = 0 padding, Delta = 0, u so small that Delta*u underflows 2^-64 -- into
# bf16 scans of one, two and four directions, with and without split sequences, and compare
# every element with the oracle.

ZERO_DIRS = {"fwd": ((wl.DIR_FORWARD,), 0, 0),
             "fwd_rev": ((wl.DIR_FORWARD, wl.DIR_REVERSE), 0, 0),
             "cross4": ((wl.DIR_FORWARD, wl.DIR_COLUMN, wl.DIR_REVERSE, wl.DIR_COLUMN_REVERSE), 30, 30)}


def _zero_step_case(dirs_key, seed):
    dirs, H, W = ZERO_DIRS[dirs_key]
    L = H * W if H else 900
    w = wl.Workload("zs_" + dirs_key, 4, L, 80, 16, wl.BF16, dirs=dirs, H=H, W=W, seed=seed)
    inp = wl.make_inputs(w)
    u = inp["u"]  # bf16 bit patterns [b, L, D]
    u[0, :17] = 0                 # a padding run at the start
    u[0, 400:401] = 0             # and a single padded step
    u[1, 250:550] = 0             # 300 steps, across the segment boundaries of 3 segments
    u[2, ::37] = 0                # scattered single steps
    u[3] = 0                      # a whole row of padding
    tiny = wl.f32_to_bf16_bits(np.full((20, w.dim), 1e-25, dtype=np.float32))
    u[1, 600:620] = tiny          # Delta*u below 2^-64
    u[2, 5:8, ::3] = tiny[:3, ::3]
    return w, inp


@pytest.mark.parametrize("segments", [1, 3])
@pytest.mark.parametrize("dirs_key", sorted(ZERO_DIRS))
def test_bf16_zero_and_tiny_input_steps(cuda_device, dirs_key, segments):
    w, inp = _zero_step_case(dirs_key, 300 + segments)
    _check(inp, cuda_device, segments=segments)


@pytest.mark.parametrize("segments", [1, 3])
@pytest.mark.parametrize("dirs_key", sorted(ZERO_DIRS))
def test_bf16_zero_delta_steps(cuda_device, dirs_key, segments):
    # softplus off, Delta = delta_raw + bias: bias values exact in bf16 and delta_raw = -bias at
    # chosen steps give Delta = 0 there (h unchanged); elsewhere Delta is positive
    dirs, H, W = ZERO_DIRS[dirs_key]
    L = H * W if H else 900
    w = wl.Workload("zd_" + dirs_key, 3, L, 64, 16, wl.BF16, dirs=dirs, H=H, W=W, seed=310,
                    softplus=False)
    inp = wl.make_inputs(w)
    rng = np.random.default_rng(311)
    bias = (rng.integers(1, 9, size=w.dim) / 16.0).astype(np.float32)   # exact in bf16
    inp["delta_bias"] = bias
    raw = rng.uniform(-bias[None, None, None, :] + 0.01, 0.3, size=inp["delta"].shape)
    zero = [0, 1, 2, 17, 300, 301, 302, 303, 304, 305, L - 1]
    raw[:, :, zero, :] = -bias[None, None, :]
    raw[:, 1, 100:400, :] = -bias[None, :]                               # a long run
    inp["delta"] = wl.f32_to_bf16_bits(raw.astype(np.float32))
    _check(inp, cuda_device, segments=segments)


@pytest.mark.parametrize("segments", [0, 1, 3])
@pytest.mark.parametrize("dtype", [wl.BF16, wl.F32])
def test_single_direction_ragged(cuda_device, dtype, segments):
    w = wl.variant("m130", name="small", batch=2, seqlen=300, dim=136, dtype=dtype, seed=71)
    _check(wl.make_inputs(w), cuda_device, segments=segments)


@pytest.mark.parametrize("N", [1, 3, 4, 5, 8, 11, 16])
def test_state_sizes(cuda_device, N):
    w = wl.variant("m130", name="nstate", batch=2, seqlen=97, dim=72, dstate=N, seed=100 + N)
    _check(wl.make_inputs(w), cuda_device)


@pytest.mark.parametrize("flags", [0, 1])
def test_generic_A(cuda_device, flags):
    w = wl.variant("m130", name="genA", batch=2, seqlen=130, dim=64, dtype=wl.F32, seed=81)
    inp = wl.make_inputs(w)
    if flags == 0:
        rng = np.random.default_rng(5)
        inp["A"] = (-rng.uniform(0.05, 3.0, size=inp["A"].shape)).astype(np.float32)
    _check(inp, cuda_device, flags=flags)


def test_mixed_chain_and_generic_channels(cuda_device):
    # some channels satisfy A[d,n] = (n+1) A[d,0], others do not, inside one warp
    w = wl.variant("m130", name="mixA", batch=1, seqlen=77, dim=64, dtype=wl.F32, seed=82)
    inp = wl.make_inputs(w)
    inp["A"][::3] *= np.float32(0.37)  # still a chain
    inp["A"][1::5, 2] = np.float32(-0.123)  # breaks the chain for these channels
    _check(inp, cuda_device)


@pytest.mark.parametrize("L", [1, 2, 31, 32, 33, 65])
def test_short_sequences(cuda_device, L):
    w = wl.variant("m130", name="short", batch=3, seqlen=L, dim=40, seed=90 + L)
    _check(wl.make_inputs(w), cuda_device)


def test_vim_like_bidirectional(cuda_device):
    w = wl.variant("vim", name="vim_small", batch=3, dim=64, seed=91)
    _check(wl.make_inputs(w), cuda_device)


@pytest.mark.parametrize("segments", [0, 2])
def test_ss2d_like_cross_scan(cuda_device, segments):
    w = wl.variant("ss2d", name="ss2d_small", batch=2, seqlen=120, H=12, W=10, dim=32, seed=92)
    _check(wl.make_inputs(w), cuda_device, segments=segments)


def test_directions_fp32_gate(cuda_device):
    w = wl.Workload("dirs32", 2, 48, 16, 4, wl.F32, dirs=(wl.DIR_COLUMN_REVERSE, wl.DIR_REVERSE,
                                                          wl.DIR_COLUMN), H=6, W=8, seed=93,
                    dskip="normal")
    _check(wl.make_inputs(w), cuda_device)


def test_optional_inputs_absent(cuda_device):
    w = wl.variant("m130", name="opt", batch=2, seqlen=70, dim=48, seed=94)
    inp = wl.make_inputs(w)
    _check(inp, cuda_device, use_z=False, use_D=False, use_bias=False)


def test_softplus_off_zero_delta_steps(cuda_device):
    w = wl.variant("m130", name="dz", batch=2, seqlen=90, dim=32, dtype=wl.F32, seed=95)
    inp = wl.make_inputs(w)
    rng = np.random.default_rng(6)
    # Delta = delta + bias; positive steps, with some steps exactly zero
    inp["delta"] = rng.uniform(0.01, 0.4, size=inp["delta"].shape).astype(np.float32)
    inp["delta"] -= inp["delta_bias"][None, None, None, :]
    zero = [0, 1, 17, 40, 41, 42, 89]
    inp["delta"][:, :, zero, :] = -inp["delta_bias"][None, None, :]
    _check(inp, cuda_device, softplus=False)


def test_empty_problems(cuda_device):
    import torch
    from selective_state_space_13_b200 import scan
    for batch, L in ((0, 16), (2, 0)):
        u = torch.empty((batch, L, 16), device=cuda_device)
        d = torch.empty((1, batch, L, 16), device=cuda_device)
        bc = torch.empty((1, batch, L, 4), device=cuda_device)
        A = -torch.ones((16, 4), device=cuda_device)
        out, last = scan.selective_scan_fwd(u, d, A, bc, bc, return_last_state=True)
        torch.cuda.synchronize()
        assert out.shape == u.shape
        if L == 0 and batch:
            assert torch.all(last == 0)


def test_repeat_calls_identical(cuda_device):
    # the scan is deterministic: two calls give bit-identical results
    w = wl.variant("m130", name="rep", batch=2, seqlen=200, dim=64, seed=96)
    inp = wl.make_inputs(w)
    t = to_device(inp, cuda_device)
    o1, l1 = run_gpu(inp, dev_inputs=t, segments=2)
    o2, l2 = run_gpu(inp, dev_inputs=t, segments=2)
    assert bool((o1 == o2).all()) and bool((l1 == l2).all())


@pytest.mark.parametrize("segments", [1, 0, 5])
@pytest.mark.parametrize("L", [2048, 4096])
def test_fp32_long_memory_from_random_state(cuda_device, L, segments):
    # fp32 inputs for thousands of steps with the long-sequence recipe's Delta (log-uniform bias
    # down to 1e-3: memories of ~1000 steps) from an N(0, 1) initial state, scanned whole, with
    # the library's segment choice, and in five segments.  The fp64 state keeps the fp32 bar at
    # these lengths; an fp32 state loses one rounding of |h| per step and does not.
    w = wl.variant("long", name="f32long%d" % L, seqlen=L, dim=64, dtype=wl.F32, seed=98 + L)
    inp = wl.make_inputs(w)
    h0 = np.random.default_rng(L).standard_normal((1, 1, w.dim, w.dstate)).astype(np.float32)
    _check(inp, cuda_device, segments=segments, initial_state=h0)


@pytest.mark.parametrize("segments", [1, 3])
@pytest.mark.parametrize("dtype", [wl.BF16, wl.F32])
def test_initial_state(cuda_device, dtype, segments):
    w = wl.variant("vim", name="h0", batch=2, seqlen=250, dim=64, dtype=dtype, seed=97)
    inp = wl.make_inputs(w)
    h0 = np.random.default_rng(8).standard_normal((w.K, w.batch, w.dim, w.dstate)).astype(np.float32)
    _check(inp, cuda_device, segments=segments, initial_state=h0)


@pytest.mark.parametrize("case", ["bf16", "f32", "bf16_split", "f32_genericA"])
def test_exact_zoh(cuda_device, case):
    dtype = wl.F32 if case.startswith("f32") else wl.BF16
    w = wl.variant("m130", name="zoh", batch=2, seqlen=180, dim=72, dtype=dtype, seed=98)
    inp = wl.make_inputs(w)
    if case == "f32_genericA":
        rng = np.random.default_rng(9)
        inp["A"] = (-rng.uniform(0.05, 3.0, size=inp["A"].shape)).astype(np.float32)
        inp["A"][3, 5] = 0.0  # A = 0: Bbar falls back to Delta*B
    segments = 3 if case == "bf16_split" else 1
    _check(inp, cuda_device, segments=segments, zoh_exact=True)


def test_initial_state_with_empty_sequence(cuda_device):
    import torch
    from selective_state_space_13_b200 import scan
    h0 = torch.randn((1, 2, 16, 4), device=cuda_device)
    u = torch.empty((2, 0, 16), device=cuda_device)
    e = torch.empty((1, 2, 0, 16), device=cuda_device)
    bc = torch.empty((1, 2, 0, 4), device=cuda_device)
    out, last = scan.selective_scan_fwd(u, e, -torch.ones((16, 4), device=cuda_device), bc, bc,
                                        return_last_state=True, initial_state=h0)
    torch.cuda.synchronize()
    assert torch.equal(last, h0)


def test_bounded_wait_gives_up_and_reports(cuda_device):
    # a wait on a barrier that nothing completes must run out, leave the outputs alone, report
    # SS_ERR_DEVICE_TIMEOUT, and leave the context usable
    import torch
    from selective_state_space_13_b200 import scan
    w = wl.variant("m130", name="tmo", batch=1, seqlen=64, dim=64, seed=99)
    inp = wl.make_inputs(w)
    t = to_device(inp, cuda_device)
    assert scan.selective_scan_device_status(clear=True) == scan.SS_OK
    sentinel = torch.full_like(t["u"], 7.0)
    out = scan.selective_scan_fwd(t["u"], t["delta"], t["A"], t["B"], t["C"], D=t["D"], z=t["z"],
                                  delta_bias=t["delta_bias"], out=sentinel,
                                  flags=scan.SS_FLAG_TEST_WAIT_TIMEOUT)
    assert scan.selective_scan_device_status(clear=False) == scan.SS_ERR_DEVICE_TIMEOUT
    assert torch.all(out == 7.0)
    assert scan.selective_scan_device_status(clear=True) == scan.SS_ERR_DEVICE_TIMEOUT
    assert scan.selective_scan_device_status(clear=True) == scan.SS_OK
    _check(inp, cuda_device)
    assert scan.selective_scan_device_status(clear=True) == scan.SS_OK


def test_device_status_clean(cuda_device):
    from selective_state_space_13_b200 import scan
    assert scan.selective_scan_device_status(clear=True) == scan.SS_OK


# ----------------------------------------------------------------------------- fused conv

@pytest.mark.parametrize("segments", [0, 1, 3])
@pytest.mark.parametrize("dtype", [wl.BF16, wl.F32])
def test_conv_single_direction(cuda_device, dtype, segments):
    w = wl.variant("m130", name="conv1", batch=2, seqlen=300, dim=136, dtype=dtype, conv=4,
                   seed=120)
    _check(wl.make_inputs(w), cuda_device, segments=segments)


@pytest.mark.parametrize("width", [1, 2, 3])
def test_conv_narrow_widths(cuda_device, width):
    w = wl.variant("m130", name="convw", batch=2, seqlen=77, dim=64, conv=width, seed=121 + width)
    _check(wl.make_inputs(w), cuda_device, segments=2)


@pytest.mark.parametrize("segments", [0, 2])
def test_conv_vim_per_direction(cuda_device, segments):
    w = wl.variant("vim", name="conv_vim", batch=3, dim=64, conv=4, seed=125)
    _check(wl.make_inputs(w), cuda_device, segments=segments)


@pytest.mark.parametrize("H,W", [(12, 10), (16, 8)])
def test_conv_cross_scan_orders(cuda_device, H, W):
    # H % 8 != 0 reads rows one by one, H % 8 == 0 through the 8-row column boxes
    w = wl.variant("ss2d", name="conv_ss2d", batch=2, seqlen=H * W, H=H, W=W, dim=32, conv=4,
                   seed=126 + H)
    _check(wl.make_inputs(w), cuda_device, segments=2)


def test_conv_without_bias_and_with_generic_A(cuda_device):
    w = wl.variant("m130", name="conv_nb", batch=2, seqlen=150, dim=64, conv=4, seed=128)
    inp = wl.make_inputs(w)
    rng = np.random.default_rng(10)
    inp["A"] = (-rng.uniform(0.05, 3.0, size=inp["A"].shape)).astype(np.float32)
    _check(inp, cuda_device, segments=3, use_conv_bias=False)


def test_conv_with_initial_state_and_exact_zoh(cuda_device):
    w = wl.variant("vim", name="conv_h0", batch=2, seqlen=130, dim=64, conv=4, seed=129)
    inp = wl.make_inputs(w)
    h0 = np.random.default_rng(11).standard_normal((w.K, w.batch, w.dim, w.dstate)).astype(np.float32)
    _check(inp, cuda_device, segments=2, initial_state=h0, zoh_exact=True)


# ----------------------------------------------------------------------------- input per direction

@pytest.mark.parametrize("segments", [0, 3])
@pytest.mark.parametrize("dtype", [wl.BF16, wl.F32])
def test_cromb_cross_modal(cuda_device, dtype, segments):
    w = wl.variant("cromb", name="cromb_small", batch=2, seqlen=333, dim=72, dtype=dtype, seed=140)
    _check(wl.make_inputs(w), cuda_device, segments=segments)


def test_input_per_direction_all_orders_with_conv_and_gate(cuda_device):
    w = wl.Workload("upd", 2, 16 * 6, 64, 16, wl.BF16, dirs=(wl.DIR_FORWARD, wl.DIR_COLUMN,
                                                           wl.DIR_REVERSE, wl.DIR_COLUMN_REVERSE),
                    H=16, W=6, u_per_dir=True, conv=4, seed=141)
    _check(wl.make_inputs(w), cuda_device, segments=2)


def test_input_per_direction_row_by_row_columns(cuda_device):
    # H % 8 != 0: column orders copy u row by row, from direction k's own input
    w = wl.Workload("upd2", 2, 10 * 7, 32, 8, wl.F32, dirs=(wl.DIR_COLUMN_REVERSE, wl.DIR_FORWARD),
                    H=10, W=7, u_per_dir=True, seed=142)
    _check(wl.make_inputs(w), cuda_device)


# ----------------------------------------------------------------------------- int8 Delta

@pytest.mark.parametrize("segments", [0, 1, 3])
def test_int8_delta_single_direction(cuda_device, segments):
    w = wl.variant("m130", name="i8", batch=2, seqlen=300, dim=144, delta_int8=True, seed=150)
    _check(wl.make_inputs(w), cuda_device, segments=segments)


@pytest.mark.parametrize("N", [4, 8, 16])
def test_int8_delta_state_sizes_with_conv(cuda_device, N):
    w = wl.variant("m130", name="i8c", batch=2, seqlen=97, dim=64, dstate=N, delta_int8=True,
                   conv=4, seed=151 + N)
    _check(wl.make_inputs(w), cuda_device, segments=2)


def test_int8_delta_directions_and_exact_zoh(cuda_device):
    w = wl.variant("ss2d", name="i8_ss2d", batch=2, seqlen=16 * 6, H=16, W=6, dim=48,
                   delta_int8=True, seed=156)
    _check(wl.make_inputs(w), cuda_device)
    w = wl.variant("vim", name="i8_vim", batch=3, dim=64, delta_int8=True, seed=157)
    _check(wl.make_inputs(w), cuda_device, segments=2, zoh_exact=True)


# ----------------------------------------------------------------------------- parameters per direction

@pytest.mark.parametrize("dtype", [wl.BF16, wl.F32])
def test_parameters_per_direction_vim(cuda_device, dtype):
    w = wl.variant("vim", name="ppd_vim", batch=3, dim=64, dtype=dtype, params_per_dir=True,
                   seed=160)
    _check(wl.make_inputs(w), cuda_device, segments=2)


def test_parameters_per_direction_cross_scan_generic_A_conv(cuda_device):
    w = wl.variant("ss2d", name="ppd_ss2d", batch=2, seqlen=16 * 5, H=16, W=5, dim=32,
                   params_per_dir=True, conv=4, dskip="normal", seed=161)
    inp = wl.make_inputs(w)
    _check(inp, cuda_device)
    rng = np.random.default_rng(12)
    inp["A"] = (-rng.uniform(0.05, 3.0, size=inp["A"].shape)).astype(np.float32)
    _check(inp, cuda_device, segments=3)


# ----------------------------------------------------------------------------- host buffers

def _host_case(inp, device, chunks=4, initial_state=None):
    """selective_scan_fwd_host on pinned host copies of the inputs, checked against the oracle."""
    import torch
    from selective_state_space_13_b200 import scan
    w = inp["workload"]
    t = to_device(inp, device)
    host = {k: (None if v is None else v.cpu().pin_memory()) for k, v in t.items()}
    h0 = None if initial_state is None else \
        torch.from_numpy(np.ascontiguousarray(initial_state, dtype=np.float32)).to(device)
    out, last = scan.selective_scan_fwd_host(
        host["u"], host["delta"], t["A"], host["B"], host["C"], D=t["D"], z=host["z"],
        delta_bias=t["delta_bias"], softplus=w.softplus, dirs=w.dirs, H=w.H, W=w.W,
        return_last_state=True, initial_state=h0, conv_weight=t["conv_weight"],
        conv_bias=t["conv_bias"], delta_scale=t["delta_scale"], chunks=chunks)
    torch.cuda.synchronize()
    assert out.device.type == "cpu" and last.device.type == "cpu"
    ref_out, ref_last = run_oracle(inp, initial_state=initial_state)
    tol = tol_for(w)
    e_out, e_last = rel_err(out_to_f64(out), ref_out), rel_err(out_to_f64(last), ref_last)
    assert e_out <= tol and e_last <= tol, (w.name, e_out, e_last)


@pytest.mark.parametrize("chunks", [1, 3, 8])
def test_host_buffers_batch_pieces(cuda_device, chunks):
    w = wl.variant("m130", name="host_b", batch=5, seqlen=200, dim=72, seed=170)
    _host_case(wl.make_inputs(w), cuda_device, chunks=chunks)


def test_host_buffers_sequence_pieces(cuda_device):
    # one batch row of one forward direction: pieces along the sequence, chained by the state
    w = wl.variant("long", name="host_l", seqlen=1000, dim=64, seed=171)
    h0 = np.random.default_rng(13).standard_normal((1, 1, 64, 16)).astype(np.float32)
    _host_case(wl.make_inputs(w), cuda_device, chunks=5, initial_state=h0)


def test_host_buffers_sequence_pieces_fp32(cuda_device):
    # pieces of whole tiles continued through the stored final state: against the oracle within
    # the fp32 bar, and against one unsplit scan within one fp32 rounding of the carried state
    # per piece boundary (the scan's own state is fp64)
    import torch
    from selective_state_space_13_b200 import scan
    w = wl.variant("long", name="host_l32", seqlen=1000, dim=64, dtype=wl.F32, seed=171)
    inp = wl.make_inputs(w)
    t = to_device(inp, cuda_device)
    h0 = torch.from_numpy(np.random.default_rng(13).standard_normal((1, 1, 64, 16))
                          .astype(np.float32)).to(cuda_device)
    ref, ref_last = scan.selective_scan_fwd(t["u"], t["delta"], t["A"], t["B"], t["C"], D=t["D"],
                                            z=t["z"], delta_bias=t["delta_bias"],
                                            return_last_state=True, segments=1, initial_state=h0)
    host = {k: (None if v is None else v.cpu().pin_memory()) for k, v in t.items()}
    out, last = scan.selective_scan_fwd_host(host["u"], host["delta"], t["A"], host["B"], host["C"],
                                             D=t["D"], z=host["z"], delta_bias=t["delta_bias"],
                                             return_last_state=True, initial_state=h0, chunks=5)
    torch.cuda.synchronize()
    _pieces_close(inp, h0, out, last, ref, ref_last)


def test_host_buffers_rows_and_sequence_pieces(cuda_device):
    # more pieces than batch rows, one forward direction: every row is cut along the sequence,
    # each piece continuing from the previous piece of its row
    w = wl.variant("m130", name="host_rs", batch=3, seqlen=700, dim=48, seed=174)
    h0 = np.random.default_rng(14).standard_normal((1, 3, 48, 16)).astype(np.float32)
    _host_case(wl.make_inputs(w), cuda_device, chunks=7, initial_state=h0)
    _host_case(wl.make_inputs(w), cuda_device, chunks=4)


def _pieces_close(inp, h0, out, last, ref, ref_last):
    ref_out, ref_l = run_oracle(inp, initial_state=h0.cpu().numpy())
    assert rel_err(out_to_f64(out), ref_out) <= TOL_F32
    assert rel_err(out_to_f64(last), ref_l) <= TOL_F32
    assert rel_err(out_to_f64(out), out_to_f64(ref)) <= 1e-5
    assert rel_err(out_to_f64(last), out_to_f64(ref_last)) <= 1e-5


def test_host_buffers_rows_and_sequence_pieces_fp32(cuda_device):
    # pieces of whole tiles per row, chained through the stored final state (see the test
    # above)
    import torch
    from selective_state_space_13_b200 import scan
    w = wl.variant("m130", name="host_rs32", batch=2, seqlen=1000, dim=64, dtype=wl.F32,
                   seed=175)
    inp = wl.make_inputs(w)
    t = to_device(inp, cuda_device)
    h0 = torch.from_numpy(np.random.default_rng(15).standard_normal((1, 2, 64, 16))
                          .astype(np.float32)).to(cuda_device)
    ref, ref_last = scan.selective_scan_fwd(t["u"], t["delta"], t["A"], t["B"], t["C"], D=t["D"],
                                            z=t["z"], delta_bias=t["delta_bias"],
                                            return_last_state=True, segments=1, initial_state=h0)
    host = {k: (None if v is None else v.cpu().pin_memory()) for k, v in t.items()}
    out, last = scan.selective_scan_fwd_host(host["u"], host["delta"], t["A"], host["B"], host["C"],
                                             D=t["D"], z=host["z"], delta_bias=t["delta_bias"],
                                             return_last_state=True, initial_state=h0, chunks=6)
    torch.cuda.synchronize()
    _pieces_close(inp, h0, out, last, ref, ref_last)


def test_host_buffers_back_to_back_calls(cuda_device):
    # consecutive calls without a synchronisation in between, each with its own inputs and
    # outputs: the copies of a call may start while the previous call's last scans still run,
    # and every call must still see only its own inputs
    import torch
    from selective_state_space_13_b200 import scan
    w = wl.variant("m130", name="host_bb", batch=4, seqlen=300, dim=64, seed=176)
    cases = []
    for j in range(4):
        inp = wl.make_inputs(wl.variant("m130", name="host_bb%d" % j, batch=4, seqlen=300, dim=64,
                                        seed=176 + j))
        t = to_device(inp, cuda_device)
        ref = scan.selective_scan_fwd(t["u"], t["delta"], t["A"], t["B"], t["C"], D=t["D"],
                                      z=t["z"], delta_bias=t["delta_bias"])
        host = {k: (None if v is None else v.cpu().pin_memory()) for k, v in t.items()}
        cases.append((t, host, ref))
    torch.cuda.synchronize()
    outs = []
    for rep in range(2):
        for t, host, _ in cases:
            o = torch.empty((w.batch, w.seqlen, w.dim), dtype=torch.bfloat16, pin_memory=True)
            scan.selective_scan_fwd_host(host["u"], host["delta"], t["A"], host["B"], host["C"],
                                         D=t["D"], z=host["z"], delta_bias=t["delta_bias"],
                                         out=o, chunks=4)
            outs.append(o)
    torch.cuda.synchronize()
    for i, o in enumerate(outs):
        assert torch.equal(o, cases[i % len(cases)][2].cpu()), i


def test_host_buffers_directions_inputs_and_conv(cuda_device):
    w = wl.variant("cromb", name="host_c", batch=3, seqlen=150, dim=32, conv=4, seed=172)
    _host_case(wl.make_inputs(w), cuda_device, chunks=2)
    w = wl.variant("vim", name="host_v", batch=4, dim=64, delta_int8=True, seed=173)
    _host_case(wl.make_inputs(w), cuda_device, chunks=3)


# ----------------------------------------------------------------------------- full size

FULL_SAMPLES = {
    # workload: (batch rows sampled, channels sampled)
    "tiny": (None, None),
    "m130": (None, 24),
    "long": (None, 64),
    "vim": (8, 32),
    "ss2d": (4, 16),
    "m130_conv": (None, 24),
    "cromb": (4, 16),
    "m130_int8": (None, 24),
}

FULL_VARIANTS = {"m130_conv": dict(conv=4), "m130_int8": dict(delta_int8=True)}


@pytest.mark.parametrize("name", ["tiny", "m130", "long", "vim", "ss2d", "m130_conv", "cromb",
                                  "m130_int8"])
def test_full_size_workloads_sampled(cuda_device, name):
    import torch
    w = wl.variant("m130", **FULL_VARIANTS[name]) if name in FULL_VARIANTS else wl.WORKLOADS[name]
    inp = wl.make_inputs(w)
    t = to_device(inp, cuda_device)
    out, last = run_gpu(inp, dev_inputs=t)            # default launch = the benchmark's
    torch.cuda.synchronize()
    nb, nc = FULL_SAMPLES[name]
    rng = np.random.default_rng(7)
    bsel = None if nb is None else np.sort(rng.choice(w.batch, size=nb, replace=False))
    csel = None if nc is None else np.sort(rng.choice(w.dim, size=nc, replace=False))
    ref_out, ref_last = run_oracle(inp, channels=csel, batches=bsel)
    bi = torch.arange(w.batch) if bsel is None else torch.from_numpy(bsel)
    ci = torch.arange(w.dim) if csel is None else torch.from_numpy(csel)
    got = out.index_select(0, bi.to(out.device)).index_select(2, ci.to(out.device))
    got_last = last.index_select(1, bi.to(out.device)).index_select(2, ci.to(out.device))
    e_out = rel_err(out_to_f64(got), ref_out)
    e_last = rel_err(out_to_f64(got_last), ref_last)
    tol = TOL_F32 if w.dtype == wl.F32 else TOL_BF16
    del t, out, last, got, got_last
    torch.cuda.empty_cache()
    assert e_out <= tol and e_last <= tol, (name, e_out, e_last)


# ----------------------------------------------------------------------------- largest offsets

def test_largest_row_offsets(cuda_device):
    # L * D just under the 2^31 the ABI allows (1 x 1048576 x 2040 bf16, 4.3 GB per tensor): the
    # kernels' 32-bit row offsets and tensor-map coordinates at their limit.  The inputs are
    # drawn on the device from a seeded generator (the host generator would take minutes); the
    # oracle receives the exact stored values of a few channels.
    import torch
    from selective_state_space_13_b200 import scan
    L, D, N = 1 << 20, 2040, 16
    assert L * D < 2 ** 31 and L * D > 2 ** 31 - 2 ** 24
    g = torch.Generator(device=cuda_device).manual_seed(2031)

    def normal(*shape):
        return torch.randn(shape, generator=g, device=cuda_device).to(torch.bfloat16)

    u, z, delta = normal(1, L, D), normal(1, L, D), normal(1, 1, L, D)
    B, C = normal(1, 1, L, N), normal(1, 1, L, N)
    A = -torch.arange(1, N + 1, device=cuda_device, dtype=torch.float32).repeat(D, 1)
    Dskip = torch.ones(D, device=cuda_device)
    d0 = torch.exp(torch.empty(D, device=cuda_device).uniform_(np.log(1e-3), np.log(0.1),
                                                                generator=g))
    bias = d0 + torch.log(-torch.expm1(-d0))
    out, last = scan.selective_scan_fwd(u, delta, A, B, C, D=Dskip, z=z, delta_bias=bias,
                                        return_last_state=True)
    torch.cuda.synchronize()
    assert scan.selective_scan_device_status() == scan.SS_OK
    ch = torch.tensor([0, 1, 1023, 2038, 2039], device=cuda_device)  # both ends of the rows
    f64 = lambda x: x.double().cpu().numpy()  # noqa: E731
    ref_out, ref_last = oracle.selective_scan(
        f64(u.index_select(2, ch)), f64(delta.index_select(3, ch)), f64(A.index_select(0, ch)),
        f64(B), f64(C), Dskip=f64(Dskip.index_select(0, ch)), z=f64(z.index_select(2, ch)),
        delta_bias=f64(bias.index_select(0, ch)))
    e_out = rel_err(f64(out.index_select(2, ch)), ref_out)
    e_last = rel_err(f64(last.index_select(2, ch)), ref_last)
    del u, z, delta, out
    torch.cuda.empty_cache()
    assert e_out <= TOL_BF16 and e_last <= TOL_BF16, (e_out, e_last)


# ----------------------------------------------------------------------------- guard bands

GUARD_CASES = {
    "one_dir_segments": (wl.variant("m130", name="g1", batch=3, seqlen=333, dim=136, seed=180),
                         dict(segments=5)),
    "two_dirs": (wl.variant("vim", name="g2", batch=3, seqlen=77, dim=72, seed=181), {}),
    "cross_scan_rows": (wl.variant("ss2d", name="g3", batch=2, seqlen=10 * 7, H=10, W=7, dim=40,
                                   seed=182), dict(segments=2)),
    "conv_int8_per_dir_u": (wl.variant("cromb", name="g4", batch=2, seqlen=150, dim=48, conv=3,
                                       delta_int8=True, seed=183), dict(segments=3)),
    "fp32_zoh": (wl.variant("m130", name="g5", batch=2, seqlen=45, dim=20, dtype=wl.F32,
                            seed=184), dict(zoh_exact=True)),
}


@pytest.mark.parametrize("case", sorted(GUARD_CASES))
def test_outputs_written_once_inside_their_bounds(cuda_device, case):
    # out, last_state and the workspace sit inside larger buffers whose margins hold a canary;
    # out and last_state start as NaN.  After the call every output element must have been
    # written (no NaN left) and no margin byte changed.
    import torch
    from selective_state_space_13_b200 import scan
    w, kw = GUARD_CASES[case]
    inp = wl.make_inputs(w)
    t = to_device(inp, cuda_device)
    io = t["u"].dtype
    pad = 64  # elements; keeps every base 16-byte aligned

    def guarded(shape, dtype, canary):
        n = int(np.prod(shape))
        buf = torch.full((pad + n + pad,), canary, dtype=dtype, device=cuda_device)
        view = buf[pad:pad + n].view(shape)
        view.fill_(float("nan"))
        return buf, view

    ob, out = guarded((w.batch, w.seqlen, w.dim), io, -8192.0)
    lb, last = guarded((w.K, w.batch, w.dim, w.dstate), torch.float32, -8192.0)
    shape = scan.make_shape(w.batch, w.seqlen, w.dim, w.dstate,
                            scan.SS_BF16 if w.dtype == wl.BF16 else scan.SS_F32)
    # (the options that change the workspace are the direction map and the segments)
    nws = scan.selective_scan_workspace_size(shape, scan.make_dirmap(w.dirs, w.H, w.W),
                                             scan.make_opts(kw.get("segments", 0)))
    wpad = 256
    wb = torch.full((wpad + nws + wpad,), 0xA5, dtype=torch.uint8, device=cuda_device)
    ws = wb[wpad:wpad + nws] if nws else None
    scan.selective_scan_fwd(t["u"], t["delta"], t["A"], t["B"], t["C"], D=t["D"], z=t["z"],
                            delta_bias=t["delta_bias"], softplus=w.softplus, dirs=w.dirs, H=w.H,
                            W=w.W, out=out, last_state=last, workspace=ws,
                            conv_weight=t["conv_weight"], conv_bias=t["conv_bias"],
                            delta_scale=t["delta_scale"], **kw)
    torch.cuda.synchronize()
    assert scan.selective_scan_device_status() == scan.SS_OK
    assert not torch.isnan(out.float()).any() and not torch.isnan(last).any()
    for buf in (ob, lb):
        assert bool((buf[:pad] == -8192.0).all()) and bool((buf[-pad:] == -8192.0).all())
    assert bool((wb[:wpad] == 0xA5).all()) and bool((wb[-wpad:] == 0xA5).all())
    # and the results are the scan's
    ref_out, ref_last = run_oracle(inp, zoh_exact=kw.get("zoh_exact", False))
    tol = tol_for(w)
    assert rel_err(out_to_f64(out), ref_out) <= tol and rel_err(out_to_f64(last), ref_last) <= tol


# ----------------------------------------------------------------------------- decoding step by step

@pytest.mark.parametrize("dtype", [wl.BF16, wl.F32])
def test_step_by_step_decoding_matches_one_scan(cuda_device, dtype):
    # the recurrent form at inference ("Understanding Mamba from zero" sec. 2.3): one step per
    # call, the state carried through initial_state / last_state, equals one scan of all steps
    import torch
    from selective_state_space_13_b200 import scan
    w = wl.variant("m130", name="decode", batch=4, seqlen=5, dim=256, dtype=dtype, seed=190)
    inp = wl.make_inputs(w)
    t = to_device(inp, cuda_device)
    h = torch.zeros((1, w.batch, w.dim, w.dstate), dtype=torch.float32, device=cuda_device)
    outs = []
    for s in range(w.seqlen):
        o, h = scan.selective_scan_fwd(
            t["u"][:, s:s + 1].contiguous(), t["delta"][:, :, s:s + 1].contiguous(), t["A"],
            t["B"][:, :, s:s + 1].contiguous(), t["C"][:, :, s:s + 1].contiguous(), D=t["D"],
            z=t["z"][:, s:s + 1].contiguous(), delta_bias=t["delta_bias"], initial_state=h,
            return_last_state=True)
        outs.append(o)
    out = torch.cat(outs, dim=1)
    torch.cuda.synchronize()
    ref_out, ref_last = run_oracle(inp)
    tol = tol_for(w)
    assert rel_err(out_to_f64(out), ref_out) <= tol and rel_err(out_to_f64(h), ref_last) <= tol
    if dtype == wl.F32:
        # the steps differ from one unsplit scan (fp64 state) only by the fp32 rounding of the
        # state handed from step to step
        full, last = scan.selective_scan_fwd(t["u"], t["delta"], t["A"], t["B"], t["C"], D=t["D"],
                                             z=t["z"], delta_bias=t["delta_bias"], segments=1,
                                             return_last_state=True)
        assert rel_err(out_to_f64(out), out_to_f64(full)) <= 1e-5
        assert rel_err(out_to_f64(h), out_to_f64(last)) <= 1e-5


# ----------------------------------------------------------------------------- random combinations

def _random_case(i):
    """A seeded random combination of shape and options, within what the ABI accepts."""
    rng = np.random.default_rng(5000 + i)
    dtype = wl.BF16 if rng.random() < 0.7 else wl.F32
    int8 = dtype == wl.BF16 and rng.random() < 0.3
    step = 16 if int8 else (8 if dtype == wl.BF16 else 4)
    D = int(step * rng.integers(1, 200 // step + 1))
    kind = rng.integers(0, 4)
    if kind == 0:
        dirs, H, W = (wl.DIR_FORWARD,), 0, 0
        L = int(rng.integers(1, 400))
    elif kind == 1:
        dirs, H, W = (wl.DIR_FORWARD, wl.DIR_REVERSE), 0, 0
        L = int(rng.integers(1, 300))
    else:
        H, W = int(rng.integers(1, 20)), int(rng.integers(1, 20))
        L = H * W
        pool = [wl.DIR_FORWARD, wl.DIR_REVERSE, wl.DIR_COLUMN, wl.DIR_COLUMN_REVERSE]
        dirs = tuple(int(d) for d in rng.choice(pool, size=int(rng.integers(1, 5)),
                                                replace=bool(rng.random() < 0.3)))
    w = wl.Workload("rand%d" % i, int(rng.integers(1, 4)), L, D, int(rng.integers(1, 17)), dtype,
                    dirs=dirs, H=H, W=W, gate=bool(rng.random() < 0.6),
                    softplus=bool(rng.random() < 0.85),
                    bias="zero" if rng.random() < 0.2 else "loguniform",
                    dskip="normal" if rng.random() < 0.5 else "one", seed=6000 + i,
                    conv=int(rng.integers(1, 5)) if rng.random() < 0.3 else 0,
                    u_per_dir=bool(len(dirs) > 1 and rng.random() < 0.3), delta_int8=int8,
                    params_per_dir=bool(len(dirs) > 1 and rng.random() < 0.3))
    kw = dict(segments=int(rng.choice([0, 1, 2, 3, 7])))
    if rng.random() < 0.25:
        kw["initial_state"] = rng.standard_normal((w.K, w.batch, w.dim, w.dstate)).astype(np.float32)
    if rng.random() < 0.15:
        kw["zoh_exact"] = True
    if rng.random() < 0.1:
        kw["use_D"] = False
    return w, kw


@pytest.mark.parametrize("i", range(120))
def test_random_option_combinations(cuda_device, i):
    w, kw = _random_case(i)
    inp = wl.make_inputs(w)
    if not w.softplus:
        # Delta = delta_raw + bias must stay positive without softplus: the bias of each channel
        # (and direction) is raised above the largest |delta_raw| it meets
        raw = wl.inputs_f64(inp)["delta"]                       # [K, b, L, D] raw values
        need = np.abs(raw).max(axis=(1, 2)) + 0.01                 # [K, D]
        bias = need.max(axis=0) if inp["delta_bias"].ndim == 1 else need
        inp["delta_bias"] = bias.astype(np.float32)
    _check(inp, cuda_device, **kw)
