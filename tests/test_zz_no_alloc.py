"""selective_scan_fwd_noalloc, the entry point for callers that cannot allocate device memory.

Such callers (a plugin whose host owns the allocator, a server that sizes one arena at start-up,
a latency-critical loop that must not call cudaMalloc) cannot hand selective_scan_fwd a
workspace; this entry point takes its scratch from the library's own fixed device array.  The
test calls it through the C ABI, twice in a row, on problems that do need scratch (a split
sequence, whose segment carries live there, and two directions, whose fp32 per-direction outputs
live there), and checks each result against selective_scan_fwd with a caller-provided workspace,
within the parity tolerance of the other GPU tests.  It also checks that a problem needing more
scratch than the array holds is refused before anything runs.

This file is collected last on purpose: if it fails, a run that stops at the first failure has
already run every other test.
"""

import pytest

from selective_state_space_13_b200 import workloads as wl
from tests.scan_util import out_to_f64, rel_err, to_device, tol_for

pytestmark = pytest.mark.gpu


def _noalloc(t, w, out, last, segments):
    import torch
    from selective_state_space_13_b200 import scan
    shape = scan.make_shape(w.batch, w.seqlen, w.dim, w.dstate,
                            scan.SS_BF16 if w.dtype == wl.BF16 else scan.SS_F32)
    dmap = scan.make_dirmap(w.dirs, w.H, w.W)
    opts = scan.make_opts(segments=segments)
    assert 0 < scan.selective_scan_workspace_size(shape, dmap, opts) <= scan.SS_NOALLOC_SCRATCH_BYTES
    p = lambda x: 0 if x is None else int(x.data_ptr())  # noqa: E731
    st = scan.selective_scan_fwd_noalloc_raw(
        shape, p(t["u"]), p(t["delta"]), p(t["A"]), p(t["B"]), p(t["C"]), p(t["D"]), p(t["z"]),
        p(t["delta_bias"]), w.softplus, dmap, p(out), p(last),
        torch.cuda.current_stream().cuda_stream, opts)
    assert st == scan.SS_OK, scan.ss_status_str(st)


@pytest.mark.parametrize("case", ["split_sequence", "two_directions"])
def test_noalloc_matches_workspace_entry_point_twice(cuda_device, case):
    import torch
    from selective_state_space_13_b200 import scan
    if case == "split_sequence":
        w = wl.variant("m130", name="noalloc_seg", batch=2, seqlen=1500, dim=200, seed=501)
        segments = 4
    else:
        w = wl.variant("vim", name="noalloc_dirs", batch=4, dim=192, seed=502)
        segments = 0
    t = to_device(wl.make_inputs(w), cuda_device)
    ref_out, ref_last = scan.selective_scan_fwd(
        t["u"], t["delta"], t["A"], t["B"], t["C"], D=t["D"], z=t["z"],
        delta_bias=t["delta_bias"], softplus=w.softplus, dirs=w.dirs, H=w.H, W=w.W,
        return_last_state=True, segments=segments)
    torch.cuda.synchronize()
    tol = tol_for(w)
    for _ in range(2):
        out = torch.full_like(ref_out, float("nan"))
        last = torch.full_like(ref_last, float("nan"))
        _noalloc(t, w, out, last, segments)
        torch.cuda.synchronize()
        assert rel_err(out_to_f64(out), out_to_f64(ref_out)) <= tol
        assert rel_err(out_to_f64(last), out_to_f64(ref_last)) <= tol
    assert scan.selective_scan_device_status(clear=True) == scan.SS_OK


def test_noalloc_refuses_problems_beyond_its_scratch(cuda_device):
    from selective_state_space_13_b200 import scan
    w = wl.WORKLOADS["vim"]  # 77 MB of per-direction outputs: more than the fixed array
    shape = scan.make_shape(w.batch, w.seqlen, w.dim, w.dstate, scan.SS_BF16)
    dmap = scan.make_dirmap(w.dirs)
    assert scan.selective_scan_workspace_size(shape, dmap) > scan.SS_NOALLOC_SCRATCH_BYTES
    fake = 1 << 20  # never dereferenced: the size check comes first
    st = scan.selective_scan_fwd_noalloc_raw(shape, fake, fake, fake, fake, fake, 0, fake, 0, 1,
                                             dmap, fake, 0, 0)
    assert st == scan.SS_ERR_SCRATCH_LIMIT
