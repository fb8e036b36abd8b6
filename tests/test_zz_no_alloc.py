"""selective_scan_fwd_noalloc, the entry point for callers that cannot allocate device memory.

Such callers (a plugin whose host owns the allocator, a server that sizes one arena at start-up,
a latency-critical loop that must not call cudaMalloc) cannot hand selective_scan_fwd a
workspace; this entry point takes its scratch from the library's own fixed device array.  The
test calls it through the C ABI on problems that do need scratch (a split sequence, whose segment
carries live there, and two directions, whose fp32 per-direction outputs live there).  First a
call on NaN inputs of another shape fills the shared array with NaN; then two calls in a row,
each on its own seeded inputs, must give results bit-identical to selective_scan_fwd with a
caller-provided workspace (same kernels, same launch plan, deterministic).  So every scratch
value a call reads must have been written by that same call.  It also checks that a problem
needing more scratch than the array holds is refused before anything runs.

This file is collected last on purpose: if it fails, a run that stops at the first failure has
already run every other test.
"""

import pytest

from selective_state_space_13_b200 import workloads as wl
from tests.scan_util import to_device

pytestmark = pytest.mark.gpu

CASES = {
    # name: (workload, segments)
    "split_sequence": (dict(base="m130", batch=2, seqlen=1500, dim=200), 4),
    "two_directions": (dict(base="vim", batch=4, dim=192), 0),
}


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


def _workload(spec, seed):
    spec = dict(spec)
    base = spec.pop("base")
    return wl.variant(base, name="noalloc_%s_%d" % (base, seed), seed=seed, **spec)


def _poison_scratch(device):
    # NaN inputs of other shapes through both scratch regions (carries, per-direction outputs)
    import torch
    for spec, segments in (dict(base="m130", batch=3, seqlen=2000, dim=256), 5), \
                          (dict(base="vim", batch=6, dim=256), 0):
        w = _workload(spec, 999)
        t = to_device(wl.make_inputs(w), device)
        t["u"].fill_(float("nan"))
        out = torch.empty((w.batch, w.seqlen, w.dim), dtype=t["u"].dtype, device=device)
        last = torch.empty((w.K, w.batch, w.dim, w.dstate), dtype=torch.float32, device=device)
        _noalloc(t, w, out, last, segments)
        torch.cuda.synchronize()
        assert torch.isnan(last).all()


@pytest.mark.parametrize("case", sorted(CASES))
def test_noalloc_matches_workspace_entry_point_twice(cuda_device, case):
    import torch
    from selective_state_space_13_b200 import scan
    spec, segments = CASES[case]
    _poison_scratch(cuda_device)
    for call, seed in enumerate((501, 502)):
        w = _workload(spec, seed + 10 * len(case))
        t = to_device(wl.make_inputs(w), cuda_device)
        ref_out, ref_last = scan.selective_scan_fwd(
            t["u"], t["delta"], t["A"], t["B"], t["C"], D=t["D"], z=t["z"],
            delta_bias=t["delta_bias"], softplus=w.softplus, dirs=w.dirs, H=w.H, W=w.W,
            return_last_state=True, segments=segments)
        out = torch.full_like(ref_out, float("nan"))
        last = torch.full_like(ref_last, float("nan"))
        _noalloc(t, w, out, last, segments)
        torch.cuda.synchronize()
        assert torch.equal(out, ref_out), (case, call)
        assert torch.equal(last, ref_last), (case, call)
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
