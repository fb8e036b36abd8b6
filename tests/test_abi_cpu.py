"""The C ABI on the host, without a GPU: the library loads, exports every symbol the header
declares, rejects bad arguments with the documented status before touching any device, and its
index map (the very function the kernels use) matches the oracle's independent one bit for bit."""

import ctypes
import os
import re

import pytest

import oracle
from selective_state_space_13_b200 import scan

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "selective_scan.h")


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*"
                                 r"([A-Za-z_][A-Za-z0-9_]*)\s*\(", text, flags=re.M)))


def test_library_exports_every_declared_symbol():
    lib = scan.load()
    names = header_functions()
    assert set(names) == set(scan.EXPORTED), names
    for name in names:
        assert hasattr(lib, name), name
    assert scan.ss_abi_version() == 5


def test_status_strings():
    for code, name in scan.STATUS_NAMES.items():
        assert scan.ss_status_str(code).startswith(name)


def _shape(**kw):
    base = dict(batch=2, seqlen=64, dim=32, dstate=16, io_dtype=scan.SS_BF16)
    base.update(kw)
    return scan.make_shape(**base)


FAKE = 1 << 20  # a 16-byte aligned, never dereferenced address: validation must fail first


@pytest.mark.parametrize("kw,expect", [
    (dict(dstate=0), 2),
    (dict(dstate=17), 6),
    (dict(batch=-1), 2),
    (dict(seqlen=1 << 31), 2),
    (dict(io_dtype=7), 3),
    (dict(dim=12), 4),            # 12 * 2 bytes is not a multiple of 16
])
def test_shape_validation(kw, expect):
    sh = _shape(**kw)
    with pytest.raises(scan.ScanError) as ei:
        scan.selective_scan_workspace_size(sh)
    assert ei.value.status == expect
    st = scan.selective_scan_fwd_raw(sh, FAKE, FAKE, FAKE, FAKE, FAKE, 0, 0, 0, 1, None, FAKE, 0,
                                     0, 0, 0)
    assert st == expect


@pytest.mark.parametrize("dirs,H,W,expect", [
    ((), 0, 0, 5), ((0, 1, 2, 3, 0), 8, 8, 5), ((4,), 0, 0, 5), ((2,), 8, 7, 5),
    ((2,), 0, 64, 5), ((0, 1), 0, 0, 0), ((2, 3), 8, 8, 0), ((3,), 4, 16, 0)])
def test_dirmap_validation(dirs, H, W, expect):
    sh = _shape()
    dm = scan.make_dirmap(dirs, H, W) if dirs else scan.SsDirectionMap()
    if len(dirs) > 4:
        dm.num_dirs = 5
    if expect:
        with pytest.raises(scan.ScanError) as ei:
            scan.selective_scan_workspace_size(sh, dm)
        assert ei.value.status == expect
    else:
        assert scan.selective_scan_workspace_size(sh, dm) >= 0


def test_null_alignment_and_workspace_errors():
    sh = _shape()
    args = [FAKE] * 5
    # missing required pointers
    for i in range(5):
        a = list(args)
        a[i] = 0
        u, delta, A, B, C = a
        st = scan.selective_scan_fwd_raw(sh, u, delta, A, B, C, 0, 0, 0, 1, None, FAKE, 0, 0, 0, 0)
        assert st == 1
    st = scan.selective_scan_fwd_raw(sh, FAKE, FAKE, FAKE, FAKE, FAKE, 0, 0, 0, 1, None, 0, 0, 0, 0, 0)
    assert st == 1
    # misaligned io pointer / float pointer
    st = scan.selective_scan_fwd_raw(sh, FAKE + 8, FAKE, FAKE, FAKE, FAKE, 0, 0, 0, 1, None, FAKE,
                                     0, 0, 0, 0)
    assert st == 4
    st = scan.selective_scan_fwd_raw(sh, FAKE, FAKE, FAKE + 2, FAKE, FAKE, 0, 0, 0, 1, None, FAKE,
                                     0, 0, 0, 0)
    assert st == 4
    # two directions need a workspace
    dm = scan.make_dirmap((0, 1))
    need = scan.selective_scan_workspace_size(sh, dm)
    assert need > 0
    st = scan.selective_scan_fwd_raw(sh, FAKE, FAKE, FAKE, FAKE, FAKE, 0, 0, 0, 1, dm, FAKE, 0,
                                     0, 0, 0)
    assert st == 8
    st = scan.selective_scan_fwd_raw(sh, FAKE, FAKE, FAKE, FAKE, FAKE, 0, 0, 0, 1, dm, FAKE, 0,
                                     FAKE, need - 1, 0)
    assert st == 8
    # unknown option bits / reserved fields
    o = scan.make_opts(flags=4)
    with pytest.raises(scan.ScanError):
        scan.selective_scan_workspace_size(sh, None, o)
    o = scan.make_opts(segments=-1)
    with pytest.raises(scan.ScanError):
        scan.selective_scan_workspace_size(sh, None, o)
    o = scan.make_opts()
    o.reserved = 1
    with pytest.raises(scan.ScanError):
        scan.selective_scan_workspace_size(sh, None, o)


def test_input_per_direction_flag_accepted():
    sh = _shape()
    o = scan.make_opts(flags=scan.SS_FLAG_U_PER_DIRECTION | scan.SS_FLAG_PARAMS_PER_DIRECTION)
    assert scan.selective_scan_workspace_size(sh, scan.make_dirmap((0, 0)), o) > 0


def test_int8_delta_options_validated():
    I8 = scan.SS_FLAG_DELTA_INT8
    ok = scan.make_opts(flags=I8, delta_scale=FAKE)
    assert scan.selective_scan_workspace_size(_shape(), None, ok) == 0
    cases = [(_shape(io_dtype=scan.SS_F32), ok, 6),          # int8 delta needs bf16 io
             (_shape(), scan.make_opts(flags=I8), 1),          # scales missing
             (_shape(dim=40), ok, 4),                           # code rows not 16-byte multiples
             (_shape(), scan.make_opts(delta_scale=FAKE), 6)]   # scales without the flag
    for sh, o, want in cases:
        with pytest.raises(scan.ScanError) as e:
            scan.selective_scan_workspace_size(sh, None, o)
        assert e.value.status == want
    st = scan.selective_scan_fwd_raw(_shape(), FAKE, FAKE, FAKE, FAKE, FAKE, 0, 0, 0, 1, None, FAKE,
                                     0, 0, 0, 0, scan.make_opts(flags=I8, delta_scale=FAKE + 2))
    assert st == 4


def test_conv_options_validated():
    sh = _shape()
    ok = scan.make_opts(conv_weight=FAKE, conv_bias=FAKE, conv_width=4)
    assert scan.selective_scan_workspace_size(sh, None, ok) == 0
    for bad in (dict(conv_weight=FAKE, conv_width=0), dict(conv_weight=FAKE, conv_width=5),
                dict(conv_weight=FAKE, conv_width=-1), dict(conv_bias=FAKE),
                dict(conv_width=4)):
        with pytest.raises(scan.ScanError) as e:
            scan.selective_scan_workspace_size(sh, None, scan.make_opts(**bad))
        assert e.value.status == 6, bad
    # misaligned taps or bias are refused before any launch
    for kw in (dict(conv_weight=FAKE + 2, conv_width=4),
               dict(conv_weight=FAKE, conv_bias=FAKE + 1, conv_width=4)):
        st = scan.selective_scan_fwd_raw(sh, FAKE, FAKE, FAKE, FAKE, FAKE, 0, 0, 0, 1, None,
                                         FAKE, 0, 0, 0, 0, scan.make_opts(**kw))
        assert st == 4, kw


def test_workspace_sizes():
    # one direction, one segment: no scratch
    assert scan.selective_scan_workspace_size(_shape(), None, scan.make_opts(segments=1)) == 0
    # segments: carries of K*b*S*D*(N+1) floats
    n = scan.selective_scan_workspace_size(_shape(seqlen=4096), None, scan.make_opts(segments=4))
    assert n >= 2 * 4 * 32 * 17 * 4
    # directions: per-direction fp32 outputs
    n = scan.selective_scan_workspace_size(_shape(), scan.make_dirmap((0, 1)))
    assert n >= 2 * 2 * 64 * 32 * 4


def test_empty_problem_needs_no_pointers():
    for kw in (dict(batch=0), dict(seqlen=0), dict(dim=0)):
        sh = _shape(**kw)
        st = scan.selective_scan_fwd_raw(sh, 0, 0, FAKE if kw.get("dim", 1) else 0, 0, 0, 0, 0, 0,
                                         1, None, 0, 0, 0, 0, 0)
        assert st == 0, kw


@pytest.mark.parametrize("H,W", [(56, 56), (5, 7), (1, 13), (13, 1), (3, 200)])
def test_index_map_bit_exact_against_oracle(H, W):
    L = H * W
    dm = scan.make_dirmap((0, 1, 2, 3), H, W)
    for k, d in enumerate((0, 1, 2, 3)):
        got = [scan.ss_direction_position(dm, k, L, t) for t in range(L)]
        ref = [oracle.position(d, L, t, H, W) for t in range(L)]
        assert got == ref
        assert sorted(got) == list(range(L))
    assert scan.ss_direction_position(dm, 4, L, 0) == -1
    assert scan.ss_direction_position(dm, 0, L, L) == -1
    assert scan.ss_direction_position(None, 0, L, 3) == 3


def test_index_map_large_L():
    L = 131072
    for t in (0, 1, 65535, L - 1):
        assert scan.ss_direction_position(None, 0, L, t) == t
        dm = scan.make_dirmap((1,))
        assert scan.ss_direction_position(dm, 0, L, t) == L - 1 - t


def test_host_buffer_call_checks_arguments_before_any_cuda_call():
    # selective_scan_fwd_host validates every argument once, up front: shapes and dtypes of the
    # host tensors first, then that the parameters are device tensors
    import torch
    dev = torch.device("cuda", 0)
    b, L, D, N = 2, 48, 16, 4
    u = torch.zeros((b, L, D), dtype=torch.bfloat16)
    delta = torch.zeros((1, b, L, D), dtype=torch.bfloat16)
    B = torch.zeros((1, b, L, N), dtype=torch.bfloat16)
    C = torch.zeros((1, b, L, N), dtype=torch.bfloat16)
    A = torch.zeros((D, N), dtype=torch.float32)  # not on the device
    with pytest.raises(ValueError, match="delta"):
        scan.selective_scan_fwd_host(u, delta[:, :, :-1], A, B, C, device=dev)
    with pytest.raises(TypeError, match="B"):
        scan.selective_scan_fwd_host(u, delta, A, B.float(), C, device=dev)
    with pytest.raises(ValueError, match="z"):
        scan.selective_scan_fwd_host(u, delta, A, B, C, z=u[:, 1:], device=dev)
    with pytest.raises(ValueError, match="A must be a CUDA tensor"):
        scan.selective_scan_fwd_host(u, delta, A, B, C, device=dev)


def test_host_entry_point_validation():
    # selective_scan_fwd_host and its workspace size validate like the device entry point, and
    # check the piece count, the workspace and its alignment before any CUDA call
    sh = _shape(batch=4, seqlen=256)
    for bad in (0, -1, scan.SS_HOST_MAX_PIECES + 1):
        with pytest.raises(scan.ScanError) as e:
            scan.selective_scan_host_workspace_size(sh, None, None, bad)
        assert e.value.status == 6
    n1 = scan.selective_scan_host_workspace_size(sh, None, None, 1)
    n4 = scan.selective_scan_host_workspace_size(sh, None, None, 4)
    # two slots of the largest piece: one piece holds all rows, four pieces one row each
    assert n1 > n4 > 0
    assert scan.selective_scan_host_workspace_size(_shape(batch=0), None, None, 4) == 0
    with pytest.raises(scan.ScanError) as e:
        scan.selective_scan_host_workspace_size(_shape(dstate=17), None, None, 4)
    assert e.value.status == 6

    def call(u=FAKE, ws=FAKE, nws=None, pieces=4, A=FAKE):
        return scan.selective_scan_fwd_host_raw(sh, u, FAKE, A, FAKE, FAKE, 0, 0, 0, 1, None, FAKE,
                                                0, ws, n4 if nws is None else nws, pieces, 0)
    assert call(u=0) == 1                 # a missing input
    assert call(A=0) == 1                 # a missing parameter
    assert call(ws=0) == 8                # no workspace
    assert call(nws=n4 - 1) == 8          # too small
    assert call(ws=FAKE + 16) == 4        # not 256-byte aligned
    assert call(pieces=0) == 6
    # well-formed: without a device the runtime fails, and says so
    assert call() == 7
