"""Python binding of the C ABI in include/selective_scan.h (argument marshalling only).

Every step of the scan runs in the CUDA library libss_b200.so; this module checks tensor
shapes, dtypes and devices, allocates outputs and the workspace through PyTorch when the
caller did not pass them, and calls the library on the current CUDA stream.  There is no CPU
path: without the library, or without a CUDA device, every call raises.

The functions carry the C names: selective_scan_fwd, selective_scan_workspace_size,
selective_scan_fwd_host, selective_scan_host_workspace_size, selective_scan_fwd_noalloc,
ss_direction_position, selective_scan_device_status, ss_status_str, ss_abi_version.
"""

from __future__ import annotations

import ctypes
import hashlib
import os
import threading

from . import build as _build

SS_OK = 0
SS_ERR_SCRATCH_LIMIT = 10
SS_F32, SS_BF16 = 0, 1
SS_DIR_FWD, SS_DIR_REV, SS_DIR_COL, SS_DIR_COL_REV = 0, 1, 2, 3
SS_FLAG_GENERIC_A = 1
SS_FLAG_ZOH_EXACT = 2
SS_FLAG_TEST_WAIT_TIMEOUT = 8
SS_FLAG_U_PER_DIRECTION = 16
SS_FLAG_DELTA_INT8 = 32
SS_FLAG_PARAMS_PER_DIRECTION = 64
SS_ERR_DEVICE_TIMEOUT = 9
SS_MAX_DSTATE = 16
SS_MAX_DIRS = 4
SS_MAX_CONV_WIDTH = 4

STATUS_NAMES = {0: "SS_OK", 1: "SS_ERR_NULL", 2: "SS_ERR_SHAPE", 3: "SS_ERR_DTYPE",
                4: "SS_ERR_ALIGN", 5: "SS_ERR_DIRMAP", 6: "SS_ERR_UNSUPPORTED", 7: "SS_ERR_CUDA",
                8: "SS_ERR_WORKSPACE", 9: "SS_ERR_DEVICE_TIMEOUT", 10: "SS_ERR_SCRATCH_LIMIT",
                11: "SS_ERR_DEVICE"}
SS_ERR_DEVICE = 11
SS_HOST_MAX_PIECES = 64
SS_NOALLOC_SCRATCH_BYTES = 16 << 20

EXPORTED = ("selective_scan_workspace_size", "selective_scan_fwd", "ss_direction_position",
            "selective_scan_device_status", "ss_status_str", "ss_abi_version",
            "selective_scan_fwd_noalloc", "selective_scan_host_workspace_size",
            "selective_scan_fwd_host")


class SsShape(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64), ("dim", ctypes.c_int64),
                ("dstate", ctypes.c_int64), ("io_dtype", ctypes.c_int32),
                ("reserved", ctypes.c_int32)]


class SsDirectionMap(ctypes.Structure):
    _fields_ = [("num_dirs", ctypes.c_int32), ("dir", ctypes.c_int32 * SS_MAX_DIRS),
                ("H", ctypes.c_int32), ("W", ctypes.c_int32)]


class SsLaunchOpts(ctypes.Structure):
    _fields_ = [("segments", ctypes.c_int32), ("flags", ctypes.c_int32),
                ("scan_begin_event", ctypes.c_void_p), ("scan_end_event", ctypes.c_void_p),
                ("initial_state", ctypes.c_void_p), ("conv_weight", ctypes.c_void_p),
                ("conv_bias", ctypes.c_void_p), ("conv_width", ctypes.c_int32),
                ("reserved", ctypes.c_int32), ("delta_scale", ctypes.c_void_p)]


class ScanError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__("%s%s" % (ss_status_str(status), (": " + what) if what else ""))


_lock = threading.Lock()
_lib = None


def _source_digest() -> str:
    h = hashlib.sha256()
    for f in _build.SOURCES + _build.HEADERS:
        with open(f, "rb") as fh:
            h.update(os.path.basename(f).encode())
            h.update(fh.read())
    return h.hexdigest()


def library_path() -> str:
    return _build.LIB


def ensure_built() -> str:
    """Build libss_b200.so when it is missing or its sources changed (by content)."""
    stamp = _build.LIB + ".srchash"
    digest = _source_digest()
    have = None
    if os.path.exists(_build.LIB) and os.path.exists(stamp):
        with open(stamp) as fh:
            have = fh.read().strip()
    if have != digest:
        _build.build(force=True)
        with open(stamp, "w") as fh:
            fh.write(digest)
    return _build.LIB


def load():
    """Load the CUDA library (building it first if needed) and declare its signatures."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        path = ensure_built()
        lib = ctypes.CDLL(path)
        vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
        lib.selective_scan_workspace_size.restype = ctypes.c_int
        lib.selective_scan_workspace_size.argtypes = [ctypes.POINTER(SsShape),
                                                      ctypes.POINTER(SsDirectionMap),
                                                      ctypes.POINTER(SsLaunchOpts),
                                                      ctypes.POINTER(sz)]
        lib.selective_scan_fwd.restype = ctypes.c_int
        lib.selective_scan_fwd.argtypes = [ctypes.POINTER(SsShape), vp, vp, vp, vp, vp, vp, vp, vp,
                                           i32, ctypes.POINTER(SsDirectionMap), vp, vp, vp, sz, vp,
                                           ctypes.POINTER(SsLaunchOpts)]
        lib.ss_direction_position.restype = i64
        lib.ss_direction_position.argtypes = [ctypes.POINTER(SsDirectionMap), i32, i64, i64]
        lib.selective_scan_device_status.restype = ctypes.c_int
        lib.selective_scan_device_status.argtypes = [vp, i32]
        lib.ss_status_str.restype = ctypes.c_char_p
        lib.ss_status_str.argtypes = [ctypes.c_int]
        lib.ss_abi_version.restype = i32
        lib.ss_abi_version.argtypes = []
        lib.selective_scan_host_workspace_size.restype = ctypes.c_int
        lib.selective_scan_host_workspace_size.argtypes = [ctypes.POINTER(SsShape),
                                                           ctypes.POINTER(SsDirectionMap),
                                                           ctypes.POINTER(SsLaunchOpts), i32,
                                                           ctypes.POINTER(sz)]
        lib.selective_scan_fwd_host.restype = ctypes.c_int
        lib.selective_scan_fwd_host.argtypes = [ctypes.POINTER(SsShape), vp, vp, vp, vp, vp, vp, vp,
                                                vp, i32, ctypes.POINTER(SsDirectionMap), vp, vp,
                                                vp, sz, i32, vp, ctypes.POINTER(SsLaunchOpts)]
        lib.selective_scan_fwd_noalloc.restype = ctypes.c_int
        lib.selective_scan_fwd_noalloc.argtypes = [ctypes.POINTER(SsShape), vp, vp, vp, vp, vp, vp,
                                                   vp, vp, i32, ctypes.POINTER(SsDirectionMap), vp,
                                                   vp, vp, ctypes.POINTER(SsLaunchOpts)]
        _lib = lib
        return lib


# ----------------------------------------------------------------------------- thin C wrappers

def ss_status_str(status: int) -> str:
    try:
        return load().ss_status_str(int(status)).decode()
    except OSError:
        return STATUS_NAMES.get(int(status), "unknown ss_status %d" % status)


def ss_abi_version() -> int:
    return int(load().ss_abi_version())


def make_shape(batch, seqlen, dim, dstate, io_dtype) -> SsShape:
    return SsShape(int(batch), int(seqlen), int(dim), int(dstate), int(io_dtype), 0)


def make_dirmap(dirs=(SS_DIR_FWD,), H=0, W=0) -> SsDirectionMap:
    m = SsDirectionMap()
    m.num_dirs = len(dirs)
    for i, d in enumerate(list(dirs)[:SS_MAX_DIRS]):
        m.dir[i] = int(d)
    m.H, m.W = int(H), int(W)
    return m


def make_opts(segments=0, flags=0, events=None, initial_state=0, conv_weight=0, conv_bias=0,
              conv_width=0, delta_scale=0) -> SsLaunchOpts:
    """events: optional (begin, end) torch.cuda.Event pair, recorded by the library around its
    main scan launch on the call's stream (each must have been recorded once before, so that
    its CUDA event exists).  initial_state: device address of a [K, batch, D, N] fp32 array
    (0 = zero state).  conv_weight / conv_bias: device addresses of the [K, D, conv_width] and
    [K, D] fp32 causal-convolution taps and bias (0 = none).  delta_scale: device address of
    the [D] fp32 scales of int8 delta codes (used with SS_FLAG_DELTA_INT8)."""
    o = SsLaunchOpts()
    o.segments, o.flags = int(segments), int(flags)
    o.initial_state = int(initial_state) or None
    o.conv_weight = int(conv_weight) or None
    o.conv_bias = int(conv_bias) or None
    o.conv_width = int(conv_width)
    o.delta_scale = int(delta_scale) or None
    if events is not None:
        o.scan_begin_event = int(events[0].cuda_event) or None
        o.scan_end_event = int(events[1].cuda_event) or None
    return o


def selective_scan_workspace_size(shape: SsShape, dmap: SsDirectionMap | None = None,
                                  opts: SsLaunchOpts | None = None) -> int:
    n = ctypes.c_size_t(0)
    st = load().selective_scan_workspace_size(ctypes.byref(shape),
                                              ctypes.byref(dmap) if dmap is not None else None,
                                              ctypes.byref(opts) if opts is not None else None,
                                              ctypes.byref(n))
    if st != SS_OK:
        raise ScanError(st, "selective_scan_workspace_size")
    return int(n.value)


def ss_direction_position(dmap: SsDirectionMap | None, k: int, L: int, t: int) -> int:
    return int(load().ss_direction_position(ctypes.byref(dmap) if dmap is not None else None,
                                            int(k), int(L), int(t)))


def selective_scan_device_status(stream=None, clear: bool = True) -> int:
    """Synchronise the stream and return SS_OK or SS_ERR_DEVICE_TIMEOUT (see the C header)."""
    return int(load().selective_scan_device_status(_stream_handle(stream), int(bool(clear))))


def selective_scan_fwd_raw(shape: SsShape, u, delta, A, B, C, Dskip, z, delta_bias, softplus,
                           dmap, out, last_state, workspace, workspace_bytes, stream,
                           opts=None) -> int:
    """Direct call with integer device addresses (0 = NULL); returns the ss_status."""
    return int(load().selective_scan_fwd(
        ctypes.byref(shape), u or None, delta or None, A or None, B or None, C or None,
        Dskip or None, z or None, delta_bias or None, int(bool(softplus)),
        ctypes.byref(dmap) if dmap is not None else None, out or None, last_state or None,
        workspace or None, int(workspace_bytes), stream or None,
        ctypes.byref(opts) if opts is not None else None))


def selective_scan_fwd_noalloc_raw(shape: SsShape, u, delta, A, B, C, Dskip, z, delta_bias,
                                   softplus, dmap, out, last_state, stream, opts=None) -> int:
    """selective_scan_fwd_noalloc with integer device addresses (0 = NULL); returns the
    ss_status.  For callers that cannot allocate device memory: the scratch is the library's own
    fixed array (SS_NOALLOC_SCRATCH_BYTES), shared by all calls."""
    return int(load().selective_scan_fwd_noalloc(
        ctypes.byref(shape), u or None, delta or None, A or None, B or None, C or None,
        Dskip or None, z or None, delta_bias or None, int(bool(softplus)),
        ctypes.byref(dmap) if dmap is not None else None, out or None, last_state or None,
        stream or None, ctypes.byref(opts) if opts is not None else None))


# ----------------------------------------------------------------------------- torch front end

def _stream_handle(stream):
    import torch
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _ptr(t):
    return 0 if t is None else int(t.data_ptr())


def _io_code(dtype):
    import torch
    if dtype == torch.float32:
        return SS_F32
    if dtype == torch.bfloat16:
        return SS_BF16
    raise TypeError("io tensors must be float32 or bfloat16, got %s" % dtype)


def _check(t, name, shape, dtype, device):
    if t is None:
        return
    if not t.is_cuda or t.device != device:
        raise ValueError("%s must be a CUDA tensor on %s" % (name, device))
    if tuple(t.shape) != tuple(shape):
        raise ValueError("%s must have shape %s, got %s" % (name, tuple(shape), tuple(t.shape)))
    if t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)


_ws_cache = {}


def _workspace(nbytes, device):
    import torch
    key = (device.index, torch.cuda.current_stream(device).cuda_stream)
    buf = _ws_cache.get(key)
    if buf is None or buf.numel() < nbytes:
        buf = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=device)
        _ws_cache[key] = buf
    return buf


def selective_scan_fwd(u, delta, A, B, C, D=None, z=None, delta_bias=None, softplus=True,
                       dirs=(SS_DIR_FWD,), H=0, W=0, out=None, last_state=None,
                       return_last_state=False, workspace=None, stream=None, segments=0,
                       flags=0, events=None, initial_state=None, zoh_exact=False,
                       conv_weight=None, conv_bias=None, delta_scale=None):
    """Selective scan forward on CUDA tensors.

    u, z: [batch, L, D] (u may be [K, batch, L, D]: direction k scans its own input u[k],
    e.g. the two modalities of a cross-modal scan); delta: [K, batch, L, D] (or [batch, L, D] when K = 1); B, C:
    [K, batch, L, N] (or [batch, L, N]); A: [D, N] float32; D (skip) and delta_bias: [D] float32
    (or A [K, D, N], D and delta_bias [K, D]: parameters per direction).
    u, delta, B, C, z share one dtype (float32 or bfloat16); out has that dtype.
    initial_state: [K, batch, D, N] float32 state before step 0 (None = zero); zoh_exact: use
    Bbar = (exp(Delta*A) - 1) / A * B instead of Delta*B.
    conv_weight: [K, D, width] float32 (width <= 4), the causal depthwise convolution each
    direction applies to u along its own scan order, followed by SiLU (None = no convolution);
    conv_bias: [K, D] float32 or None.  delta may be int8 codes (bfloat16 io only) with
    delta_scale [D] float32: the raw value is code * delta_scale[d].
    Returns out, or (out, last_state [K, batch, D, N] float32) with return_last_state.
    """
    import torch
    device = u.device
    K = len(dirs)
    if u.dim() == 4 and u.shape[0] == K:
        flags = int(flags) | SS_FLAG_U_PER_DIRECTION
    elif u.dim() != 3:
        raise ValueError("u must be [batch, L, D] or [K, batch, L, D]")
    batch, L, Dm = u.shape[-3:]
    if delta.dim() == 3:
        delta = delta.unsqueeze(0)
    if B.dim() == 3:
        B = B.unsqueeze(0)
    if C.dim() == 3:
        C = C.unsqueeze(0)
    N = A.shape[-1]
    pshape = (Dm,)
    if A.dim() == 3:
        flags = int(flags) | SS_FLAG_PARAMS_PER_DIRECTION
        pshape = (K, Dm)
    io = u.dtype
    _io_code(io)
    _check(u, "u", tuple(u.shape[:-3]) + (batch, L, Dm), io, device)
    if delta.dtype == torch.int8:
        if delta_scale is None:
            raise ValueError("int8 delta needs delta_scale")
        flags = int(flags) | SS_FLAG_DELTA_INT8
        _check(delta, "delta", (K, batch, L, Dm), torch.int8, device)
    else:
        _check(delta, "delta", (K, batch, L, Dm), io, device)
    _check(delta_scale, "delta_scale", (Dm,), torch.float32, device)
    _check(B, "B", (K, batch, L, N), io, device)
    _check(C, "C", (K, batch, L, N), io, device)
    _check(z, "z", (batch, L, Dm), io, device)
    _check(A, "A", pshape[:-1] + (Dm, N), torch.float32, device)
    _check(D, "D", pshape, torch.float32, device)
    _check(delta_bias, "delta_bias", pshape, torch.float32, device)
    if out is None:
        out = torch.empty((batch, L, Dm), dtype=io, device=device)
    _check(out, "out", (batch, L, Dm), io, device)
    if return_last_state and last_state is None:
        last_state = torch.empty((K, batch, Dm, N), dtype=torch.float32, device=device)
    _check(last_state, "last_state", (K, batch, Dm, N), torch.float32, device)
    _check(initial_state, "initial_state", (K, batch, Dm, N), torch.float32, device)
    width = 0
    if conv_weight is not None:
        if conv_weight.dim() != 3:
            raise ValueError("conv_weight must be [K, D, width]")
        width = int(conv_weight.shape[2])
        _check(conv_weight, "conv_weight", (K, Dm, width), torch.float32, device)
    elif conv_bias is not None:
        raise ValueError("conv_bias needs conv_weight")
    _check(conv_bias, "conv_bias", (K, Dm), torch.float32, device)
    if zoh_exact:
        flags = int(flags) | SS_FLAG_ZOH_EXACT
    shape = make_shape(batch, L, Dm, N, _io_code(io))
    dmap = make_dirmap(dirs, H, W)
    opts = make_opts(segments, flags, events, _ptr(initial_state), _ptr(conv_weight),
                     _ptr(conv_bias), width, _ptr(delta_scale))
    nws = selective_scan_workspace_size(shape, dmap, opts)
    if workspace is None and nws > 0:
        workspace = _workspace(nws, device)
    wsb = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = selective_scan_fwd_raw(shape, _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                                _ptr(z), _ptr(delta_bias), softplus, dmap, _ptr(out),
                                _ptr(last_state), _ptr(workspace), wsb, _stream_handle(stream),
                                opts)
    if st != SS_OK:
        raise ScanError(st, "selective_scan_fwd")
    return (out, last_state) if return_last_state else out


# ----------------------------------------------------------------------------- host buffers

def _check_host(t, name, shape, dtype):
    if t is None:
        return
    if t.is_cuda:
        raise ValueError("%s must be a host (CPU) tensor" % name)
    if tuple(t.shape) != tuple(shape):
        raise ValueError("%s must have shape %s, got %s" % (name, tuple(shape), tuple(t.shape)))
    if t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)


def selective_scan_host_workspace_size(shape: SsShape, dmap: SsDirectionMap | None, opts,
                                       pieces: int) -> int:
    n = ctypes.c_size_t(0)
    st = load().selective_scan_host_workspace_size(
        ctypes.byref(shape), ctypes.byref(dmap) if dmap is not None else None,
        ctypes.byref(opts) if opts is not None else None, int(pieces), ctypes.byref(n))
    if st != SS_OK:
        raise ScanError(st, "selective_scan_host_workspace_size")
    return int(n.value)


def selective_scan_fwd_host_raw(shape: SsShape, u, delta, A, B, C, Dskip, z, delta_bias, softplus,
                                dmap, out, last_state, workspace, workspace_bytes, pieces, stream,
                                opts=None) -> int:
    """selective_scan_fwd_host with integer addresses (host addresses for u, delta, B, C, z,
    out and last_state; device addresses for the rest; 0 = NULL); returns the ss_status."""
    return int(load().selective_scan_fwd_host(
        ctypes.byref(shape), u or None, delta or None, A or None, B or None, C or None,
        Dskip or None, z or None, delta_bias or None, int(bool(softplus)),
        ctypes.byref(dmap) if dmap is not None else None, out or None, last_state or None,
        workspace or None, int(workspace_bytes), int(pieces), stream or None,
        ctypes.byref(opts) if opts is not None else None))


def selective_scan_fwd_host(u, delta, A, B, C, D=None, z=None, delta_bias=None, softplus=True,
                            dirs=(SS_DIR_FWD,), H=0, W=0, out=None, last_state=None,
                            return_last_state=False, flags=0, initial_state=None,
                            zoh_exact=False, conv_weight=None, conv_bias=None, delta_scale=None,
                            chunks=8, device=None, stream=None):
    """Selective scan of inputs held in host memory, with the results written back to host
    memory: one call of the C entry point selective_scan_fwd_host.

    u, delta, B, C, z (and out, last_state) are CPU tensors -- pinned, so that the copies are
    asynchronous -- with the shapes of selective_scan_fwd; A, D, delta_bias, conv_weight,
    conv_bias, delta_scale and initial_state are parameters already on the device.  The library
    cuts the work into `chunks` pieces and pipelines the host->device copies, the scans and the
    device->host copies of successive pieces on its own streams, ordered after the current
    stream, which continues once everything is done (synchronise it before reading out).
    Returns out, or (out, last_state) with return_last_state.
    """
    import torch
    if device is None:
        device = torch.device("cuda", torch.cuda.current_device())
    K = len(dirs)
    if delta.dim() == 3:
        delta = delta.unsqueeze(0)
    if B.dim() == 3:
        B = B.unsqueeze(0)
    if C.dim() == 3:
        C = C.unsqueeze(0)
    u_per_dir = u.dim() == 4
    if u_per_dir and u.shape[0] != K:
        raise ValueError("u must be [batch, L, D] or [K, batch, L, D]")
    batch, L, Dm = u.shape[-3:]
    N = A.shape[-1]
    io = u.dtype
    io_code = _io_code(io)
    if u_per_dir:
        flags = int(flags) | SS_FLAG_U_PER_DIRECTION
    pshape = (Dm,)
    if A.dim() == 3:
        flags = int(flags) | SS_FLAG_PARAMS_PER_DIRECTION
        pshape = (K, Dm)
    if zoh_exact:
        flags = int(flags) | SS_FLAG_ZOH_EXACT
    _check_host(u, "u", tuple(u.shape[:-3]) + (batch, L, Dm), io)
    if delta.dtype == torch.int8:
        if delta_scale is None:
            raise ValueError("int8 delta needs delta_scale")
        flags = int(flags) | SS_FLAG_DELTA_INT8
        _check_host(delta, "delta", (K, batch, L, Dm), torch.int8)
    else:
        _check_host(delta, "delta", (K, batch, L, Dm), io)
    _check_host(B, "B", (K, batch, L, N), io)
    _check_host(C, "C", (K, batch, L, N), io)
    _check_host(z, "z", (batch, L, Dm), io)
    _check(A, "A", pshape[:-1] + (Dm, N), torch.float32, device)
    _check(D, "D", pshape, torch.float32, device)
    _check(delta_bias, "delta_bias", pshape, torch.float32, device)
    _check(delta_scale, "delta_scale", (Dm,), torch.float32, device)
    _check(initial_state, "initial_state", (K, batch, Dm, N), torch.float32, device)
    width = 0
    if conv_weight is not None:
        if conv_weight.dim() != 3:
            raise ValueError("conv_weight must be [K, D, width]")
        width = int(conv_weight.shape[2])
        _check(conv_weight, "conv_weight", (K, Dm, width), torch.float32, device)
    elif conv_bias is not None:
        raise ValueError("conv_bias needs conv_weight")
    _check(conv_bias, "conv_bias", (K, Dm), torch.float32, device)
    if out is None:
        out = torch.empty((batch, L, Dm), dtype=io, pin_memory=True)
    _check_host(out, "out", (batch, L, Dm), io)
    if return_last_state and last_state is None:
        last_state = torch.empty((K, batch, Dm, N), dtype=torch.float32, pin_memory=True)
    _check_host(last_state, "last_state", (K, batch, Dm, N), torch.float32)

    shape = make_shape(batch, L, Dm, N, io_code)
    dmap = make_dirmap(dirs, H, W)
    opts = make_opts(0, flags, None, _ptr(initial_state), _ptr(conv_weight), _ptr(conv_bias),
                     width, _ptr(delta_scale))
    nws = selective_scan_host_workspace_size(shape, dmap, opts, int(chunks))
    ws = _host_workspace(nws, device) if nws > 0 else None
    st = selective_scan_fwd_host_raw(shape, _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C),
                                     _ptr(D), _ptr(z), _ptr(delta_bias), softplus, dmap, _ptr(out),
                                     _ptr(last_state), _ptr(ws), nws, int(chunks),
                                     _stream_handle(stream), opts)
    if st != SS_OK:
        raise ScanError(st, "selective_scan_fwd_host")
    return (out, last_state) if return_last_state else out


_host_ws = {}


def _host_workspace(nbytes, device):
    """The device workspace of the host-buffer call: one allocation per device, grown as needed.
    Calls on one device are serialised on the library's streams, so they can share it as long
    as the current stream orders a new allocation after the previous calls."""
    import torch
    buf = _host_ws.get(device.index)
    if buf is None or buf.numel() < nbytes:
        if buf is not None:
            torch.cuda.current_stream(device).synchronize()
        buf = torch.empty(nbytes, dtype=torch.uint8, device=device)
        _host_ws[device.index] = buf
    return buf
