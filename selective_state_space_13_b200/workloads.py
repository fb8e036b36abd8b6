"""Seeded synthetic inputs for the selective scan: the five workloads and smaller variants.

This module is shared by the tests, the benchmark and the smoke check.  It holds no step of the
scan itself: it only draws random numbers, rounds them to the storage type, and builds the
parameter tensors the workloads prescribe.  Both the CUDA path and the CPU oracle receive the
arrays it returns (the oracle as their exact float64 upcast).

Recipe (identical for every workload, seed = 20260 + workload index):
  * u, z, delta_raw[k], B[k], C[k] ~ N(0, 1), drawn in that order, each tensor from its own
    child stream of ``SeedSequence([seed, tensor_id, k])`` and, inside a tensor, one further
    child stream per block of rows, so that the values do not depend on the thread count;
  * values are drawn in float32 and rounded to bfloat16 with round-to-nearest-even when the
    workload stores bfloat16;
  * A[d, n] = -(n + 1) (fp32);
  * Dskip = 1 (fp32), except the tiny workload where Dskip ~ N(0, 1);
  * delta_bias: Delta0 ~ exp(U[ln 1e-3, ln 0.1]) per channel, bias = softplus^-1(Delta0) =
    Delta0 + log(-expm1(-Delta0)); the tiny workload uses bias = 0;
  * with parameters per direction (`params_per_dir`): A[k, d, n] = -(n + 1) * (1 + k/4),
    Dskip[k] = 1 + k/4 (or N(0, 1) per direction), delta_bias drawn per direction as above, so
    that every direction's parameters differ;
  * with int8 Delta (`delta_int8`): delta_raw is drawn as above in float32, then quantised
    symmetrically per channel: scale[d] = max |delta_raw[:, :, :, d]| / 127 over directions,
    batch rows and steps, q = round-half-even(delta_raw / scale[d]) (in [-127, 127]); the
    arrays are the int8 codes and the float32 scales;
  * with a causal convolution of `conv` taps before the scan (no named workload has one; the
    variants that test it do): taps and bias per direction and channel ~ U(-1/sqrt(conv),
    1/sqrt(conv)) in fp32, the usual initial scale of a depthwise convolution of that width
    (the pages give no weights).

The pages name no dataset for this path; the shapes stand for a Mamba-130M layer (8 x 2048 x
1536, N = 16), a 131072-token sequence, a Vim-S block (64 images of 14 x 14 patches + a class
token = 197 tokens, D = 768, two directions), a VMamba stage-1 map (56 x 56, D = 192, four
cross-scan orders) and a cross-modal (CroMB) scan of two modalities over a 120 x 160 feature map
(a 480 x 640 RGB-D frame at 1/4 resolution, D = 192): one input per modality (u[k] ~ N(0, 1),
``SeedSequence([seed, 0, k])``), where C[k] stands for the C computed from the other modality.
"""

from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field, replace

import numpy as np

DIR_FORWARD, DIR_REVERSE, DIR_COLUMN, DIR_COLUMN_REVERSE = 0, 1, 2, 3
F32, BF16 = "f32", "bf16"


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    seqlen: int
    dim: int
    dstate: int
    dtype: str                      # storage type of u, delta_raw, z, B, C and out
    dirs: tuple = (DIR_FORWARD,)
    H: int = 0                      # image height/width for column-order directions
    W: int = 0
    gate: bool = True               # z given (silu(z) gate) or not
    softplus: bool = True
    bias: str = "loguniform"        # "loguniform" or "zero"
    dskip: str = "one"              # "one" or "normal"
    seed: int = 20260
    conv: int = 0                   # taps of the causal convolution before the scan (0: none)
    u_per_dir: bool = False         # one input u[k] per direction ([K, batch, L, D])
    delta_int8: bool = False        # delta_raw as int8 codes with one fp32 scale per channel
    params_per_dir: bool = False    # A [K, D, N], Dskip and delta_bias [K, D]
    extra: dict = field(default_factory=dict, compare=False)

    @property
    def K(self) -> int:
        return len(self.dirs)

    @property
    def io_bytes(self) -> int:
        return 4 if self.dtype == F32 else 2

    def updates(self) -> int:
        """State updates of one pass: sum over directions of batch * L * D * N."""
        return self.K * self.batch * self.seqlen * self.dim * self.dstate

    def algorithmic_bytes(self, with_last_state: bool = True) -> int:
        """Bytes a pass must move at least once: u, z, delta_raw, B, C read; out written;
        A, Dskip, delta_bias read; last_state written."""
        e = self.io_bytes
        bld = self.batch * self.seqlen * self.dim
        bln = self.batch * self.seqlen * self.dstate
        nbytes = bld * e * ((self.K if self.u_per_dir else 1) + 1 + (1 if self.gate else 0))
        # u (per direction or shared), out, z
        nbytes += self.K * bld * (1 if self.delta_int8 else e)     # delta_raw per direction
        if self.delta_int8:
            nbytes += self.dim * 4                                 # its scales
        nbytes += 2 * self.K * bln * e                             # B, C per direction
        nbytes += (self.K if self.params_per_dir else 1) * (self.dim * self.dstate + 2 * self.dim) * 4
        # A, Dskip, delta_bias
        if with_last_state:
            nbytes += self.K * self.batch * self.dim * self.dstate * 4
        if self.conv:
            nbytes += self.K * self.dim * (self.conv + 1) * 4         # conv taps and bias
        return nbytes


WORKLOADS = {
    "tiny": Workload("tiny", 1, 64, 16, 4, F32, bias="zero", dskip="normal", seed=20260),
    "m130": Workload("m130", 8, 2048, 1536, 16, BF16, seed=20261),
    "long": Workload("long", 1, 131072, 5120, 16, BF16, seed=20262),
    "vim": Workload("vim", 64, 197, 768, 16, BF16, dirs=(DIR_FORWARD, DIR_REVERSE), seed=20263),
    "ss2d": Workload("ss2d", 32, 3136, 192, 16, BF16,
                     dirs=(DIR_FORWARD, DIR_COLUMN, DIR_REVERSE, DIR_COLUMN_REVERSE),
                     H=56, W=56, gate=False, seed=20264),
    "cromb": Workload("cromb", 8, 19200, 192, 16, BF16, dirs=(DIR_FORWARD, DIR_FORWARD),
                      gate=False, u_per_dir=True, seed=20265),
}

DESCRIPTIONS = {
    "tiny": "tiny S6 scan: batch 1, L 64, D 16, N 4, fp32",
    "m130": "Mamba-130M-layer scan: batch 8, L 2048, D 1536, N 16, bf16",
    "long": "long-sequence scan: batch 1, L 131072, D 5120, N 16, bf16",
    "vim": "Vim-S bidirectional scan: batch 64, M 197, D 768, N 16, bf16, 2 directions",
    "ss2d": "SS2D cross-scan: batch 32, 56x56 (L 3136), D 192, N 16, bf16, 4 directions, no gate",
    "cromb": "CroMB cross-modal scan: 2 modalities, batch 8, 120x160 (L 19200), D 192, N 16, bf16, "
             "outputs summed, no gate",
}


def variant(base: str, **kw) -> Workload:
    """A workload with the recipe of ``base`` and some fields changed (smaller parity cases)."""
    return replace(WORKLOADS[base], **kw)


# ----------------------------------------------------------------------------- bf16 helpers

def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16, round-to-nearest-even; returns the uint16 bit patterns."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (b >> np.uint32(16)) & np.uint32(1)
    r = (b + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    nan = np.isnan(x)
    out = r.astype(np.uint16)
    if nan.any():
        out[nan] = np.uint16(0x7FC0)
    return out


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def to_f64(arr: np.ndarray, dtype: str) -> np.ndarray:
    """Exact float64 value of a stored array (bf16 arrays are held as uint16 bit patterns)."""
    if dtype == BF16:
        return bf16_bits_to_f32(arr).astype(np.float64)
    return np.asarray(arr, dtype=np.float64)


# ----------------------------------------------------------------------------- generation

_ROWS_PER_BLOCK = 1 << 21  # elements per independent child stream


def _normal(shape, ss: np.random.SeedSequence, dtype: str, threads: int) -> np.ndarray:
    total = int(np.prod(shape))
    nblk = max(1, -(-total // _ROWS_PER_BLOCK))
    children = ss.spawn(nblk)
    out = np.empty(total, dtype=np.uint16 if dtype == BF16 else np.float32)

    def fill(i):
        lo = i * _ROWS_PER_BLOCK
        hi = min(total, lo + _ROWS_PER_BLOCK)
        g = np.random.Generator(np.random.PCG64(children[i]))
        v = g.standard_normal(hi - lo, dtype=np.float32)
        out[lo:hi] = f32_to_bf16_bits(v) if dtype == BF16 else v

    if nblk == 1 or threads <= 1:
        for i in range(nblk):
            fill(i)
    else:
        with ThreadPoolExecutor(min(threads, nblk)) as ex:
            list(ex.map(fill, range(nblk)))
    return out.reshape(shape)


def make_inputs(w: Workload | str, threads: int | None = None) -> dict:
    """Draw the seeded inputs of a workload.

    Returns a dict with numpy arrays
      u [batch, L, D] (or [K, batch, L, D] with one input per direction), z (None without a
      gate) [batch, L, D]; delta [K, batch, L, D]; B, C [K, batch, L, N]
      (uint16 bfloat16 bit patterns or float32), A [D, N], Dskip [D], delta_bias [D] or None
      (float32), plus the workload under key "workload".
    """
    if isinstance(w, str):
        w = WORKLOADS[w]
    if threads is None:
        threads = min(32, os.cpu_count() or 1)
    b, L, D, N, K = w.batch, w.seqlen, w.dim, w.dstate, w.K
    root = w.seed
    ss = lambda tid, k=0: np.random.SeedSequence([root, tid, k])  # noqa: E731
    if w.u_per_dir:
        u = np.stack([_normal((b, L, D), ss(0, k), w.dtype, threads) for k in range(K)])
    else:
        u = _normal((b, L, D), ss(0), w.dtype, threads)
    z = _normal((b, L, D), ss(1), w.dtype, threads) if w.gate else None
    ddtype = F32 if w.delta_int8 else w.dtype
    delta = np.stack([_normal((b, L, D), ss(2, k), ddtype, threads) for k in range(K)]) \
        if K > 1 else _normal((b, L, D), ss(2, 0), ddtype, threads)[None]
    delta_scale = None
    if w.delta_int8:
        delta, delta_scale = quantize_int8_per_channel(delta)
    B = np.stack([_normal((b, L, N), ss(3, k), w.dtype, threads) for k in range(K)])
    C = np.stack([_normal((b, L, N), ss(4, k), w.dtype, threads) for k in range(K)])
    g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([root, 5])))
    P = K if w.params_per_dir else 1               # parameter sets
    if w.dskip == "normal":
        Dskip = g.standard_normal((P, D)).astype(np.float32)
    else:
        Dskip = np.stack([np.full(D, 1.0 + k / 4.0, dtype=np.float32) for k in range(P)])
    if w.bias == "zero":
        bias = np.zeros((P, D), dtype=np.float32)
    else:
        d0 = np.exp(g.uniform(math.log(1e-3), math.log(0.1), size=(P, D)))
        bias = (d0 + np.log(-np.expm1(-d0))).astype(np.float32)
    A = np.stack([np.tile(-(np.arange(N, dtype=np.float32) + 1.0) * np.float32(1.0 + k / 4.0), (D, 1))
                  for k in range(P)])
    if not w.params_per_dir:
        A, Dskip, bias = A[0], Dskip[0], bias[0]
    conv_weight = conv_bias = None
    if w.conv:
        gc = np.random.Generator(np.random.PCG64(np.random.SeedSequence([root, 6])))
        lim = 1.0 / math.sqrt(w.conv)
        conv_weight = gc.uniform(-lim, lim, size=(K, D, w.conv)).astype(np.float32)
        conv_bias = gc.uniform(-lim, lim, size=(K, D)).astype(np.float32)
    return dict(workload=w, u=u, z=z, delta=delta, B=B, C=C, A=A, Dskip=Dskip, delta_bias=bias,
                conv_weight=conv_weight, conv_bias=conv_bias, delta_scale=delta_scale)


def quantize_int8_per_channel(x: np.ndarray):
    """Symmetric int8 codes of a float32 [..., D] array with one scale per channel (the last
    axis): scale = max |x| / 127 over all other axes, codes = round-half-even(x / scale)."""
    D = x.shape[-1]
    amax = np.abs(x.reshape(-1, D)).max(axis=0).astype(np.float32)
    scale = np.where(amax > 0, amax / np.float32(127.0), np.float32(1.0)).astype(np.float32)
    q = np.rint(x / scale).clip(-127, 127).astype(np.int8)
    return q, scale


def inputs_f64(inp: dict, channels=None, batches=None) -> dict:
    """Float64 views for the oracle, optionally restricted to some channels and batch rows."""
    w = inp["workload"]
    bsel = slice(None) if batches is None else np.asarray(batches)
    dsel = slice(None) if channels is None else np.asarray(channels)

    def big(x, lead):  # [..., batch, L, D]
        if x is None:
            return None
        v = x[:, bsel] if lead else x[bsel]
        v = v[..., dsel]
        if v.dtype == np.int8:
            return v.astype(np.float64)
        return to_f64(v, w.dtype)

    def bc(x):
        return to_f64(x[:, bsel], w.dtype)

    return dict(u=big(inp["u"], w.u_per_dir), z=big(inp["z"], False), delta=big(inp["delta"], True),
                B=bc(inp["B"]), C=bc(inp["C"]),
                A=np.asarray(inp["A"][..., dsel, :], dtype=np.float64),
                Dskip=np.asarray(inp["Dskip"][..., dsel], dtype=np.float64),
                delta_bias=None if inp["delta_bias"] is None else
                np.asarray(inp["delta_bias"][..., dsel], dtype=np.float64),
                conv_weight=None if inp.get("conv_weight") is None else
                np.asarray(inp["conv_weight"][:, dsel], dtype=np.float64),
                conv_bias=None if inp.get("conv_bias") is None else
                np.asarray(inp["conv_bias"][:, dsel], dtype=np.float64),
                delta_scale=None if inp.get("delta_scale") is None else
                np.asarray(inp["delta_scale"][dsel], dtype=np.float64),
                softplus=w.softplus, dirs=w.dirs, H=w.H, W=w.W)


def to_torch(arr, dtype: str, device):
    """A stored array as a torch tensor on `device` (bf16 bit patterns become bfloat16)."""
    import torch
    if arr is None:
        return None
    if dtype == BF16 and arr.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(arr).view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(np.ascontiguousarray(arr)).to(device)


def to_device(inp: dict, device) -> dict:
    """The arrays of ``make_inputs`` as torch tensors on `device`, keyed as the binding names
    its arguments (u, z, delta, B, C, A, D, delta_bias, conv_weight, conv_bias)."""
    w = inp["workload"]
    return dict(u=to_torch(inp["u"], w.dtype, device), z=to_torch(inp["z"], w.dtype, device),
                delta=to_torch(inp["delta"], w.dtype, device), B=to_torch(inp["B"], w.dtype, device),
                C=to_torch(inp["C"], w.dtype, device), A=to_torch(inp["A"], F32, device),
                D=to_torch(inp["Dskip"], F32, device),
                delta_bias=to_torch(inp["delta_bias"], F32, device),
                conv_weight=to_torch(inp.get("conv_weight"), F32, device),
                conv_bias=to_torch(inp.get("conv_bias"), F32, device),
                delta_scale=to_torch(inp.get("delta_scale"), F32, device))
