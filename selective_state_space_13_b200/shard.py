"""Partition of one workload across ranks (one process per GPU): the slice arithmetic.

The scans of different batch rows and of different channels are independent (the state of a
channel never meets another channel's, and B and C are read-only), so one workload splits into
per-rank problems with no exchange at all: rank r scans a contiguous slice of the batch rows, or,
for a workload with fewer batch rows than ranks, a slice of the channels (with all batch rows and
the whole B and C).  Putting the output slices back together gives the unsplit result exactly.

This module holds only that bookkeeping (which rows or channels a rank owns, how to cut the inputs
and how to reassemble the outputs); every scan is the library's.
"""

from __future__ import annotations

from dataclasses import replace

import numpy as np

from . import workloads as wl

# channel slices are whole 64-channel tiles of the kernels (which also keeps every row pitch a
# multiple of 16 bytes)
CHANNEL_ALIGN = 64


def slice_bounds(n: int, world: int, rank: int, align: int = 1):
    """The contiguous share [lo, hi) of n units that `rank` of `world` owns: equal shares rounded
    up to multiples of `align`, the last ranks taking what is left (possibly nothing)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank %d of world %d" % (rank, world))
    per = -(-n // world)
    per = -(-per // align) * align
    lo = min(n, rank * per)
    hi = min(n, lo + per)
    return lo, hi


def shard_axis(w: wl.Workload, world: int) -> str:
    """'batch' when every rank can own whole batch rows, else 'channels'."""
    return "batch" if w.batch >= world else "channels"


def shard_workload(w: wl.Workload, world: int, rank: int, axis: str | None = None):
    """(axis, lo, hi, sub-workload) of rank `rank`: the slice's shape as a workload."""
    axis = axis or shard_axis(w, world)
    if axis == "batch":
        lo, hi = slice_bounds(w.batch, world, rank)
        return axis, lo, hi, replace(w, batch=hi - lo)
    if axis == "channels":
        lo, hi = slice_bounds(w.dim, world, rank, CHANNEL_ALIGN)
        return axis, lo, hi, replace(w, dim=hi - lo)
    raise ValueError("axis must be 'batch' or 'channels'")


def plan(w: wl.Workload, world: int, rank: int, axis: str | None = None):
    """shard_workload for `rank`, after checking every rank's slice: a split that would leave a
    rank without work raises ValueError on every rank alike (so all stop before any collective)."""
    axis = axis or shard_axis(w, world)
    empty = [r for r in range(world)
             if (lambda s: s[2] <= s[1])(shard_workload(w, world, r, axis))]
    if empty:
        raise ValueError("splitting by %s leaves rank(s) %s of %d without work" % (axis, empty, world))
    return shard_workload(w, world, rank, axis)


def shard_inputs(inp: dict, axis: str, lo: int, hi: int) -> dict:
    """The inputs of one slice (arrays as make_inputs returns them), contiguous."""
    w = inp["workload"]
    c = np.ascontiguousarray
    out = dict(inp)
    if axis == "batch":
        out["workload"] = replace(w, batch=hi - lo)
        out["u"] = c(inp["u"][:, lo:hi] if w.u_per_dir else inp["u"][lo:hi])
        out["z"] = None if inp["z"] is None else c(inp["z"][lo:hi])
        for k in ("delta", "B", "C"):
            out[k] = c(inp[k][:, lo:hi])
        return out
    out["workload"] = replace(w, dim=hi - lo)
    for k in ("u", "z", "delta"):
        out[k] = None if inp[k] is None else c(inp[k][..., lo:hi])
    out["A"] = c(inp["A"][..., lo:hi, :])
    out["Dskip"] = c(inp["Dskip"][..., lo:hi])
    out["delta_bias"] = None if inp["delta_bias"] is None else c(inp["delta_bias"][..., lo:hi])
    if inp.get("conv_weight") is not None:
        out["conv_weight"] = c(inp["conv_weight"][:, lo:hi])
        out["conv_bias"] = c(inp["conv_bias"][:, lo:hi])
    if inp.get("delta_scale") is not None:
        out["delta_scale"] = c(inp["delta_scale"][lo:hi])
    return out


def reassemble(axis: str, outs, lasts):
    """The whole workload's out [batch, L, D] and last_state [K, batch, D, N] from the ranks'
    slices, in rank order."""
    if axis == "batch":
        return np.concatenate(outs, axis=0), np.concatenate(lasts, axis=1)
    return np.concatenate(outs, axis=-1), np.concatenate(lasts, axis=2)
