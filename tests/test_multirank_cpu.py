"""Multi-rank host logic of bench.py on CPU (gloo, world size 2).

Every rank scans its own copy of the workload (independent problems; no collective on the data
path).  The only cross-rank steps are the timing reductions: the step time is the max over
ranks and the throughput is summed over ranks.
"""

import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist

    import bench
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=30))
    try:
        r, w, lr = bench.dist_env()
        step_ms = 1.0 + rank            # rank 1 is slower
        mx = bench.max_over_ranks(step_ms, world)
        total = bench.sum_over_ranks(100.0 * (rank + 1), world)
        q.put((r, w, lr, mx, total))
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_reductions():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[:3] for r in res] == [(0, 2, 0), (1, 2, 1)]
    for r in res:
        assert r[3] == pytest.approx(2.0)      # max over ranks
        assert r[4] == pytest.approx(300.0)    # summed throughput


def test_reference_arm_other_ranks_exit_without_work(monkeypatch, capsys):
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    assert bench.main(["--impl", "reference", "--workload", "tiny", "--steps", "1"]) == 0
    assert capsys.readouterr().out == ""


def test_reference_arm_line_on_cpu(monkeypatch, capsys):
    import json

    import bench
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    assert bench.main(["--impl", "reference", "--workload", "tiny", "--steps", "2",
                       "--warmup", "3"]) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "GB/s" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"


# ----------------------------------------------------------------------------- partitioned workload

def test_slice_bounds_cover_every_unit_once():
    from selective_state_space_13_b200 import shard
    for n, world, align in ((8, 2, 1), (8, 3, 1), (5120, 8, 64), (1536, 3, 64), (100, 8, 64),
                            (3, 8, 1), (0, 2, 1)):
        spans = [shard.slice_bounds(n, world, r, align) for r in range(world)]
        covered = []
        for lo, hi in spans:
            assert 0 <= lo <= hi <= n
            assert lo % align == 0 or lo == n
            covered.extend(range(lo, hi))
        assert covered == list(range(n)), (n, world, align, spans)
    with pytest.raises(ValueError):
        shard.slice_bounds(10, 2, 2)


def test_shard_plans_of_the_workloads():
    # the bench's split of each workload over 2, 4 and 8 ranks: by batch rows when there are
    # enough, else by 64-channel tiles; a split that leaves a rank idle is refused for every rank
    from selective_state_space_13_b200 import shard, workloads as wl
    for name in ("m130", "long", "vim", "ss2d", "cromb"):
        w = wl.WORKLOADS[name]
        for world in (2, 4, 8):
            axis = shard.shard_axis(w, world)
            n = w.batch if axis == "batch" else w.dim
            try:
                parts = [shard.plan(w, world, r) for r in range(world)]
            except ValueError:
                # only a channel split can leave a rank idle (rows are split only when there
                # are at least as many as ranks)
                assert axis == "channels"
                continue
            assert sum(p[2] - p[1] for p in parts) == n
            assert all(p[0] == axis and p[2] > p[1] for p in parts)
    # long (one batch row) over 8 ranks: 640 channels each
    parts = [shard.plan(wl.WORKLOADS["long"], 8, r) for r in range(8)]
    assert {p[3].dim for p in parts} == {640}
    # 192 channels cannot feed 8 ranks with whole 64-channel tiles
    with pytest.raises(ValueError):
        shard.plan(wl.variant("ss2d", batch=1), 8, 0)


def _shard_worker(rank, world, port, q, axis):
    import datetime

    import numpy as np
    import torch
    import torch.distributed as dist

    import oracle
    from selective_state_space_13_b200 import shard, workloads as wl
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        # a small workload with several directions, a gate, int8-free bf16 inputs
        base = wl.variant("vim", name="shard_case", batch=3, seqlen=40, dim=200, seed=77)
        inp = wl.make_inputs(base)
        ax, lo, hi, sub = shard.shard_workload(base, world, rank, axis)
        part = shard.shard_inputs(inp, ax, lo, hi)
        assert part["workload"] == sub
        # the host stand-in for the kernel call: the oracle on the slice
        f = wl.inputs_f64(part)
        out, last = oracle.selective_scan(f["u"], f["delta"], f["A"], f["B"], f["C"],
                                          Dskip=f["Dskip"], z=f["z"], delta_bias=f["delta_bias"],
                                          softplus=sub.softplus, dirs=sub.dirs)
        # gather the slices (test only: the benchmark's ranks exchange nothing)
        got = [None] * world
        dist.all_gather_object(got, (ax, out, last))
        if rank == 0:
            outs = [g[1] for g in got]
            lasts = [g[2] for g in got]
            whole_out, whole_last = shard.reassemble(ax, outs, lasts)
            f = wl.inputs_f64(inp)
            ref_out, ref_last = oracle.selective_scan(f["u"], f["delta"], f["A"], f["B"], f["C"],
                                                      Dskip=f["Dskip"], z=f["z"],
                                                      delta_bias=f["delta_bias"],
                                                      softplus=base.softplus, dirs=base.dirs)
            q.put((ax, bool(np.array_equal(whole_out, ref_out)),
                   bool(np.array_equal(whole_last, ref_last))))
        del torch
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("axis", ["batch", "channels"])
def test_two_rank_partition_reassembles_exactly(axis):
    # two gloo ranks each scan their slice of one workload (batch rows or channels); the slices,
    # put back together, equal the unsplit scan bit for bit
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_worker, args=(r, 2, port, q, axis)) for r in range(2)]
    for p in procs:
        p.start()
    ax, ok_out, ok_last = q.get(timeout=180)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert ax == axis and ok_out and ok_last
