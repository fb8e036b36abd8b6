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
