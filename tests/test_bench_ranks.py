"""Host-side logic of bench.py: the multi-rank reduction (max of device time,
sum of bytes) on two gloo ranks, and the clock-sample summary."""
from __future__ import annotations

import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r: device time 10 + r ms, kernel time 5 + 2r, e2e 20 - r; bytes 1000 (r + 1)
        out = bench.combine_ranks(dist, torch.device("cpu"), 10.0 + rank, 5.0 + 2 * rank, 20.0 - rank,
                                  1000 * (rank + 1), 7 * (rank + 1))
        q.put((rank, out))
    finally:
        dist.destroy_process_group()


def test_combine_ranks_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in (0, 1):
        ms, kern, e2e, b, eb = res[r]
        assert ms == 11.0 and kern == 7.0 and e2e == 20.0  # max over ranks
        assert b == 3000.0 and eb == 21.0                 # sum over ranks


def test_summarize_clocks_keeps_only_the_timed_window():
    import datetime
    base = datetime.datetime(2026, 1, 2, 3, 4, 5)

    def row(dt_s, clk, slowdown="Not Active"):
        ts = (base + datetime.timedelta(seconds=dt_s)).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
        return [ts, "0", str(clk), "1965", "700.0", "0x0", slowdown, "Not Active", "Not Active", "Active"]

    rows = [row(0.0, 900), row(1.0, 1965), row(1.5, 1965), row(2.0, 1800, "Active"), row(5.0, 600)]
    t0 = (base + datetime.timedelta(seconds=0.9)).timestamp()
    t1 = (base + datetime.timedelta(seconds=2.1)).timestamp()
    s = bench.summarize_clocks(rows, (t0, t1))
    assert s["samples"] == 3
    assert s["sm_mhz"] == 1965.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["hw_slowdown", "sw_power_cap"]
    assert bench.summarize_clocks(rows, None)["samples"] == 5


def test_launch_count_per_path():
    import synth
    assert bench.launches_per_step(synth.workload(5)) == 6   # fp8 MLA: + query split
    assert bench.launches_per_step(synth.workload(4)) == 5
    assert bench.launches_per_step(synth.workload(3)) == 5
