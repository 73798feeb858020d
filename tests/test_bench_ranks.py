"""Host-side logic of bench.py: the multi-rank reduction (max of device time,
sum of bytes) on two gloo ranks, the clock-sample summary, which source changes
void a stored DRAM-traffic capture, and the reference arm's JSON line (the oracle
on host cores)."""
from __future__ import annotations

import os
import socket
import sys

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
        out = bench.combine_ranks(dist, torch.device("cpu"), [10.0 + rank, 5.0 + 2 * rank, 20.0 - rank],
                                  [1000 * (rank + 1), 7 * (rank + 1)])
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
        (ms, kern, e2e), (b, eb) = res[r]
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
    # shard map, append, plan, decode, merge; fp8 MLA adds the query split
    assert bench.launches_per_step(synth.workload(5)) == 6
    assert bench.launches_per_step(synth.workload(4)) == 5
    assert bench.launches_per_step(synth.workload(3)) == 5


def test_band_latency_summary():
    """Requests fall in the bands by length; percentiles and the band's rate come from
    the per-request completion times."""
    import numpy as np
    L = np.array([1_000, 31_999, 32_000, 100_000, 250_000, 250_001])
    fin = np.array([0.5, 1.0, 1.5, 2.0, 4.0, 3.0])
    d = bench.band_latency(L, fin, 4.2, 580)
    assert set(d) == {"<32k", "32-64k", "64-128k", "200k+", "batch_decode_ms"}
    assert d["<32k"]["requests"] == 2 and d["<32k"]["tokens"] == 32_999
    assert d["<32k"]["done_ms_max"] == 1.0 and d["<32k"]["done_ms_p50"] == 0.75
    assert d["200k+"]["done_ms_max"] == 4.0
    assert d["32-64k"]["kv_gbs_by_band_done"] == round(32_000 * 580 / 1.5e-3 / 1e9, 1)
    assert d["batch_decode_ms"] == 4.2


def test_traffic_digest_is_per_kernel(tmp_path, monkeypatch):
    """Editing one decode kernel's file voids that kernel's counters only; a shared
    header voids them all."""
    import shutil
    src = tmp_path / "csrc"
    shutil.copytree(bench.KERNEL_SOURCES, src)
    monkeypatch.setattr(bench, "KERNEL_SOURCES", str(src))
    kernels = ["gqa_mma_kernel<128,4>", "mla_bf16_kernel<64>", "mla_fp8_kernel<64>"]
    before = {k: bench.kernel_sources_digest(k) for k in kernels}
    with open(src / "decode_mla_fp8.cu", "a") as f:
        f.write("\n// edited\n")
    after = {k: bench.kernel_sources_digest(k) for k in kernels}
    assert after["mla_fp8_kernel<64>"] != before["mla_fp8_kernel<64>"]
    assert after["gqa_mma_kernel<128,4>"] == before["gqa_mma_kernel<128,4>"]
    assert after["mla_bf16_kernel<64>"] == before["mla_bf16_kernel<64>"]
    with open(src / "common.cuh", "a") as f:
        f.write("\n// edited\n")
    shared = {k: bench.kernel_sources_digest(k) for k in kernels}
    assert all(shared[k] != after[k] for k in kernels)


def test_committed_traffic_file_is_well_formed():
    """Each capture names a known decode kernel, carries its sources' digest, and reads
    no fewer bytes than the launch's KV cache."""
    import json
    d = json.load(open(bench.TRAFFIC_FILE))
    for key, e in d["workloads"].items():
        assert e["kernel"].split("<")[0] in bench.KERNEL_FILES, key
        assert len(e["sources_sha256"]) == 64, key
        assert abs(e["dram_read"] + e["dram_write"] - e["dram_bytes_per_launch"]) < 1e3, key
        assert 0.99 < e["dram_bytes_per_launch"] / e["algorithmic_kv_bytes"] < 1.3, key


def _bench_reference(env_extra):
    import json
    import subprocess
    env = dict(os.environ, **env_extra)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "1",
                        "--steps", "2", "--warmup", "1"], capture_output=True, text=True, env=env, timeout=600,
                       cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    return [json.loads(l) for l in lines]


def test_reference_arm_json_line():
    """The reference arm (the oracle on host cores) prints one JSON line with the bench contract's keys."""
    (d,) = _bench_reference({"WORLD_SIZE": "1", "RANK": "0"})
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == "GB/s"
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert (d["n_gpus"], d["steps"], d["warmup"]) == (1, 2, 1)
    assert d["higher_is_better"] is True and d["scaling"] == "weak" and d["vs_baseline"] is None
    assert d["dtype"] == "f64" and "synthetic" in d["data"] and "workload" in d["config"]
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"] and cb["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_are_silent():
    """Under torchrun only rank 0 runs the oracle and prints; the other ranks exit 0 without output."""
    assert _bench_reference({"WORLD_SIZE": "2", "RANK": "1"}) == []
