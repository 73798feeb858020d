#!/usr/bin/env python
"""Decode-attention benchmark for libdcp (sequence-sharded paged KV cache).

One step = one pass of the whole hot path over the batch, for one new token
per request:
  dcp_shard_map (owner/slot of position L_b)  ->  dcp_kv_append (write the new
  token into its owner's page)  ->  dcp_decode_merged (every shard's partial
  attention over positions [0, L_b + 1), then the LSE merge, in one call).
Lengths grow by one token per step, as in decoding.

Metric: KV GB/s = (sum_b attended tokens x KV bytes per token) / step time,
plus decode steps/s, and the fraction of the measured HBM copy bandwidth.
Inputs are synthetic (seeded generator) with the shapes of the named
workload; the KV cache (>= several GB) is far larger than the 126 MB L2, so
no L2 flush is needed between steps.

The JSON line's headline is one workload (--config, default the
high-concurrency fp8 MLA one); at N = 1 the two other large workloads (GQA
Qwen3-shaped, MLA Kimi-shaped bf16) are measured the same way under
"per_config".  Each workload also reports:
  - "bands": per-request completion time inside the full batch, by request
    length band (<32k, 32-64k, 64-128k, 128-200k, 200k+), from the device
    timestamps dcp_decode_merged records per request;
  - "e2e": the same step through the C ABI with host buffers, the inputs copied
    in and the output copied out every step on copy streams overlapped with
    the previous / next step's compute.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config 5]
                  [--n-shards 8] [--interleave 1] [--impl ours|reference]

Multi-GPU (torchrun, one rank per GPU): each rank runs its own independent
batch (replicas of the workload, weak scaling); there is no data-path
collective.  Timing is the max over ranks of the device time.  With
--dcp-across-gpus the ranks instead form one DCP group: each holds the shard
of the positions it owns (N = number of GPUs), decodes it, and the partials
are combined by an all-gather of the LSEs and a reduce-scatter over query
heads (NCCL); the group decodes one batch (strong scaling).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "DCP decode-attn KV GB/s (% of B200 HBM peak) and decode steps/s per config"
HEADLINE_CONFIG = 5


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", type=int, default=HEADLINE_CONFIG)
    ap.add_argument("--per-config", default="3,4",
                    help="other workloads measured the same way at N = 1 ('' for none)")
    ap.add_argument("--n-shards", type=int, default=None)
    ap.add_argument("--interleave", type=int, default=None)
    ap.add_argument("--batch-limit", type=int, default=None,
                    help="keep only the first B requests of the workload (small profiling cases)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-bands", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=25.0, help="target CPU work of the oracle sample")
    ap.add_argument("--dcp-across-gpus", action="store_true",
                    help="one shard per rank (N = number of GPUs): rank-local caches and the all-gather / "
                         "reduce-scatter exchange over NCCL, one batch for the whole group (strong scaling)")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def get_workload(args, cfg=None):
    cfg = args.config if cfg is None else cfg
    own = cfg == args.config
    w = synth.workload(cfg, n_shards=args.n_shards if own else None, interleave=args.interleave if own else None)
    if args.batch_limit and own:
        w.B = min(w.B, args.batch_limit)
        w.lengths = w.lengths[:w.B]
    return w


def workload_config(w, cfg):
    return {"workload": f"config{cfg}: {w.name}", "kind": w.kind, "kv_dtype": w.dtype,
            "batch": w.B, "q_heads": w.hq, "kv_heads": w.hkv, "dk": w.dk, "dv": w.dv, "page_size": w.page_size,
            "n_shards": w.n_shards, "interleave": w.interleave, "total_tokens": int(np.sum(w.lengths)),
            "median_len": int(np.median(w.lengths)), "max_len": int(np.max(w.lengths)),
            "l2": "inputs larger than L2 (KV cache >> 126 MB); no flush"}


# ----------------------------------------------------------------------------
# clocks sampling during the timed region
# ----------------------------------------------------------------------------

class Clocks:
    """nvidia-smi sampling every 10 ms, started before the warm-up so that it is
    running when the timed region begins; only samples whose timestamp falls
    inside the timed region (host wall clock around it) are kept."""
    Q = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.p = None
        self.window = None

    def start(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.Q}",
                                       "--format=csv,noheader,nounits", "-lms", "10"], stdout=self.f,
                                      stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.p = None

    def mark(self, t0: float, t1: float):
        """Host wall-clock bounds of the timed region."""
        self.window = (t0, t1)

    def stop(self):
        if self.p is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "samples": 0, "reasons": ["nvidia-smi unavailable"]}
        self.p.terminate()
        try:
            self.p.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.p.kill()
        self.f.flush()
        rows = [r.split(",") for r in open(self.f.name).read().strip().splitlines() if r.strip()]
        os.unlink(self.f.name)
        return summarize_clocks(rows, self.window)


def summarize_clocks(rows, window):
    """rows: nvidia-smi CSV fields (timestamp first); window: (t0, t1) epoch seconds or None."""
    sm, mx, reasons = [], None, set()
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    for r in rows:
        r = [x.strip() for x in r]
        if len(r) < 10:
            continue
        try:
            ts = datetime.datetime.strptime(r[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
            clk, cmax = float(r[2]), float(r[3])
        except ValueError:
            continue
        if window is not None and not (window[0] <= ts <= window[1]):
            continue
        sm.append(clk)
        mx = cmax
        for nm, v in zip(names, r[6:10]):
            if v.lower() == "active":
                reasons.add(nm)
    return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "samples": len(sm),
            "reasons": sorted(reasons)}


# ----------------------------------------------------------------------------
# DRAM traffic of the decode launch, from an ncu capture (profiles/)
# ----------------------------------------------------------------------------

TRAFFIC_FILE = os.path.join(ROOT, "profiles", "decode_dram_traffic.json")
KERNEL_SOURCES = os.path.join(ROOT, "sequence_sharded_paged_b200", "csrc")


# the decode kernel of each capture and the source file it is built from
KERNEL_FILES = {"gqa_mma_kernel": "decode_gqa_mma.cu", "mla_bf16_kernel": "decode_mla_bf16.cu",
                "mla_fp8_kernel": "decode_mla_fp8.cu", "gqa_simt_kernel": "decode_simt.cu",
                "mla_simt_kernel": "decode_simt.cu"}


def kernel_sources_digest(kernel: str) -> str:
    """sha256 over the sources that one decode kernel is built from: the planner, the
    tensor-map code, the shared headers and the kernel's own file. A change to any of
    them voids the counters captured for that kernel; a change to another decode
    kernel does not."""
    own = KERNEL_FILES[kernel.split("<")[0]]
    h = hashlib.sha256()
    for name in sorted(os.listdir(KERNEL_SOURCES)):
        if name in ("plan.cu", "tma.cu", own) or name.endswith((".cuh", ".h")):
            h.update(name.encode())
            h.update(open(os.path.join(KERNEL_SOURCES, name), "rb").read())
    return h.hexdigest()


def measured_traffic(config_key: str):
    """dram bytes read + written per decode launch, or None when no capture of
    the current sources of that workload's decode kernel exists."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    e = json.load(open(TRAFFIC_FILE)).get("workloads", {}).get(config_key)
    if e is None or e.get("sources_sha256") != kernel_sources_digest(e["kernel"]):
        return None
    return float(e["dram_bytes_per_launch"])


def traffic_key(cfg, w) -> str:
    return f"config{cfg} B{w.B} N{w.n_shards} I{w.interleave}"


def launches_per_step(w) -> int:
    """Kernels one step launches: shard map, append, plan, [query split], decode, merge."""
    fp8_tc = w.kind == "mla" and w.dtype == "fp8" and w.hq in (16, 32, 64) and w.page_size == 64
    return 6 if fp8_tc else 5


def combine_ranks(dist, device, times, sums):
    """Max over ranks of the device times, sum over ranks of the byte counts."""
    import torch
    t = torch.tensor([float(x) for x in times], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    tb = torch.tensor([float(x) for x in sums], dtype=torch.float64, device=device)
    dist.all_reduce(tb, op=dist.ReduceOp.SUM)
    return t.tolist(), tb.tolist()


# ----------------------------------------------------------------------------
# our implementation
# ----------------------------------------------------------------------------

BANDS = [(0, 32_000, "<32k"), (32_000, 64_000, "32-64k"), (64_000, 128_000, "64-128k"),
         (128_000, 200_000, "128-200k"), (200_000, 1 << 31, "200k+")]


def band_latency(lengths, finish_ms, decode_ms, kv_bytes_per_token):
    """Per-request completion times inside one full-batch decode, by length band.
    finish_ms[b]: request b's output stored, ms after the decode's first kernel
    started (median over repeated launches)."""
    L = np.asarray(lengths)
    out = {}
    for lo, hi, name in BANDS:
        sel = (L >= lo) & (L < hi)
        if not sel.any():
            continue
        f = np.asarray(finish_ms)[sel]
        tok = int(L[sel].sum())
        out[name] = {"requests": int(sel.sum()), "tokens": tok,
                     "done_ms_p50": round(float(np.percentile(f, 50)), 4),
                     "done_ms_p99": round(float(np.percentile(f, 99)), 4),
                     "done_ms_max": round(float(f.max()), 4),
                     "kv_gbs_by_band_done": round(tok * kv_bytes_per_token / (float(f.max()) * 1e-3) / 1e9, 1)}
    out["batch_decode_ms"] = round(decode_ms, 4)
    return out


def measure(args, cfg, rank, world, local_rank, headline):
    """Time the decode step of workload `cfg` (see the module docstring); returns the
    result dict (value, ms_per_step, roofline, clocks, e2e, bands, ...) and the workload."""
    import torch
    import torch.distributed as dist

    import sequence_sharded_paged_b200 as dcp
    import synth.device as sdev
    from sequence_sharded_paged_b200 import workload as wl

    dcp.lib()  # fail loudly if libdcp.so is missing
    dev = torch.device("cuda", local_rank)
    w = get_workload(args, cfg)
    w.seed_val += 100 * rank  # each rank decodes its own independent batch
    E = 0 if args.no_e2e else args.steps
    n_total = args.warmup + args.steps + E
    growth = n_total + 1
    counts = wl.gpu_shard_counts(np.asarray(w.lengths) + growth, w.n_shards, w.interleave)
    t0 = time.time()
    dw = wl.build(w, counts)
    fill_s = time.time() - t0
    B, N = w.B, w.n_shards
    L0 = torch.as_tensor(np.asarray(w.lengths, np.int32), device=dev)
    ws = torch.empty(dcp.dcp_decode_workspace_size_ex(dw.desc, B, 1, dcp.DCP_DECODE_MERGED), dtype=torch.uint8, device=dev)

    # per-step inputs, resident in HBM before the timed region
    qs = [sdev.q(w.seed_val, B, w.hq, w.dk, step=s + 1) for s in range(n_total)]
    req = torch.arange(B, dtype=torch.int32, device=dev)
    pos_s = [(L0 + s).contiguous() for s in range(n_total)]
    lens_s = [(L0 + s + 1).contiguous() for s in range(n_total)]
    if w.kind == "gqa":
        new_rows = [sdev.gqa_rows(w.seed_val, req, pos_s[s], w.hkv, w.dk) for s in range(n_total)]
    else:
        new_rows = [(sdev.latent_rows(w.seed_val, req, pos_s[s]), None) for s in range(n_total)]
    rank_o = torch.empty(B, dtype=torch.int32, device=dev)
    local_o = torch.empty(B, dtype=torch.int32, device=dev)
    slot_o = torch.empty(B, dtype=torch.int64, device=dev)
    out = torch.empty((B, w.hq, w.dv), dtype=torch.float32, device=dev)
    lse_out = torch.empty((B, w.hq), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def step(s, ev=None, pos=None, lens=None, q=None, k=None, v=None, o=out, lo=lse_out):
        pos = pos_s[s] if pos is None else pos
        if k is None:
            k, v = new_rows[s]
        dcp.dcp_shard_map(dw.desc, pos, None, rank_o, local_o, slot_o)
        dcp.dcp_kv_append(dw.desc, None, pos, k, v)
        if ev is not None:
            ev[0].record(torch.cuda.current_stream())
        dcp.dcp_decode_merged(dw.desc, qs[s] if q is None else q, lens_s[s] if lens is None else lens, o, lo, ws)
        if ev is not None:
            ev[1].record(torch.cuda.current_stream())

    clocks = Clocks(local_rank)
    clocks.start()
    for s in range(args.warmup):
        step(s)
    torch.cuda.synchronize()
    st = dcp.dcp_get_device_status()
    if st != dcp.DCP_OK:
        raise RuntimeError(f"device status after warm-up: {dcp.status_string(st)}")

    kv_tok = [int(np.sum(w.lengths)) + B * (s + 1) for s in range(n_total)]
    bpt = w.kv_bytes_per_token
    ev_k = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_stop = torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    wall0 = time.time()
    t_start.record(stream)
    for i in range(args.steps):
        step(args.warmup + i, ev_k[i])
    t_stop.record(stream)
    torch.cuda.synchronize()
    wall1 = time.time()
    if world > 1:
        dist.barrier()
    clocks.mark(wall0, wall1)
    clk = clocks.stop()
    st = dcp.dcp_get_device_status()
    if st != dcp.DCP_OK:
        raise RuntimeError(f"device status after timed steps: {dcp.status_string(st)}")
    ms = t_start.elapsed_time(t_stop)
    kern_ms = [a.elapsed_time(b) for a, b in ev_k]
    bytes_timed = sum(kv_tok[args.warmup + i] for i in range(args.steps)) * bpt

    # extra launches on the last timed step's inputs (untimed in `value`): per-request
    # completion times
    last = args.warmup + args.steps - 1
    reps = 5
    bands = None
    if not args.no_bands:
        fin = torch.zeros((reps, B), dtype=torch.int64, device=dev)
        for r in range(reps):
            dcp.dcp_decode_merged(dw.desc, qs[last], lens_s[last], out, lse_out, ws, finish_ns=fin[r])
        torch.cuda.synchronize()
        finish_ms = np.median(fin.cpu().numpy(), axis=0) / 1e6
        bands = band_latency(np.asarray(w.lengths) + last + 1, finish_ms, float(np.median(kern_ms)), bpt)
    # end to end through the C ABI with host buffers: each step's inputs (q, new token
    # rows, positions, lengths) are copied in from pinned memory on one copy stream and
    # its output (out + lse) copied back on another, double-buffered so that the copies
    # of steps s - 1 and s + 1 overlap the compute of step s
    e2e = None
    if E:
        first_e = args.warmup + args.steps
        pin = []
        for s in range(first_e, n_total):
            k, v = new_rows[s]
            pin.append((qs[s].cpu().pin_memory(), k.cpu().pin_memory(), None if v is None else v.cpu().pin_memory(),
                        pos_s[s].cpu().pin_memory(), lens_s[s].cpu().pin_memory()))
        bufs = [tuple(None if t is None else torch.empty(t.shape, dtype=t.dtype, device=dev) for t in pin[0])
                for _ in range(2)]
        outs = [(torch.empty_like(out), torch.empty_like(lse_out)) for _ in range(2)]
        host_out = [(torch.empty(out.shape, dtype=out.dtype).pin_memory(),
                     torch.empty(lse_out.shape, dtype=lse_out.dtype).pin_memory()) for _ in range(2)]
        h2d = sum(t.numel() * t.element_size() for t in pin[0] if t is not None)
        d2h = out.numel() * 4 + lse_out.numel() * 4
        s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_done = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        e0.record(stream)
        s_in.wait_event(e0)
        s_out.wait_event(e0)
        for i, host in enumerate(pin):
            j = i % 2
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_done[j])  # step i - 2 has consumed this input buffer
                for dst, src in zip(bufs[j], host):
                    if src is not None:
                        dst.copy_(src, non_blocking=True)
                ev_in[j].record(s_in)
            stream.wait_event(ev_in[j])
            if i >= 2:
                stream.wait_event(ev_out[j])  # step i - 2's output has been copied out
            q_d, k_d, v_d, p_d, l_d = bufs[j]
            step(first_e + i, pos=p_d, lens=l_d, q=q_d, k=k_d, v=v_d, o=outs[j][0], lo=outs[j][1])
            ev_done[j].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_done[j])
                host_out[j][0].copy_(outs[j][0], non_blocking=True)
                host_out[j][1].copy_(outs[j][1], non_blocking=True)
                ev_out[j].record(s_out)
        stream.wait_stream(s_out)
        e1.record(stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        st = dcp.dcp_get_device_status()
        if st != dcp.DCP_OK:
            raise RuntimeError(f"device status after the end-to-end steps: {dcp.status_string(st)}")
        e2e_ms = e0.elapsed_time(e1)
        e2e_bytes = sum(kv_tok[first_e + i] for i in range(E)) * bpt
        e2e = (e2e_ms, e2e_bytes, h2d, d2h)

    # max over ranks of device time; whole-job bytes
    kern_total = sum(kern_ms)
    if world > 1:
        (ms, kern_total, e2e_ms_max), (bytes_all, e2e_bytes_all) = combine_ranks(
            dist, dev, [ms, kern_total, e2e[0] if e2e else 0.0], [bytes_timed, e2e[1] if e2e else 0])
    else:
        bytes_all = float(bytes_timed)
        e2e_ms_max = e2e[0] if e2e else 0.0
        e2e_bytes_all = float(e2e[1]) if e2e else 0.0

    hbm, peak_kind = peaks()
    traffic = measured_traffic(traffic_key(cfg, w))
    gbs = bytes_all / (ms * 1e-3) / 1e9
    # dominant kernel: the decode (plan + split-KV attention + merge) of one step, CUDA
    # events on its stream
    per_launch_bytes = bytes_timed / args.steps
    kern_avg_ms = kern_total / args.steps
    achieved = per_launch_bytes / (kern_avg_ms * 1e-3) / 1e9
    res = {
        "value": round(gbs, 1),
        "unit": "GB/s",
        "ms_per_step": round(ms / args.steps, 4),
        "steps_per_s": round(args.steps / (ms * 1e-3), 2),
        "pct_hbm_measured": round(100 * gbs / world / hbm, 1),
        "pct_hbm_nominal_8tbs": round(100 * gbs / world / 8000.0, 1),
        "dtype": "bf16" if w.dtype == "bf16" else "fp8_e4m3 cache, bf16 q, fp32 accumulate",
        "config": workload_config(w, cfg) | {"parallelism": f"replicas x{world} (one independent batch per GPU)"},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
                     "frac": round(achieved / hbm, 3), "traffic": traffic,
                     "algorithmic_bytes_per_launch": int(per_launch_bytes),
                     "kernel": "dcp_decode_merged (planner, [fp8 query split], split-KV attention, LSE merge)",
                     "peak_source": f"{peak_kind} hbm_gbs (MEASURED_PEAKS.json)" if peak_kind == "measured"
                     else "fallback 6650 GB/s (no MEASURED_PEAKS.json)"},
        "clocks": clk,
        "gpu_launches": launches_per_step(w) * args.steps,
        "fill_seconds": round(fill_s, 2),
    }
    if bands is not None:
        res["bands"] = bands
    if e2e:
        res["e2e"] = {"value": round(e2e_bytes_all / (e2e_ms_max * 1e-3) / 1e9, 1), "unit": "GB/s",
                      "h2d_bytes_per_step": e2e[2], "d2h_bytes_per_step": e2e[3],
                      "ms_per_step": round(e2e_ms_max / E, 4),
                      "copies": "H2D and D2H on two copy streams, double-buffered, overlapping compute"}
    del dw, ws, qs, new_rows
    torch.cuda.empty_cache()
    return res, w


def measure_dcp(args, cfg, rank, world, local_rank):
    """One DCP group across the ranks (one shard per GPU): each step appends the new
    tokens (every rank is given every token and keeps its own) and runs
    parallel.decode_distributed.  Returns the result dict and the workload."""
    import torch
    import torch.distributed as dist

    import sequence_sharded_paged_b200 as dcp
    import synth.device as sdev
    from sequence_sharded_paged_b200 import parallel
    from sequence_sharded_paged_b200 import workload as wl

    dcp.lib()
    dev = torch.device("cuda", local_rank)
    w = synth.workload(cfg, n_shards=world, interleave=args.interleave)
    if args.batch_limit:
        w.B = min(w.B, args.batch_limit)
        w.lengths = w.lengths[:w.B]
    n_total = args.warmup + args.steps
    counts = wl.gpu_shard_counts(np.asarray(w.lengths) + n_total + 1, world, w.interleave)
    t0 = time.time()
    dw = wl.build(w, counts, rank=rank)
    fill_s = time.time() - t0
    B = w.B
    ws = parallel.rank_workspace(dw.desc, B, device=dev)
    L0 = torch.as_tensor(np.asarray(w.lengths, np.int32), device=dev)
    qs = [sdev.q(w.seed_val, B, w.hq, w.dk, step=s + 1) for s in range(n_total)]
    req = torch.arange(B, dtype=torch.int32, device=dev)
    pos_s = [(L0 + s).contiguous() for s in range(n_total)]
    lens_s = [(L0 + s + 1).contiguous() for s in range(n_total)]
    if w.kind == "gqa":
        new_rows = [sdev.gqa_rows(w.seed_val, req, pos_s[s], w.hkv, w.dk) for s in range(n_total)]
    else:
        new_rows = [(sdev.latent_rows(w.seed_val, req, pos_s[s]), None) for s in range(n_total)]
    stream = torch.cuda.current_stream()

    def step(s):
        k, v = new_rows[s]
        dcp.dcp_kv_append_rank(dw.desc, rank, None, pos_s[s], k, v)
        return parallel.decode_distributed(dw.desc, rank, world, qs[s], lens_s[s], ws)

    clocks = Clocks(local_rank)
    clocks.start()
    for s in range(args.warmup):
        step(s)
    torch.cuda.synchronize()
    if dcp.dcp_get_device_status() != dcp.DCP_OK:
        raise RuntimeError("device status after warm-up")
    dist.barrier()
    torch.cuda.synchronize()
    wall0 = time.time()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(args.steps):
        step(args.warmup + i)
    e1.record(stream)
    torch.cuda.synchronize()
    wall1 = time.time()
    dist.barrier()
    clocks.mark(wall0, wall1)
    clk = clocks.stop()
    if dcp.dcp_get_device_status() != dcp.DCP_OK:
        raise RuntimeError("device status after the timed steps")
    (ms,), _ = combine_ranks(dist, dev, [e0.elapsed_time(e1)], [0])
    kv_tok = sum(int(np.sum(w.lengths)) + B * (args.warmup + i + 1) for i in range(args.steps))
    bytes_all = kv_tok * w.kv_bytes_per_token  # the group decodes the batch once per step
    hbm, peak_kind = peaks()
    gbs = bytes_all / (ms * 1e-3) / 1e9
    per_gpu = gbs / world
    res = {
        "value": round(gbs, 1), "unit": "GB/s", "ms_per_step": round(ms / args.steps, 4),
        "steps_per_s": round(args.steps / (ms * 1e-3), 2),
        "pct_hbm_measured": round(100 * per_gpu / hbm, 1), "pct_hbm_nominal_8tbs": round(100 * per_gpu / 8000.0, 1),
        "dtype": "bf16" if w.dtype == "bf16" else "fp8_e4m3 cache, bf16 q, fp32 accumulate",
        "config": workload_config(w, cfg) | {"parallelism": f"DCP across {world} GPU(s): one shard per GPU, "
                                                             f"all-gather of LSEs + reduce-scatter over heads"},
        "roofline": {"bound": "hbm", "achieved": round(per_gpu, 1), "peak": hbm, "unit": "GB/s",
                     "frac": round(per_gpu / hbm, 3), "traffic": None,
                     "kernel": "whole DCP step per GPU (append, rank decode, exchange)",
                     "peak_source": f"{peak_kind} hbm_gbs"},
        "clocks": clk,
        "gpu_launches": (5 if (w.kind == "mla" and w.dtype == "fp8") else 4) * args.steps,
        "fill_seconds": round(fill_s, 2),
    }
    del dw, ws, qs, new_rows
    torch.cuda.empty_cache()
    return res, w


# ----------------------------------------------------------------------------
# the oracle on host cores (CPU baseline / reference arm)
# ----------------------------------------------------------------------------

def _oracle_run(w, q64, reqs):
    """The oracle as it stands: unsharded float64 decode attention of the listed
    requests, reading the inputs from the counter-based generator in C."""
    import oracle
    oracle.decode_synth(w.kind, w.dtype, w.seed_val, q64, w.lengths, w.scale, w.hkv, w.dk, w.dv,
                        req_list=np.asarray(reqs, dtype=np.int64))


def oracle_sample(w, cpu_seconds: float, q64):
    """Requests (a seeded shuffle) holding about cpu_seconds of oracle work: the
    shortest request is timed first and the rate extrapolated (conservatively:
    more requests run more parallel work items)."""
    order = [int(b) for b in np.argsort(synth.bits(synth.key(w.seed_len, 7), np.arange(w.B)))]
    probe = sorted(order, key=lambda b: int(w.lengths[b]))[:4]  # enough work items for the threads
    t0 = time.perf_counter()
    _oracle_run(w, q64, probe)
    rate = max(1.0, float(sum(int(w.lengths[b]) for b in probe))) / max(time.perf_counter() - t0, 1e-4)
    budget_tok = max(int(min(w.lengths)), int(cpu_seconds * rate))
    reqs, tot = [], 0
    for b in order:
        if tot + int(w.lengths[b]) > budget_tok and reqs:
            continue
        reqs.append(b)
        tot += int(w.lengths[b])
        if tot >= budget_tok:
            break
    return sorted(reqs), tot


def time_oracle(w, cpu_seconds: float):
    """Time the oracle (as it stands) on a bounded sample; returns dict."""
    import oracle
    q64 = synth.bf16_bits_to_f64(synth.q_bf16(w.seed_val, w.B, w.hq, w.dk))
    reqs, tot = oracle_sample(w, cpu_seconds, q64)
    t0 = time.perf_counter()
    _oracle_run(w, q64, reqs)
    dt = time.perf_counter() - t0
    kv_bytes = tot * w.kv_bytes_per_token
    return {"value": round(kv_bytes / dt / 1e9, 4), "unit": "GB/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{len(reqs)} of {w.B} requests ({tot} tokens, all {w.hq} heads, unsharded "
                      f"float64 decode attention, inputs read from the generator), {dt:.1f} s"}, dt, kv_bytes


def run_reference(args):
    w = get_workload(args)
    per_step = max(1.0, min(20.0, 120.0 / max(1, args.steps + args.warmup)))
    import oracle
    q64 = synth.bf16_bits_to_f64(synth.q_bf16(w.seed_val, w.B, w.hq, w.dk))
    reqs, tot = oracle_sample(w, per_step, q64)
    kv_bytes = tot * w.kv_bytes_per_token
    for _ in range(args.warmup):
        _oracle_run(w, q64, reqs)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        _oracle_run(w, q64, reqs)
    dt = time.perf_counter() - t0
    gbs = kv_bytes * args.steps / dt / 1e9
    sample = (f"each step: {len(reqs)} of {w.B} requests ({tot} tokens, all {w.hq} heads) "
              f"of the workload, unsharded float64 decode attention on host cores")
    return {
        "impl": "reference",
        "metric": METRIC, "value": round(gbs, 4), "unit": "GB/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 2),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded counter-based generator)",
        "config": workload_config(w, args.config) | {"parallelism": "host cores (OpenMP)"},
        "cpu_baseline": {"value": round(gbs, 4), "unit": "GB/s", "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return
    import torch
    import torch.distributed as dist
    torch.cuda.set_device(local_rank)
    if args.dcp_across_gpus and world == 1:
        # a group of one still runs the exchange through NCCL
        import socket
        with socket.socket() as sk:
            sk.bind(("127.0.0.1", 0))
            port = sk.getsockname()[1]
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        os.environ.setdefault("MASTER_PORT", str(port))
        os.environ.setdefault("RANK", "0")
        os.environ.setdefault("WORLD_SIZE", "1")
    if world > 1 or args.dcp_across_gpus:
        import datetime
        # a short timeout ends a rank's collective with an error if another rank has failed
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120 if args.dcp_across_gpus else 600),
                                device_id=torch.device("cuda", local_rank))
    try:
        if args.dcp_across_gpus:
            r, w = measure_dcp(args, args.config, rank, world, local_rank)
        else:
            r, w = measure(args, args.config, rank, world, local_rank, True)
        res = {"metric": METRIC, "value": r["value"], "unit": "GB/s", "n_gpus": world, "steps": args.steps,
               "warmup": args.warmup, "ms_per_step": r["ms_per_step"], "steps_per_s": r["steps_per_s"],
               "higher_is_better": True, "scaling": "strong" if args.dcp_across_gpus else "weak",
               "vs_baseline": None, "dtype": r["dtype"],
               "data": "synthetic (seeded counter-based generator; lengths shaped like the agentic trace)"}
        res.update({k: v for k, v in r.items() if k not in res})
        others = ([int(c) for c in args.per_config.split(",") if c.strip()]
                  if world == 1 and not args.dcp_across_gpus else [])
        per = {}
        for cfg in others:
            if cfg == args.config:
                continue
            rc, _ = measure(args, cfg, rank, world, local_rank, False)
            per[f"config{cfg}"] = rc
        if per:
            res["per_config"] = per
        if rank == 0 and not args.no_cpu_baseline:
            cb, _, _ = time_oracle(w, args.cpu_seconds)
            res["cpu_baseline"] = cb
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1 or args.dcp_across_gpus:
            dist.barrier()
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
