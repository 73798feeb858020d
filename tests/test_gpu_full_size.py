"""Parity at the full workload sizes, in the launch configuration the benchmark
times (marked gpu).  A seeded sample of at least 16 requests, drawn from every
request-length band the workload has plus its longest, shortest and median
requests, is computed by the oracle one request at a time (all heads).  The
fused call the benchmark times (dcp_decode_merged) and dcp_decode_partial +
dcp_merge are both compared with the unsharded oracle, and the per-shard
partials of part of the sample with the oracle's per-shard partials, against
max|V| over the values those requests actually attend."""
import numpy as np
import pytest
import torch

import oracle
import sequence_sharded_paged_b200 as dcp
import synth
import synth.device as sdev
from sequence_sharded_paged_b200 import workload as wl

from gpu_util import compare, oracle_decode, run_step, vmax_attended

pytestmark = pytest.mark.gpu

BANDS = [(0, 32_000), (32_000, 64_000), (64_000, 128_000), (128_000, 200_000), (200_000, 1 << 31)]
N_SAMPLE = 16
N_SHARD_SAMPLE = 6


def _sample(w):
    """At least N_SAMPLE requests: every length band the workload has, evenly,
    plus its longest, shortest and median requests (seeded)."""
    L = np.asarray(w.lengths)
    order = np.argsort(L, kind="stable")
    picks = [int(order[-1]), int(order[0]), int(order[len(order) // 2])]
    rng = np.random.default_rng(w.seed_len + 99)
    bands = [np.flatnonzero((L >= lo) & (L < hi)) for lo, hi in BANDS]
    bands = [ix for ix in bands if ix.size]
    per = -(-(N_SAMPLE - len(picks)) // len(bands))
    for ix in bands:
        picks += [int(b) for b in rng.choice(ix, size=min(per, ix.size), replace=False)]
    # bands with fewer requests than their share: top up from the rest
    picks += [int(b) for b in rng.permutation(len(L))]
    seen, out = set(), []
    for b in picks:
        if b not in seen:
            seen.add(b)
            out.append(b)
    return out[:max(N_SAMPLE, len(set(picks[:3 + per * len(bands)])))]


def _build(w):
    counts = oracle.shard_counts(np.asarray(w.lengths), w.n_shards, w.interleave)
    return wl.build(w, counts)


def _merged(dw):
    w = dw.w
    q = sdev.q(w.seed_val, w.B, w.hq, w.dk, 0)
    ws = torch.empty(dcp.dcp_decode_workspace_size_ex(dw.desc, w.B, 1, dcp.DCP_DECODE_MERGED), dtype=torch.uint8, device="cuda")
    out = torch.full((w.B, w.hq, w.dv), float("nan"), dtype=torch.float32, device="cuda")
    lse = torch.full((w.B, w.hq), float("nan"), dtype=torch.float32, device="cuda")
    dcp.dcp_decode_merged(dw.desc, q, dw.seq_lens, out, lse, ws)
    torch.cuda.synchronize()
    assert dcp.dcp_get_device_status() == dcp.DCP_OK
    return out.cpu().numpy(), lse.cpu().numpy()


def _check_full(w, reqs=None, ref=None, vmax=None, shards=True):
    dw = _build(w)
    o_part, lse, out, lse_out, status = run_step(dw)
    assert status == dcp.DCP_OK, dcp.status_string(status)
    m_out, m_lse = _merged(dw)
    reqs = _sample(w) if reqs is None else reqs
    vmax = vmax_attended(w, reqs) if vmax is None else vmax
    if shards:
        rs = reqs[:N_SHARD_SAMPLE]
        for n in range(w.n_shards):
            O_n, L_n = oracle_decode(w, shard=n, req_list=rs)
            compare(f"{w.name} shard {n}", o_part[n][rs], lse[n][rs], O_n[rs], L_n[rs], w.dtype, vmax)
    O, L = oracle_decode(w, req_list=reqs) if ref is None else ref
    e1 = compare(f"{w.name} partial + merge", out[reqs], lse_out[reqs], O[reqs], L[reqs], w.dtype, vmax)
    e2 = compare(f"{w.name} merged", m_out[reqs], m_lse[reqs], O[reqs], L[reqs], w.dtype, vmax)
    print(f"{w.name}: {len(reqs)} requests, lengths {sorted(int(w.lengths[b]) for b in reqs)}, max|V| {vmax:.4f}: "
          f"partial+merge max|dO|/max|V| = {e1[0]:.2e}, merged {e2[0]:.2e}, max|dLSE| = {max(e1[1], e2[1]):.2e}")
    del dw
    torch.cuda.empty_cache()
    return (O, L), reqs, vmax


def test_sample_covers_every_band():
    for cfg in (3, 4, 5):
        w = synth.workload(cfg)
        reqs = _sample(w)
        L = np.asarray(w.lengths)
        assert len(reqs) >= N_SAMPLE and len(set(reqs)) == len(reqs)
        for lo, hi in BANDS:
            if ((L >= lo) & (L < hi)).any():
                assert any(lo <= L[b] < hi for b in reqs), (cfg, lo)


def test_fullsize_config3_gqa_qwen3():
    _check_full(synth.workload(3))


def test_fullsize_config4_mla_kimi_bf16():
    _check_full(synth.workload(4))


def test_fullsize_config5_mla_kimi_fp8_sweep():
    """The N x I sweep of the high-concurrency fp8 workload: the unsharded
    oracle answer is shared by all 12 points; per-shard partials are checked at
    the default point (N=8, I=1) and at one block-aligned point (N=4, I=64)."""
    ref, reqs, vmax = _check_full(synth.workload(5))
    for N in (1, 2, 4, 8):
        for I in (1, 16, 64):
            if (N, I) == (8, 1):
                continue
            _check_full(synth.workload(5, n_shards=N, interleave=I), reqs=reqs, ref=ref, vmax=vmax,
                        shards=(N, I) == (4, 64))
