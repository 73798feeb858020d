"""Parity at the full workload sizes, in the launch configuration the benchmark
times (marked gpu).  The oracle computes sampled requests (all heads) one by
one: the longest request (many split chunks per shard), a short one and the
median one; per-shard partials and the merged output are compared."""
import numpy as np
import pytest
import torch

import sequence_sharded_paged_b200 as dcp
import synth
from sequence_sharded_paged_b200 import workload as wl

from gpu_util import compare, oracle_decode, run_step, VMAX_BOUND
import oracle

pytestmark = pytest.mark.gpu


def _sample(w):
    L = np.asarray(w.lengths)
    order = np.argsort(L)
    return sorted({int(order[-1]), int(order[0]), int(order[len(order) // 2])})


def _build(w):
    counts = oracle.shard_counts(np.asarray(w.lengths), w.n_shards, w.interleave)
    return wl.build(w, counts)


def _check_full(w, shards=True):
    dw = _build(w)
    o_part, lse, out, lse_out, status = run_step(dw)
    assert status == dcp.DCP_OK, dcp.status_string(status)
    reqs = _sample(w)
    # max|V| bound of the generator (|x| <= 3.4641; the fp8 dequantised values obey it too)
    if shards:
        for n in range(w.n_shards):
            O_n, L_n = oracle_decode(w, shard=n, req_list=reqs)
            compare(f"{w.name} shard {n}", o_part[n][reqs], lse[n][reqs], O_n[reqs], L_n[reqs], w.dtype, VMAX_BOUND)
    O, L = oracle_decode(w, req_list=reqs)
    e = compare(f"{w.name} merged", out[reqs], lse_out[reqs], O[reqs], L[reqs], w.dtype, VMAX_BOUND)
    print(f"{w.name}: requests {reqs} lengths {[int(w.lengths[b]) for b in reqs]}: "
          f"max|dO|/3.4641 = {e[0]:.2e}, max|dLSE| = {e[1]:.2e}")
    del dw
    torch.cuda.empty_cache()
    return O, L, reqs


def test_fullsize_config3_gqa_qwen3():
    _check_full(synth.workload(3))


def test_fullsize_config4_mla_kimi_bf16():
    _check_full(synth.workload(4))


def test_fullsize_config5_mla_kimi_fp8_sweep():
    """The N x I sweep of the high-concurrency fp8 workload: the unsharded
    oracle answer is shared by all 12 points; per-shard partials are checked at
    the default point (N=8, I=1) and at one block-aligned point."""
    base = synth.workload(5)
    O, L, reqs = _check_full(base)
    for N in (1, 2, 4, 8):
        for I in (1, 16, 64):
            if (N, I) == (8, 1):
                continue
            w = synth.workload(5, n_shards=N, interleave=I)
            if (N, I) == (4, 64):
                _check_full(w)
                continue
            dw = _build(w)
            o_part, lse, out, lse_out, status = run_step(dw)
            assert status == dcp.DCP_OK
            compare(f"{w.name} N={N} I={I} merged", out[reqs], lse_out[reqs], O[reqs], L[reqs], w.dtype, VMAX_BOUND)
            del dw
            torch.cuda.empty_cache()
