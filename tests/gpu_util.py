"""Shared helpers of the GPU parity tests: build a workload through libdcp,
run one decode step, and compute the oracle's answer on the same seeded inputs."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import sequence_sharded_paged_b200 as dcp
import synth
import synth.device as sdev
from sequence_sharded_paged_b200 import workload as wl

# parity bars (float): max|O - O_oracle| <= TOL_O[dtype] * max|V|; |LSE - LSE_oracle| <= TOL_LSE
TOL_O = {"bf16": 2e-3, "fp8": 2e-2}
TOL_LSE = 1e-3
# The generator bounds every value by |x| <= 3.4641 (Irwin-Hall of four uniforms).
VMAX_BOUND = 3.4641


def small_workload(kind, dtype, lengths, hq, hkv, dk, dv, page_size, n_shards, interleave, scale=None, seed=7):
    lengths = np.asarray(lengths, dtype=np.int64)
    w = synth.Workload(f"test-{kind}-{dtype}", kind, dtype, len(lengths), hq, hkv, dk, dv, page_size, n_shards,
                       interleave, scale if scale is not None else 1.0 / np.sqrt(dk if kind == "gqa" else 192),
                       seed, seed + 1000)
    w.lengths = lengths
    return w


def build_for_test(w: synth.Workload, growth: int = 0, fill: bool = True):
    """Pages sized from the ORACLE's shard counts (no test input comes from the CUDA path)."""
    counts = oracle.shard_counts(np.asarray(w.lengths) + growth, w.n_shards, w.interleave)
    return wl.build(w, counts, fill=fill)


def run_step(dw, step: int = 0):
    w = dw.w
    q = sdev.q(w.seed_val, w.B, w.hq, w.dk, step)
    o_part = torch.empty((w.n_shards, w.B, w.hq, w.dv), dtype=torch.float32, device="cuda")
    lse = torch.empty((w.n_shards, w.B, w.hq), dtype=torch.float32, device="cuda")
    dcp.dcp_decode_partial(dw.desc, q, dw.seq_lens, o_part, lse, dw.ws)
    out = torch.empty((w.B, w.hq, w.dv), dtype=torch.float32, device="cuda")
    lse_out = torch.empty((w.B, w.hq), dtype=torch.float32, device="cuda")
    dcp.dcp_merge(o_part, lse, out, lse_out)
    torch.cuda.synchronize()
    status = dcp.dcp_get_device_status()
    return o_part.cpu().numpy(), lse.cpu().numpy(), out.cpu().numpy(), lse_out.cpu().numpy(), status


def oracle_q(w, step=0):
    return synth.bf16_bits_to_f64(synth.q_bf16(w.seed_val, w.B, w.hq, w.dk, step))


def oracle_decode(w, lengths=None, shard=-1, req_list=None, step=0):
    L = np.asarray(w.lengths if lengths is None else lengths, dtype=np.int64)
    return oracle.decode_synth(w.kind, w.dtype, w.seed_val, oracle_q(w, step), L, w.scale, w.hkv, w.dk, w.dv,
                               N=w.n_shards, I=w.interleave, shard=shard, req_list=req_list)


def vmax_attended(w, req_list=None, lengths=None):
    """max |V| over the value entries actually attended (exact, host generator);
    for fp8 the oracle's dequantised values."""
    L = np.asarray(w.lengths if lengths is None else lengths, dtype=np.int64)
    reqs = range(w.B) if req_list is None else req_list
    m = 0.0
    for b in reqs:
        if L[b] == 0:
            continue
        if w.kind == "gqa":
            rows = synth.kv_rows_bf16(w.seed_val, synth.T_V, b, np.arange(L[b]), w.hkv, w.dv)
            m = max(m, float(np.abs(synth.bf16_bits_to_f64(rows)).max()))
        else:
            rows = synth.kv_rows_bf16(w.seed_val, synth.T_LATENT, b, np.arange(L[b]), 1, 576)[:, 0, :]
            if w.dtype == "fp8":
                codes, sc = oracle.quantize_rows_e4m3(rows)
                deq = oracle.e4m3_table()[codes[:, :w.dv]] * sc.astype(np.float64)[:, None]
                m = max(m, float(np.abs(deq).max()))
            else:
                m = max(m, float(np.abs(synth.bf16_bits_to_f64(rows[:, :w.dv])).max()))
    return m


def compare(name, o_gpu, lse_gpu, o_ref, lse_ref, dtype, vmax):
    """Assert the float parity bar; returns (max|dO|/vmax, max|dLSE|)."""
    o_gpu = np.asarray(o_gpu, np.float64)
    lse_gpu = np.asarray(lse_gpu, np.float64)
    ninf_ref = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse_gpu), ninf_ref), f"{name}: -inf pattern of LSE differs"
    assert np.all(np.isfinite(o_gpu)), f"{name}: non-finite output"
    if ninf_ref.any():
        assert np.all(o_gpu[ninf_ref] == 0.0), f"{name}: empty shard output not zero"
    fin = ~ninf_ref
    d_lse = float(np.abs(lse_gpu[fin] - lse_ref[fin]).max()) if fin.any() else 0.0
    d_o = float(np.abs(o_gpu - o_ref).max())
    tol_o = TOL_O[dtype] * vmax
    assert d_o <= tol_o, f"{name}: max|dO| = {d_o:.3e} > {tol_o:.3e}"
    assert d_lse <= TOL_LSE, f"{name}: max|dLSE| = {d_lse:.3e} > {TOL_LSE}"
    return d_o / vmax, d_lse
