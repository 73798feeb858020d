"""The multi-GPU decode on ONE GPU (marked gpu): the rank-local calls
(dcp_kv_append_rank, dcp_decode_rank, dcp_lse_rescale) against the oracle.

An N-rank group is emulated by building N rank-local caches on the one GPU,
one after the other (each holds only its shard's pages and block tables and is
filled from every position through dcp_kv_append_rank).  The all-gather is a
stack of the ranks' LSEs and the reduce-scatter a sum of their reweighted
blocks; no rank waits on another.  The real collectives run in
test_parallel_cpu.py (gloo ranks) and, here, on a one-rank NCCL group."""
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import oracle
import sequence_sharded_paged_b200 as dcp
import synth.device as sdev
from sequence_sharded_paged_b200 import parallel
from sequence_sharded_paged_b200 import workload as wl

from gpu_util import compare, oracle_decode, small_workload, vmax_attended

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clear_status():
    dcp.dcp_get_device_status()
    yield


def _rank_cache(w, rank):
    counts = oracle.shard_counts(np.asarray(w.lengths), w.n_shards, w.interleave)
    return wl.build(w, counts, rank=rank)


CASES = [
    ("gqa", "bf16", 8, 2, 64, 64, 16, 2, 1, [300, 1000, 1]),             # CUDA-core GQA
    ("gqa", "bf16", 64, 4, 128, 128, 16, 4, 16, [20_000, 129, 7]),       # tensor-core GQA
    ("mla", "bf16", 16, 1, 576, 512, 64, 2, 1, [9000, 65, 3]),           # tcgen05 bf16
    ("mla", "fp8", 64, 1, 576, 512, 64, 8, 1, [30_000, 200, 5]),         # tcgen05 fp8
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c[0]}-{c[1]}-hq{c[2]}-N{c[7]}")
def test_emulated_group_matches_oracle(case):
    kind, dtype, hq, hkv, dk, dv, P, N, I, L = case
    w = small_workload(kind, dtype, L, hq, hkv, dk, dv, P, N, I, seed=61)
    q = sdev.q(w.seed_val, w.B, w.hq, w.dk, 0)
    vmax = vmax_attended(w)
    o_r, lse_r = [], []
    for r in range(N):
        dw = _rank_cache(w, r)
        o = torch.full((w.B, hq, dv), float("nan"), dtype=torch.float32, device="cuda")
        lse = torch.full((w.B, hq), float("nan"), dtype=torch.float32, device="cuda")
        dcp.dcp_decode_rank(dw.desc, r, q, dw.seq_lens, o, lse, dw.ws)
        torch.cuda.synchronize()
        assert dcp.dcp_get_device_status() == dcp.DCP_OK
        O_n, L_n = oracle_decode(w, shard=r)
        compare(f"{w.name} rank {r}", o.cpu().numpy(), lse.cpu().numpy(), O_n, L_n, w.dtype, vmax)
        o_r.append(o)
        lse_r.append(lse)
        del dw
    lse_all = torch.stack(lse_r)                      # the all-gather
    out = torch.zeros((N, w.B, hq // N, dv), dtype=torch.float32, device="cuda")
    lse_full = None
    for r in range(N):
        o_rs = torch.full((N, w.B, hq // N, dv), float("nan"), dtype=torch.float32, device="cuda")
        lf = torch.empty((w.B, hq), dtype=torch.float32, device="cuda")
        dcp.dcp_lse_rescale(lse_all, r, o_r[r], o_rs, lf)
        out += o_rs                                   # the reduce-scatter's sum
        lse_full = lf
    torch.cuda.synchronize()
    merged = out.permute(1, 0, 2, 3).reshape(w.B, hq, dv).cpu().numpy()  # rank n holds rows n*hq/N ..
    O, Lf = oracle_decode(w)
    e = compare(f"{w.name} emulated {N}-rank group", merged, lse_full.cpu().numpy(), O, Lf, w.dtype, vmax)
    print(f"{w.name} {N} ranks: max|dO|/max|V| = {e[0]:.2e}, max|dLSE| = {e[1]:.2e}")


def test_append_rank_stores_only_owned_rows():
    """A rank given every new token stores exactly its own (no status error for the others)."""
    w = small_workload("mla", "bf16", [130, 64], 16, 1, 576, 512, 64, 4, 1, seed=63)
    for r in range(4):
        dw = _rank_cache(w, r)
        assert dcp.dcp_get_device_status() == dcp.DCP_OK
        counts = oracle.shard_counts(np.asarray(w.lengths), 4, 1)[r]
        q = sdev.q(w.seed_val, w.B, w.hq, w.dk, 0)
        o = torch.empty((w.B, 16, 512), dtype=torch.float32, device="cuda")
        lse = torch.empty((w.B, 16), dtype=torch.float32, device="cuda")
        dcp.dcp_decode_rank(dw.desc, r, q, dw.seq_lens, o, lse, dw.ws)
        O_n, L_n = oracle_decode(w, shard=r)
        compare(f"rank {r} ({counts.tolist()} tokens)", o.cpu().numpy(), lse.cpu().numpy(), O_n, L_n, "bf16",
                vmax_attended(w))
        assert dcp.dcp_get_device_status() == dcp.DCP_OK


@pytest.mark.parametrize("N,B,H,Dv", [(2, 3, 8, 64), (4, 5, 64, 512), (8, 2, 16, 128), (1, 4, 4, 4)])
def test_lse_rescale_kernel(N, B, H, Dv):
    rng = np.random.default_rng(N * 100 + H)
    la = (rng.standard_normal((N, B, H)) * 4).astype(np.float32)
    la[rng.random((N, B, H)) < 0.25] = -np.inf
    la[:, 0, 0] = -np.inf                               # a row no rank attends
    o = rng.standard_normal((N, B, H, Dv)).astype(np.float32)
    O_ref, L_ref = oracle.merge(np.where(np.isneginf(la)[..., None], 0.0, o).astype(np.float64), la.astype(np.float64))
    lse_all = torch.as_tensor(la, device="cuda")
    acc = np.zeros((N, B, H // N, Dv))
    for r in range(N):
        o_rs = torch.empty((N, B, H // N, Dv), dtype=torch.float32, device="cuda")
        lo = torch.empty((B, H), dtype=torch.float32, device="cuda")
        dcp.dcp_lse_rescale(lse_all, r, torch.as_tensor(o[r], device="cuda"), o_rs, lo)
        acc += o_rs.cpu().numpy()
        lo = lo.cpu().numpy()
        assert np.array_equal(np.isneginf(lo), np.isneginf(L_ref))
        fin = ~np.isneginf(L_ref)
        assert np.abs(lo[fin] - L_ref[fin]).max() <= 1e-5
    merged = acc.transpose(1, 0, 2, 3).reshape(B, H, Dv)
    assert np.abs(merged - O_ref).max() <= 1e-5 * max(1.0, np.abs(o).max())


def test_exchange_on_a_one_rank_nccl_group():
    """parallel.decode_distributed with its real NCCL collectives, on a group of one."""
    w = small_workload("mla", "fp8", [5000, 70, 1], 64, 1, 576, 512, 64, 1, 1, seed=65)
    dw = _rank_cache(w, 0)
    q = sdev.q(w.seed_val, w.B, w.hq, w.dk, 0)
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    store = dist.TCPStore("127.0.0.1", port, 1, True)
    dist.init_process_group("nccl", store=store, rank=0, world_size=1, device_id=torch.device("cuda", 0))
    try:
        out, lse = parallel.decode_distributed(dw.desc, 0, 1, q, dw.seq_lens, parallel.rank_workspace(dw.desc, w.B,
                                                                                                      device="cuda"))
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    assert dcp.dcp_get_device_status() == dcp.DCP_OK
    O, L = oracle_decode(w)
    compare("one-rank NCCL group", out.cpu().numpy(), lse.cpu().numpy(), O, L, "fp8", vmax_attended(w))
