"""The multi-GPU exchange of sequence_sharded_paged_b200.parallel on gloo ranks
(CPU processes): all-gather of the LSEs, the local reweighting, and the
reduce-scatter of the outputs over query rows.

Each rank starts from the oracle's float64 partial of its shard (rounded to
fp32, as the decode kernels emit it).  The reweighting kernel (dcp_lse_rescale)
needs a GPU; here a float64 stand-in written from the same formula takes its
place, and the GPU tests check the kernel itself.  What this test checks is the
exchange: which tensors travel, the layout of the reduce-scatter, and that the
rows each rank ends with are the unsharded decode's."""
from __future__ import annotations

import os
import queue
import socket
import sys
import time

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rescale_f64(lse_all, rank, o, o_rs, lse_out):
    """LSE = M + ln sum_n exp(lse_n - M); o_rs[n][b][r][:] = exp(lse_rank - LSE) o[b][n*H/N + r][:]."""
    la = lse_all.double().numpy()
    N, B, H = la.shape
    M = la.max(axis=0)
    with np.errstate(invalid="ignore", divide="ignore"):
        L = np.where(np.isneginf(M), -np.inf, M + np.log(np.exp(la - np.where(np.isneginf(M), 0, M)).sum(axis=0)))
        w = np.where(np.isneginf(la[rank]), 0.0, np.exp(la[rank] - np.where(np.isneginf(L), 0, L)))
    scaled = w[:, :, None] * o.double().numpy()
    o_rs.copy_(torch.from_numpy(scaled.reshape(B, N, H // N, -1).transpose(1, 0, 2, 3).copy()).float())
    lse_out.copy_(torch.from_numpy(L).float())


def _case(N, I, kind):
    import oracle
    import synth
    rng = np.random.default_rng(N * 10 + I)
    B, Hq = 3, 8
    if kind == "gqa":
        Hkv, D, Dv = 2, 16, 16
        L = np.array([1, 37, 150])
        q = rng.standard_normal((B, Hq, D))
        K = rng.standard_normal((B, 150, Hkv, D))
        V = rng.standard_normal((B, 150, Hkv, Dv))
        parts = [oracle.decode_arrays("gqa", q, K, V, L, 0.25, hkv=Hkv, N=N, I=I, shard=n) for n in range(N)]
        full = oracle.decode_arrays("gqa", q, K, V, L, 0.25, hkv=Hkv)
    else:
        D, Dv = 24, 16
        L = np.array([2, 90, 41])
        q = rng.standard_normal((B, Hq, D))
        K = rng.standard_normal((B, 90, D))
        parts = [oracle.decode_arrays("mla", q, K, None, L, 0.2, dv=Dv, N=N, I=I, shard=n) for n in range(N)]
        full = oracle.decode_arrays("mla", q, K, None, L, 0.2, dv=Dv)
    del synth
    return parts, full


def _rank_main(rank, world, port, I, kind, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from sequence_sharded_paged_b200 import parallel
        parts, _ = _case(world, I, kind)
        O_r, L_r = parts[rank]
        out, lse = parallel.exchange(torch.from_numpy(O_r).float(), torch.from_numpy(L_r).float(), rank, world,
                                     rescale=_rescale_f64)
        q.put((rank, out.numpy(), lse.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,I,kind", [(2, 1, "gqa"), (2, 16, "mla"), (4, 3, "gqa"), (4, 1, "mla")])
def test_exchange_on_gloo_ranks(world, I, kind):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, I, kind, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    deadline = time.time() + 180
    while len(res) < world:
        try:
            r, out, lse = q.get(timeout=2)
            res[r] = (out, lse)
        except queue.Empty:
            # a rank that died will never report: fail now instead of waiting out the deadline
            assert all(p.exitcode in (None, 0) for p in procs), [p.exitcode for p in procs]
            assert time.time() < deadline, "ranks did not report"
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    _, (O, L) = _case(world, I, kind)
    H = O.shape[1]
    rows = H // world
    for r in range(world):
        out, lse = res[r]
        np.testing.assert_allclose(out, O[:, r * rows:(r + 1) * rows], rtol=0, atol=2e-6)
        fin = ~np.isneginf(L)
        assert np.array_equal(np.isneginf(lse), ~fin)
        np.testing.assert_allclose(lse[fin], L[fin], rtol=0, atol=2e-6)


def test_exchange_rejects_rows_not_divisible_by_ranks():
    from sequence_sharded_paged_b200 import parallel
    with pytest.raises(ValueError):
        parallel.exchange(torch.zeros(2, 6, 4), torch.zeros(2, 6), 0, 4)
