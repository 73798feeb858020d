"""GPU parity of the fused decode (dcp_decode_merged) and of several query
tokens per request (dcp_decode_partial_multi, dcp_decode_merged with q_len > 1)
against the float64 oracle (marked gpu).

Bars as for the other decode tests: max|O - O_oracle| <= 2e-3 max|V| (bf16
cache) or 2e-2 max|V| (fp8 cache), |LSE - LSE_oracle| <= 1e-3, with max|V| over
the values actually attended."""
import numpy as np
import pytest
import torch

import oracle
import sequence_sharded_paged_b200 as dcp
import synth
import synth.device as sdev

from gpu_util import build_for_test, compare, oracle_decode, small_workload, vmax_attended

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clear_status():
    dcp.dcp_get_device_status()
    yield


def _ws(dw, q_len, merged):
    mode = dcp.DCP_DECODE_MERGED if merged else dcp.DCP_DECODE_PARTIAL
    n = dcp.dcp_decode_workspace_size_ex(dw.desc, dw.w.B, q_len, mode)
    assert n > 0
    return torch.empty(n, dtype=torch.uint8, device="cuda")


def run_merged(dw, step=0, finish=False):
    w = dw.w
    q = sdev.q(w.seed_val, w.B, w.hq, w.dk, step)
    out = torch.full((w.B, w.hq, w.dv), float("nan"), dtype=torch.float32, device="cuda")
    lse = torch.full((w.B, w.hq), float("nan"), dtype=torch.float32, device="cuda")
    fin = torch.full((w.B,), -1, dtype=torch.int64, device="cuda") if finish else None
    dcp.dcp_decode_merged(dw.desc, q, dw.seq_lens, out, lse, _ws(dw, 1, True), finish_ns=fin)
    torch.cuda.synchronize()
    status = dcp.dcp_get_device_status()
    return out.cpu().numpy(), lse.cpu().numpy(), (fin.cpu().numpy() if finish else None), status


MERGED_CASES = [
    # (kind, dtype, hq, hkv, D, page, N, I, lengths): every kernel family, empty requests,
    # shards without tokens, shards cut into many chunks (both merge levels)
    ("gqa", "bf16", 8, 2, 64, 16, 2, 1, [300, 1000, 0, 1]),              # CUDA-core GQA
    ("gqa", "bf16", 8, 2, 64, 16, 2, 1, [20_000, 7, 0]),                 # shards of ~20 chunks
    ("gqa", "bf16", 64, 4, 128, 16, 2, 16, [20_000, 5, 1]),              # tensor-core GQA, ~10 chunks
    ("gqa", "bf16", 64, 4, 128, 16, 8, 128, [1, 200, 3000, 130, 0, 5000]),  # tensor-core GQA
    ("gqa", "bf16", 32, 2, 128, 64, 3, 16, [17, 64, 4100, 2]),
    ("mla", "bf16", 16, 1, 576, 512, 64, 2, 1, [900, 3000, 1, 0]),        # tcgen05 bf16
    ("mla", "bf16", 64, 1, 576, 512, 64, 8, 1, [40_000, 63, 64, 65, 7]),
    ("mla", "fp8", 64, 1, 576, 512, 64, 4, 16, [5000, 333, 2048, 0, 1]),  # tcgen05 fp8
    ("mla", "fp8", 32, 1, 576, 512, 64, 8, 64, [30_000, 100, 9]),
    ("mla", "bf16", 16, 1, 576, 512, 16, 2, 1, [1, 200, 3000]),           # CUDA-core MLA (page 16)
    ("mla", "bf16", 64, 1, 576, 512, 64, 8, 1, [200_000, 50, 3]),         # 8 shards of ~12 chunks each
]


def _case_workload(c, seed):
    if len(c) == 9:
        kind, dtype, hq, hkv, D, P, N, I, L = c
        return small_workload(kind, dtype, L, hq, hkv, D, D, P, N, I, seed=seed)
    kind, dtype, hq, hkv, dk, dv, P, N, I, L = c
    return small_workload(kind, dtype, L, hq, hkv, dk, dv, P, N, I, seed=seed)


@pytest.mark.parametrize("case", MERGED_CASES, ids=lambda c: f"{c[0]}-{c[1]}-hq{c[2]}-N{c[-3]}-I{c[-2]}")
def test_merged_matches_unsharded_oracle(case):
    w = _case_workload(case, seed=41)
    dw = build_for_test(w)
    out, lse, fin, status = run_merged(dw, finish=True)
    assert status == dcp.DCP_OK, dcp.status_string(status)
    O, L = oracle_decode(w)
    e = compare(f"{w.name} merged", out, lse, O, L, w.dtype, vmax_attended(w))
    # every request's completion time is recorded, inside the call
    assert np.all(fin > 0) and np.all(fin < 10_000_000_000), fin
    print(f"{w.name}: max|dO|/max|V| = {e[0]:.2e}, max|dLSE| = {e[1]:.2e}, finish_ns {fin.min()}..{fin.max()}")


def test_merged_twice_in_a_row_same_workspace():
    """The planner resets the ticket, counters and completion times on each call."""
    w = small_workload("mla", "fp8", [20_000, 50, 3], 64, 1, 576, 512, 64, 8, 1, seed=43)
    dw = build_for_test(w)
    ws = _ws(dw, 1, True)
    q = sdev.q(w.seed_val, w.B, w.hq, w.dk, 0)
    res = []
    for _ in range(2):
        out = torch.empty((w.B, w.hq, w.dv), dtype=torch.float32, device="cuda")
        lse = torch.empty((w.B, w.hq), dtype=torch.float32, device="cuda")
        fin = torch.zeros((w.B,), dtype=torch.int64, device="cuda")
        dcp.dcp_decode_merged(dw.desc, q, dw.seq_lens, out, lse, ws, finish_ns=fin)
        res.append((out.cpu().numpy(), lse.cpu().numpy(), fin.cpu().numpy()))
    torch.cuda.synchronize()
    assert dcp.dcp_get_device_status() == dcp.DCP_OK
    O, L = oracle_decode(w)
    vmax = vmax_attended(w)
    for out, lse, fin in res:
        compare("merged (repeat)", out, lse, O, L, w.dtype, vmax)
        assert np.all(fin > 0)


# ----------------------------------------------------------------------------
# several query tokens per request
# ----------------------------------------------------------------------------

def _q_multi(w, q_len, step=0):
    """bf16 q [B][q_len][hq][dk] from the generator (device) and the same bits as float64 (host)."""
    qd = sdev.q(w.seed_val, w.B, q_len * w.hq, w.dk, step).view(w.B, q_len, w.hq, w.dk)
    qh = synth.bf16_bits_to_f64(synth.q_bf16(w.seed_val, w.B, q_len * w.hq, w.dk, step)).reshape(
        w.B, q_len, w.hq, w.dk)
    return qd, qh


def _check_multi(w, q_len):
    dw = build_for_test(w)
    qd, qh = _q_multi(w, q_len)
    N, B = w.n_shards, w.B
    o = torch.full((N, B, q_len, w.hq, w.dv), float("nan"), dtype=torch.float32, device="cuda")
    l = torch.full((N, B, q_len, w.hq), float("nan"), dtype=torch.float32, device="cuda")
    dcp.dcp_decode_partial_multi(dw.desc, qd, dw.seq_lens, o, l, _ws(dw, q_len, False))
    out = torch.full((B, q_len, w.hq, w.dv), float("nan"), dtype=torch.float32, device="cuda")
    lse = torch.full((B, q_len, w.hq), float("nan"), dtype=torch.float32, device="cuda")
    dcp.dcp_decode_merged(dw.desc, qd, dw.seq_lens, out, lse, _ws(dw, q_len, True))
    torch.cuda.synchronize()
    assert dcp.dcp_get_device_status() == dcp.DCP_OK
    L = np.asarray(w.lengths)
    vmax = vmax_attended(w)
    o, l = o.cpu().numpy(), l.cpu().numpy()
    for n in range(N):
        On, Ln = oracle.decode_multi_synth(w.kind, w.dtype, w.seed_val, qh, L, w.scale, w.hkv, w.dk, w.dv,
                                           N=N, I=w.interleave, shard=n)
        compare(f"{w.name} q_len {q_len} shard {n}", o[n], l[n], On, Ln, w.dtype, vmax)
    O, Lse = oracle.decode_multi_synth(w.kind, w.dtype, w.seed_val, qh, L, w.scale, w.hkv, w.dk, w.dv)
    e = compare(f"{w.name} q_len {q_len} merged", out.cpu().numpy(), lse.cpu().numpy(), O, Lse, w.dtype, vmax)
    print(f"{w.name} q_len {q_len}: max|dO|/max|V| = {e[0]:.2e}, max|dLSE| = {e[1]:.2e}")


@pytest.mark.parametrize("dtype", ["bf16", "fp8"])
@pytest.mark.parametrize("hq,q_len,N,I", [(16, 1, 2, 1), (16, 2, 2, 1), (16, 4, 4, 1), (16, 4, 3, 16),
                                          (32, 2, 8, 1), (16, 4, 1, 1)])
def test_multi_query_mla(dtype, hq, q_len, N, I):
    # L_b = q_len (every query token's window starts at the request's first
    # position), lengths around pages, interleave blocks and chunk boundaries
    L = [q_len, q_len + 1, 63, 64, 65, 3000, 9000]
    _check_multi(small_workload("mla", dtype, L, hq, 1, 576, 512, 64, N, I, seed=51), q_len)


@pytest.mark.parametrize("hq,hkv,D,q_len,N,I", [(8, 2, 128, 4, 2, 1), (16, 2, 64, 2, 4, 16), (4, 1, 128, 4, 8, 1),
                                                (64, 4, 128, 1, 8, 128)])
def test_multi_query_gqa_tensor_core(hq, hkv, D, q_len, N, I):
    L = [q_len, 15, 16, 17, 129, 2047, 5000]
    _check_multi(small_workload("gqa", "bf16", L, hq, hkv, D, D, 16, N, I, seed=53), q_len)


def test_multi_query_unsupported_shapes():
    """Several query tokens are served by the tensor-core kernels only."""
    w = small_workload("gqa", "bf16", [40, 50], 8, 2, 64, 64, 16, 2, 1, seed=55)  # 4 heads per KV head
    dw = build_for_test(w)
    assert dcp.dcp_decode_workspace_size_ex(dw.desc, w.B, 2, dcp.DCP_DECODE_PARTIAL) == 0  # 8 MMA rows: CUDA-core path
    assert dcp.dcp_decode_workspace_size_ex(dw.desc, w.B, 4, dcp.DCP_DECODE_PARTIAL) > 0   # 16 rows: tensor cores
    qd, _ = _q_multi(w, 2)
    o = torch.empty((2, w.B, 2, w.hq, w.dv), dtype=torch.float32, device="cuda")
    l = torch.empty((2, w.B, 2, w.hq), dtype=torch.float32, device="cuda")
    ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    with pytest.raises(dcp.DcpError) as e:
        dcp.dcp_decode_partial_multi(dw.desc, qd, dw.seq_lens, o, l, ws)
    assert e.value.status == dcp.DCP_ERR_UNSUPPORTED
