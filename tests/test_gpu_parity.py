"""GPU parity of libdcp against the float64 oracle (marked gpu).

Integer work (shard counts, shard map, block-table slots, appended bytes,
fp8 codes and scales) must match bit for bit.  Attention outputs must satisfy
max|O - O_oracle| <= 2e-3 max|V| (bf16 cache) or 2e-2 max|V| (fp8 cache), and
|LSE - LSE_oracle| <= 1e-3, per shard partial and after the merge.
"""
import numpy as np
import pytest
import torch

import oracle
import sequence_sharded_paged_b200 as dcp
import synth
import synth.device as sdev
from sequence_sharded_paged_b200 import workload as wl

from gpu_util import (build_for_test, compare, oracle_decode, run_step, small_workload, vmax_attended)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clear_status():
    dcp.dcp_get_device_status()
    yield


# ----------------------------------------------------------------------------
# generator (device bits == host bits)
# ----------------------------------------------------------------------------

def test_device_generator_matches_host():
    q = sdev.q(2001, 3, 8, 64, step=5).view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(q, synth.q_bf16(2001, 3, 8, 64, step=5))
    req = torch.tensor([0, 1, 1, 2], dtype=torch.int32, device="cuda")
    pos = torch.tensor([0, 5, 999_999, 77], dtype=torch.int32, device="cuda")
    rows = sdev.kv_rows(9, synth.T_LATENT, req, pos, 1, 576).view(torch.int16).cpu().numpy().view(np.uint16)
    for i in range(4):
        ref = synth.kv_rows_bf16(9, synth.T_LATENT, int(req[i]), [int(pos[i])], 1, 576)
        assert np.array_equal(rows[i], ref[0])


# ----------------------------------------------------------------------------
# shard map (bit-exact)
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("N,I", [(1, 1), (2, 1), (3, 7), (8, 1), (8, 16), (8, 128), (4, 50_000)])
def test_shard_counts_bit_exact(N, I):
    rng = np.random.default_rng(N * 7 + I)
    L = np.concatenate([[0, 1, I - 1, I, I * N - 1, I * N, I * N + 1], rng.integers(0, 1_200_000, 50)])
    L = np.maximum(L, 0)
    gpu = wl.gpu_shard_counts(L, N, I)
    assert np.array_equal(gpu, oracle.shard_counts(L, N, I))


@pytest.mark.parametrize("N,I,P", [(2, 1, 16), (8, 128, 16), (3, 5, 16), (4, 64, 64), (8, 1, 64)])
def test_shard_map_bit_exact(N, I, P):
    rng = np.random.default_rng(N + I + P)
    B = 6
    L = rng.integers(1, 3000, size=B)
    counts = oracle.shard_counts(L, N, I)
    need = (counts + P - 1) // P
    bt, num_pages = synth.deal_block_tables(5, need, slack_pages=2)
    # knock out one page: positions mapping there must come back as -1
    bt[N - 1, B - 1, 0] = -1
    pos = np.concatenate([np.arange(L[b]) for b in range(B)]).astype(np.int32)
    req = np.concatenate([np.full(L[b], b) for b in range(B)]).astype(np.int32)
    st_o, rank_o, local_o, slot_o = oracle.shard_map(pos, req, N, I, P, bt, num_pages)
    bt_d = torch.as_tensor(bt, device="cuda")
    desc = dcp.make_cache_desc(kind=dcp.DCP_GQA, dtype=dcp.DCP_BF16, n_shards=N, interleave=I, page_size=P,
                               num_pages=num_pages, hq=8, hkv=2, dk=64, dv=64, scale=0.125, batch=B, block_tables=bt_d)
    pos_d = torch.as_tensor(pos, device="cuda")
    req_d = torch.as_tensor(req, device="cuda")
    rank = torch.empty_like(pos_d)
    local = torch.empty_like(pos_d)
    slot = torch.empty(pos.size, dtype=torch.int64, device="cuda")
    dcp.dcp_shard_map(desc, pos_d, req_d, rank, local, slot)
    status = dcp.dcp_get_device_status()
    assert np.array_equal(rank.cpu().numpy(), rank_o)
    assert np.array_equal(local.cpu().numpy(), local_o)
    assert np.array_equal(slot.cpu().numpy(), slot_o)
    assert (status == dcp.DCP_ERR_UNALLOCATED_PAGE) == (st_o == oracle.ORC_ERR_UNALLOCATED)


# ----------------------------------------------------------------------------
# append (bit-exact bytes in the owner's page)
# ----------------------------------------------------------------------------

def _slots(w, dw, b, positions):
    bt = dw.block_tables.cpu().numpy()
    pos = np.asarray(positions, np.int32)
    st, rank, local, slot = oracle.shard_map(pos, np.full(pos.size, b, np.int32), w.n_shards, w.interleave,
                                             w.page_size, bt, dw.num_pages)
    assert st == oracle.ORC_OK
    return slot


@pytest.mark.parametrize("kind,dtype", [("gqa", "bf16"), ("mla", "bf16"), ("mla", "fp8")])
def test_append_writes_owner_page_bit_exact(kind, dtype):
    if kind == "gqa":
        w = small_workload("gqa", "bf16", [37, 300, 5], 8, 2, 64, 64, 16, 3, 4)
    else:
        w = small_workload("mla", dtype, [70, 129, 1], 16, 1, 576, 512, 64, 2, 3)
    dw = build_for_test(w)
    assert dcp.dcp_get_device_status() == dcp.DCP_OK
    P = w.page_size
    for b in range(w.B):
        pos = np.arange(w.lengths[b])
        slot = _slots(w, dw, b, pos)
        page, off = slot // P, slot % P
        if kind == "gqa":
            K = dw.k_pages.view(torch.int16).cpu().numpy().view(np.uint16)
            V = dw.v_pages.view(torch.int16).cpu().numpy().view(np.uint16)
            refK = synth.kv_rows_bf16(w.seed_val, synth.T_K, b, pos, w.hkv, w.dk)
            refV = synth.kv_rows_bf16(w.seed_val, synth.T_V, b, pos, w.hkv, w.dv)
            for g in range(w.hkv):
                assert np.array_equal(K[page, g, off], refK[:, g])
                assert np.array_equal(V[page, g, off], refV[:, g])
        else:
            ref = synth.kv_rows_bf16(w.seed_val, synth.T_LATENT, b, pos, 1, 576)[:, 0]
            if dtype == "bf16":
                lat = dw.k_pages.view(torch.int16).cpu().numpy().view(np.uint16)
                assert np.array_equal(lat[page, off], ref)
            else:
                lat = dw.k_pages.cpu().numpy()
                sc = dw.kv_scales.cpu().numpy()
                for i, p in enumerate(pos):
                    codes, s = oracle.quantize_row_e4m3(ref[i])
                    assert np.array_equal(lat[page[i], off[i]], codes), (b, p)
                    assert sc[page[i], off[i]] == np.float32(s), (b, p)


def test_append_unallocated_page_reports_status():
    w = small_workload("gqa", "bf16", [40], 4, 1, 64, 64, 16, 2, 1)
    dw = build_for_test(w, fill=False)
    bt = dw.block_tables.clone()
    bt[1, 0, 0] = -1
    desc = dcp.make_cache_desc(kind=dcp.DCP_GQA, dtype=dcp.DCP_BF16, n_shards=2, interleave=1, page_size=16,
                               num_pages=dw.num_pages, hq=4, hkv=1, dk=64, dv=64, scale=0.1, batch=1, block_tables=bt,
                               k_pages=dw.k_pages, v_pages=dw.v_pages)
    pos = torch.tensor([0, 1, 2, 3], dtype=torch.int32, device="cuda")
    k, v = sdev.gqa_rows(w.seed_val, torch.zeros(4, dtype=torch.int32, device="cuda"), pos, 1, 64)
    dcp.dcp_kv_append(desc, None, pos, k, v)
    assert dcp.dcp_get_device_status() == dcp.DCP_ERR_UNALLOCATED_PAGE
    assert dcp.dcp_get_device_status() == dcp.DCP_OK  # read clears


# ----------------------------------------------------------------------------
# decode: per-shard partials and merged output against the oracle
# ----------------------------------------------------------------------------

def _check_decode(w, dw=None, req_list=None, vmax=None):
    dw = dw or build_for_test(w)
    o_part, lse, out, lse_out, status = run_step(dw)
    assert status == dcp.DCP_OK, dcp.status_string(status)
    reqs = list(range(w.B)) if req_list is None else list(req_list)
    vmax = vmax if vmax is not None else vmax_attended(w, reqs)
    worst = (0.0, 0.0)
    for n in range(w.n_shards):
        O_n, L_n = oracle_decode(w, shard=n, req_list=reqs)
        e = compare(f"shard {n}", o_part[n][reqs], lse[n][reqs], O_n[reqs], L_n[reqs], w.dtype, vmax)
        worst = (max(worst[0], e[0]), max(worst[1], e[1]))
    O, L = oracle_decode(w, req_list=reqs)
    e = compare("merged", out[reqs], lse_out[reqs], O[reqs], L[reqs], w.dtype, vmax)
    print(f"{w.name}: max|dO|/max|V| = {max(worst[0], e[0]):.2e}, max|dLSE| = {max(worst[1], e[1]):.2e}")
    return dw


def test_decode_config1_gqa_tiny():
    _check_decode(synth.workload(1))


def test_decode_config2_mla_v2_lite():
    _check_decode(synth.workload(2))


@pytest.mark.parametrize("N,I", [(1, 1), (2, 1), (3, 16), (8, 5)])
def test_decode_gqa_ragged(N, I):
    # lengths around page, interleave and chunk boundaries; some shards empty
    L = [1, 15, 16, 17, I * N - 1, I * N + 1, 2500, 700]
    _check_decode(small_workload("gqa", "bf16", L, 16 if N == 3 else 8, 2, 128 if N > 2 else 64,
                                 128 if N > 2 else 64, 16, N, I))


@pytest.mark.parametrize("dtype", ["bf16", "fp8"])
@pytest.mark.parametrize("N,I", [(1, 1), (2, 1), (4, 16), (8, 64)])
def test_decode_mla_ragged(dtype, N, I):
    L = [1, 63, 64, 65, 3000, 1200]
    _check_decode(small_workload("mla", dtype, L, 64, 1, 576, 512, 64, N, I))


def test_decode_mla_many_chunks():
    # one long request, split into many chunks per shard (split-KV reduce path)
    _check_decode(small_workload("mla", "bf16", [40_000, 3], 16, 1, 576, 512, 64, 2, 1))


def test_decode_unallocated_page_is_reported_not_fatal():
    w = small_workload("gqa", "bf16", [300, 40], 8, 2, 64, 64, 16, 2, 1)
    dw = build_for_test(w)
    dw.block_tables[0, 0, 3] = -1
    o_part, lse, out, lse_out, status = run_step(dw)
    assert status == dcp.DCP_ERR_UNALLOCATED_PAGE
    assert np.all(np.isfinite(out))


# ----------------------------------------------------------------------------
# merge kernel
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("N,B,H,Dv", [(1, 3, 4, 64), (2, 5, 16, 512), (8, 7, 64, 128), (3, 2, 2, 4)])
def test_merge_kernel(N, B, H, Dv):
    rng = np.random.default_rng(N * B)
    Op = rng.standard_normal((N, B, H, Dv)).astype(np.float32)
    Lp = (rng.standard_normal((N, B, H)) * 3).astype(np.float32)
    Lp[rng.random((N, B, H)) < 0.2] = -np.inf
    Lp[:, 0, 0] = -np.inf
    Op[np.isneginf(Lp)] = 0
    O_ref, L_ref = oracle.merge(Op.astype(np.float64), Lp.astype(np.float64))
    out = torch.empty((B, H, Dv), dtype=torch.float32, device="cuda")
    lo = torch.empty((B, H), dtype=torch.float32, device="cuda")
    dcp.dcp_merge(torch.as_tensor(Op, device="cuda"), torch.as_tensor(Lp, device="cuda"), out, lo)
    torch.cuda.synchronize()
    out = out.cpu().numpy()
    lo = lo.cpu().numpy()
    assert np.array_equal(np.isneginf(lo), np.isneginf(L_ref))
    fin = ~np.isneginf(L_ref)
    assert np.abs(lo[fin] - L_ref[fin]).max() <= 1e-5
    assert np.abs(out - O_ref).max() <= 1e-5 * max(1.0, np.abs(Op).max())


# ----------------------------------------------------------------------------
# host-side validation through the C ABI
# ----------------------------------------------------------------------------

def test_invalid_arguments_raise():
    w = small_workload("gqa", "bf16", [10], 8, 2, 64, 64, 16, 2, 1)
    dw = build_for_test(w)
    q = sdev.q(w.seed_val, 1, 8, 64)
    o = torch.empty((2, 1, 8, 64), dtype=torch.float32, device="cuda")
    lse = torch.empty((2, 1, 8), dtype=torch.float32, device="cuda")
    with pytest.raises(dcp.DcpError) as e:
        dcp.dcp_decode_partial(dw.desc, q, dw.seq_lens, o, lse, dw.ws[:16])
    assert e.value.status == dcp.DCP_ERR_WORKSPACE_TOO_SMALL
    bad = dcp.CacheDesc.from_buffer_copy(dw.desc)
    bad.page_size = 8
    with pytest.raises(dcp.DcpError) as e:
        dcp.dcp_decode_partial(bad, q, dw.seq_lens, o, lse, dw.ws)
    assert e.value.status == dcp.DCP_ERR_UNSUPPORTED
    with pytest.raises(dcp.DcpError) as e:
        dcp.dcp_merge(o, lse, torch.empty((1, 8, 64), device="cuda")[:, :, 1:], None)
    assert e.value.status in (dcp.DCP_ERR_MISALIGNED, dcp.DCP_ERR_INVALID_ARG)


# ----------------------------------------------------------------------------
# GQA with a 16-head group: the tensor-core kernel
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("hkv,D,N,I", [(4, 128, 8, 128), (4, 128, 3, 16), (1, 128, 2, 1), (2, 64, 4, 5),
                                       (8, 128, 2, 16), (4, 64, 1, 1)])
def test_decode_gqa_group16_tensor_core(hkv, D, N, I):
    L = [1, 15, 16, 17, 129, 2047, 5000, 333]
    _check_decode(small_workload("gqa", "bf16", L, 16 * hkv, hkv, D, D, 16, N, I))


def test_decode_gqa_group16_page64():
    _check_decode(small_workload("gqa", "bf16", [70, 64, 1000, 3], 64, 4, 128, 128, 64, 2, 64))


def test_decode_mla_page16_cuda_core_path():
    # page size 16 is served by the CUDA-core MLA kernel
    _check_decode(small_workload("mla", "bf16", [1, 200, 3000], 16, 1, 576, 512, 16, 2, 1))
    _check_decode(small_workload("mla", "fp8", [17, 900], 32, 1, 576, 512, 16, 3, 4))


@pytest.mark.parametrize("hq", [16, 32, 64])
@pytest.mark.parametrize("dtype", ["bf16", "fp8"])
def test_decode_mla_heads(hq, dtype):
    _check_decode(small_workload("mla", dtype, [31, 32, 33, 64, 97, 4100], hq, 1, 576, 512, 64, 2, 1))
