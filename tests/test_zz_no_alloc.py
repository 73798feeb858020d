"""dcp_decode_partial_noalloc: the decode on the library's built-in scratch.

Kept in a file of its own, collected last, so that it runs both alone and after
every other test has used the library (the scratch then holds an earlier
call's plan and partials, which the plan kernel must clear or overwrite).
Where the no-alloc plan equals dcp_decode_partial's, the two entry points must
agree bit for bit, on two calls in a row (dcp_decode_partial is held to the
oracle by the parity tests).  Where the scratch forces a smaller plan, the
results are compared with the oracle directly."""
from __future__ import annotations

import os
import re

import numpy as np
import pytest
import torch

import sequence_sharded_paged_b200 as dcp
import synth.device as sdev
from gpu_util import build_for_test, compare, oracle_decode, small_workload, vmax_attended

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "dcp.h")


def test_scratch_size_matches_header():
    text = open(HEADER).read()
    m = re.search(r"#define DCP_STATIC_SCRATCH_BYTES \(\(size_t\)(\d+) << (\d+)\)", text)
    assert m, "DCP_STATIC_SCRATCH_BYTES not found in dcp.h"
    assert int(m.group(1)) << int(m.group(2)) == dcp.DCP_STATIC_SCRATCH_BYTES


# (kind, dtype, hq, hkv, dk, dv, page_size, N, I, lengths)
CASES = [
    ("gqa", "bf16", 32, 2, 128, 128, 16, 4, 16, [1, 0, 300, 4097, 2500, 77]),
    ("mla", "bf16", 16, 1, 576, 512, 64, 2, 64, [5000, 1, 130, 0, 2049]),
    ("mla", "fp8", 32, 1, 576, 512, 64, 4, 1, [900, 3333, 64]),
    # the standard workspace of 64 heads exceeds the scratch: the shrunk plan runs
    ("mla", "bf16", 64, 1, 576, 512, 64, 8, 16, [7000, 12, 4096]),
]


@pytest.mark.gpu
@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c[0]}-{c[1]}-hq{c[2]}-N{c[7]}")
def test_noalloc_matches_decode_partial(case):
    kind, dtype, hq, hkv, dk, dv, P, N, I, lengths = case
    w = small_workload(kind, dtype, lengths, hq, hkv, dk, dv, P, N, I, seed=31)
    dw = build_for_test(w)
    q = sdev.q(w.seed_val, w.B, w.hq, w.dk, 0)
    shape_o, shape_l = (N, w.B, hq, dv), (N, w.B, hq)
    o_ref = torch.empty(shape_o, dtype=torch.float32, device="cuda")
    l_ref = torch.empty(shape_l, dtype=torch.float32, device="cuda")
    dcp.dcp_decode_partial(dw.desc, q, dw.seq_lens, o_ref, l_ref, dw.ws)
    outs = []
    for _ in range(2):
        o = torch.full(shape_o, float("nan"), dtype=torch.float32, device="cuda")
        l = torch.full(shape_l, float("nan"), dtype=torch.float32, device="cuda")
        dcp.dcp_decode_partial_noalloc(dw.desc, q, dw.seq_lens, o, l)
        outs.append((o, l))
    torch.cuda.synchronize()
    assert dcp.dcp_get_device_status() == dcp.DCP_OK
    # every chunk of these sizes is the planner's minimum chunk under either
    # split-slot bound, so the units, and with them the results, are the same
    for o, l in outs:
        assert torch.equal(o, o_ref)
        assert torch.equal(l, l_ref)
    assert np.isfinite(o_ref.cpu().numpy()).all()


@pytest.mark.gpu
@pytest.mark.parametrize("N", [1, 8])
def test_noalloc_rejects_fp8_high_concurrency_shape(N):
    """The fp8 MLA shape with B = 512 requests and 64 heads needs more than the
    built-in scratch at any N: the query split into two e4m3 terms alone is
    B * (128 * 576 + 256) bytes (37.9 MB) and the smallest split area 39 MB.
    The call must say so on the host and launch nothing."""
    B, hq, P = 512, 64, 64
    dev = "cuda"
    lat = torch.zeros((1, P, 576), dtype=torch.uint8, device=dev)
    scales = torch.ones((1, P), dtype=torch.float32, device=dev)
    bt = torch.zeros((N, B, 1), dtype=torch.int32, device=dev)
    desc = dcp.make_cache_desc(kind=dcp.DCP_MLA, dtype=dcp.DCP_FP8_E4M3, n_shards=N, interleave=1, page_size=P,
                               num_pages=1, hq=hq, hkv=1, dk=576, dv=512, scale=0.072, batch=B, block_tables=bt,
                               k_pages=lat, kv_scales=scales)
    # full-size inputs and outputs, so that nothing could be read or written out of bounds
    q = torch.zeros((B, hq, 576), dtype=torch.bfloat16, device=dev)
    seq_lens = torch.zeros((B,), dtype=torch.int32, device=dev)
    o = torch.empty((N, B, hq, 512), dtype=torch.float32, device=dev)
    lse = torch.empty((N, B, hq), dtype=torch.float32, device=dev)
    assert dcp.dcp_decode_workspace_size(desc, B) > dcp.DCP_STATIC_SCRATCH_BYTES
    with pytest.raises(dcp.DcpError) as ei:
        dcp.dcp_decode_partial_noalloc(desc, q, seq_lens, o, lse)
    assert ei.value.status == dcp.DCP_ERR_WORKSPACE_TOO_SMALL
    torch.cuda.synchronize()
    assert dcp.dcp_get_device_status() == dcp.DCP_OK


@pytest.mark.gpu
def test_noalloc_shrunk_plan_against_oracle():
    """64 heads, 8 shards and 380k tokens: the standard plan (1,184 target units,
    2,048-token chunks) needs 311 MB of split area, so the no-alloc plan drops to
    one unit per CTA and cuts chunks of ~2,600 tokens instead.  Different units
    give different rounding, so this case is held to the oracle's bar rather than
    to bit-equality with dcp_decode_partial."""
    w = small_workload("mla", "bf16", [200_000, 180_000, 3], 64, 1, 576, 512, 64, 8, 1, seed=37)
    dw = build_for_test(w)
    q = sdev.q(w.seed_val, w.B, w.hq, w.dk, 0)
    N = w.n_shards
    o = torch.empty((N, w.B, w.hq, w.dv), dtype=torch.float32, device="cuda")
    lse = torch.empty((N, w.B, w.hq), dtype=torch.float32, device="cuda")
    out = torch.empty((w.B, w.hq, w.dv), dtype=torch.float32, device="cuda")
    lse_out = torch.empty((w.B, w.hq), dtype=torch.float32, device="cuda")
    assert dcp.dcp_decode_workspace_size(dw.desc, w.B) > dcp.DCP_STATIC_SCRATCH_BYTES
    for _ in range(2):
        dcp.dcp_decode_partial_noalloc(dw.desc, q, dw.seq_lens, o, lse)
        dcp.dcp_merge(o, lse, out, lse_out)
        torch.cuda.synchronize()
        assert dcp.dcp_get_device_status() == dcp.DCP_OK
        vmax = vmax_attended(w)
        for n in range(N):
            O_n, L_n = oracle_decode(w, shard=n)
            compare(f"no-alloc shard {n}", o[n].cpu().numpy(), lse[n].cpu().numpy(), O_n, L_n, w.dtype, vmax)
        O, L = oracle_decode(w)
        compare("no-alloc merged", out.cpu().numpy(), lse_out.cpu().numpy(), O, L, w.dtype, vmax)
