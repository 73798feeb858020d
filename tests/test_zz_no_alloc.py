"""dcp_decode_partial_noalloc: the decode on the library's built-in scratch.

Kept in a file of its own, collected last, so that it runs both alone and after
every other test has used the library (the scratch then holds an earlier
call's plan and partials, which the plan kernel must clear or overwrite).
The expected values are dcp_decode_partial's on its own workspace, which the
parity tests compare with the oracle; here the two entry points must agree bit
for bit, on two calls in a row."""
from __future__ import annotations

import os
import re

import numpy as np
import pytest
import torch

import sequence_sharded_paged_b200 as dcp
import synth.device as sdev
from gpu_util import build_for_test, small_workload

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
def test_noalloc_rejects_work_beyond_scratch():
    # per-shard done counters alone: N * B * hq * 4 bytes > DCP_STATIC_SCRATCH_BYTES
    N, hq, hkv, D, P = 8, 8, 1, 64, 16
    B = dcp.DCP_STATIC_SCRATCH_BYTES // (N * hq * 4) + 1000
    dev = "cuda"
    k_pages = torch.zeros((1, hkv, P, D), dtype=torch.bfloat16, device=dev)
    v_pages = torch.zeros_like(k_pages)
    bt = torch.zeros((N, B, 1), dtype=torch.int32, device=dev)
    desc = dcp.make_cache_desc(kind=dcp.DCP_GQA, dtype=dcp.DCP_BF16, n_shards=N, interleave=1, page_size=P,
                               num_pages=1, hq=hq, hkv=hkv, dk=D, dv=D, scale=0.125, batch=B, block_tables=bt,
                               k_pages=k_pages, v_pages=v_pages)
    q = torch.zeros((B, hq, D), dtype=torch.bfloat16, device=dev)
    seq_lens = torch.zeros((B,), dtype=torch.int32, device=dev)
    o = torch.empty((N, B, hq, D), dtype=torch.float32, device=dev)
    lse = torch.empty((N, B, hq), dtype=torch.float32, device=dev)
    with pytest.raises(dcp.DcpError) as ei:
        dcp.dcp_decode_partial_noalloc(desc, q, seq_lens, o, lse)
    assert ei.value.status == dcp.DCP_ERR_WORKSPACE_TOO_SMALL
    torch.cuda.synchronize()
    assert dcp.dcp_get_device_status() == dcp.DCP_OK
