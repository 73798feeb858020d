"""Block-table entries that name no page (marked gpu).

Every kernel family checks each block-table entry it reads against
[0, num_pages) before it issues a copy: an entry of -1 (unallocated) or one past
the pool records DCP_ERR_UNALLOCATED_PAGE in the sticky status word, and the
page's tokens are treated as absent.  These inputs are caught by the kernels'
own bounds checks, so nothing out of bounds is ever read.  Here request 0 gets
one entry of each kind; the call must report the status, keep every output
finite, and leave the other requests exactly as the oracle computes them."""
import numpy as np
import pytest

import sequence_sharded_paged_b200 as dcp

from gpu_util import build_for_test, compare, oracle_decode, run_step, small_workload, vmax_attended

pytestmark = pytest.mark.gpu

# kind, dtype, hq, hkv, dk, dv, page, N, I, lengths (request 0 spans several pages on shards 0 and 1)
CASES = [
    ("gqa", "bf16", 8, 2, 64, 64, 16, 2, 1, [5000, 300, 41]),           # CUDA-core GQA
    ("gqa", "bf16", 64, 4, 128, 128, 16, 4, 16, [6000, 129, 7]),        # tensor-core GQA
    ("mla", "bf16", 16, 1, 576, 512, 64, 2, 1, [9000, 65, 3]),          # tcgen05 bf16
    ("mla", "fp8", 64, 1, 576, 512, 64, 8, 1, [30000, 200, 5]),         # tcgen05 fp8
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c[0]}-{c[1]}-hq{c[2]}")
def test_bad_block_table_entries_are_reported_and_skipped(case):
    kind, dtype, hq, hkv, dk, dv, P, N, I, L = case
    w = small_workload(kind, dtype, L, hq, hkv, dk, dv, P, N, I, seed=73)
    dw = build_for_test(w)
    dw.block_tables[0, 0, 1] = dw.num_pages + 7     # past the pool
    dw.block_tables[1, 0, 0] = -1                   # unallocated
    o_part, lse, out, lse_out, status = run_step(dw)
    assert status == dcp.DCP_ERR_UNALLOCATED_PAGE
    assert np.all(np.isfinite(o_part)) and np.all(np.isfinite(out))
    others = list(range(1, w.B))
    O, Lf = oracle_decode(w, req_list=others)
    compare(f"{w.name} untouched requests", out[others], lse_out[others], O[others], Lf[others], w.dtype,
            vmax_attended(w, others))
    # request 0 lost exactly two pages' worth of tokens, so its LSE cannot exceed the full one
    _, L0 = oracle_decode(w, req_list=[0])
    assert np.all(lse_out[0] <= L0[0] + 1e-3)
