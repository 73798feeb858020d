"""Failure detection on the GPU without a fault (marked gpu).

The persistent decode kernels wait on mbarriers with a time limit; a wait that
runs out records DCP_ERR_TIMEOUT in the sticky status word, raises the CTA's
abort flag and lets the kernel return.  dcp_selftest_bounded_wait runs that
branch through the same wait code, on a barrier that nothing arrives on (no
trap, no bad address, no endless loop).  The test checks what the host reads
afterwards, and that the context still decodes correctly."""
import pytest
import torch

import sequence_sharded_paged_b200 as dcp

from gpu_util import build_for_test, compare, oracle_decode, run_step, small_workload, vmax_attended

pytestmark = pytest.mark.gpu

WAIT_LIMIT_NS = 4_000_000_000  # the kernels' wait limit


def test_bounded_wait_gives_up_and_reports_timeout():
    dcp.dcp_get_device_status()  # clear
    res = torch.full((4,), -1, dtype=torch.int64, device="cuda")
    dcp.dcp_selftest_bounded_wait(res)
    torch.cuda.synchronize()
    completed, abort_flag, waited_ns = res[:3].cpu().tolist()
    assert dcp.dcp_get_device_status() == dcp.DCP_ERR_TIMEOUT
    assert dcp.dcp_get_device_status() == dcp.DCP_OK   # reading clears it
    assert completed == 0
    assert abort_flag == 1
    assert WAIT_LIMIT_NS <= waited_ns < 10 * WAIT_LIMIT_NS


def test_context_still_decodes_after_a_timeout():
    res = torch.zeros((4,), dtype=torch.int64, device="cuda")
    dcp.dcp_selftest_bounded_wait(res)
    assert dcp.dcp_get_device_status() == dcp.DCP_ERR_TIMEOUT
    w = small_workload("mla", "fp8", [3000, 65, 1], 64, 1, 576, 512, 64, 4, 1, seed=71)
    dw = build_for_test(w)
    _, _, out, lse_out, status = run_step(dw)
    assert status == dcp.DCP_OK
    O, L = oracle_decode(w)
    compare("decode after a timeout", out, lse_out, O, L, "fp8", vmax_attended(w))
