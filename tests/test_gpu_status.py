"""Failure detection on the GPU without a fault: bounded waits and device-side input checks
report through the device status word; the context stays usable afterwards."""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import check_tol, dev

pytestmark = pytest.mark.gpu
moe = pytest.importorskip("quantized_mixture_experts_softmax_b200")


def test_bounded_wait_times_out_and_reports():
    moe.moe_get_device_status()
    moe.moe_debug_wait_timeout(2_000_000)  # 2 ms on a barrier nothing arrives on
    assert moe.moe_get_device_status() == moe.MOE_ERR_TIMEOUT
    assert moe.moe_get_device_status() == 0
    # the context is still healthy: a normal call works and reports nothing
    lg = np.random.default_rng(0).normal(size=(4, 16)).astype(np.float32)
    ids, _ = moe.moe_route(dev(lg), 2)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == 0
    assert ids.shape == (4, 2)


def test_bad_offsets_in_grouped_gemm_are_flagged_not_used():
    a = torch.zeros(16, 128, dtype=torch.bfloat16, device="cuda")
    w_q = torch.zeros(2, 128, 16, dtype=torch.int32, device="cuda")
    w_s = torch.zeros(2, 128, 4, dtype=torch.bfloat16, device="cuda")
    off = dev(np.array([0, 20, 16], np.int32))  # expert 0 reaches past M: flagged and skipped
    moe.moe_get_device_status()
    moe.moe_w4a16_gemm(a, w_q, w_s, off, out_fp32=True)
    assert moe.moe_get_device_status() == moe.MOE_ERR_DEVICE_CHECK


def test_bad_offsets_with_k_splits_leave_the_flagged_rows_untouched():
    """M=2 rows against [7168 x 512] weights has 4 work items, so the K range is split and the
    fp32 partial sums are reduced by a second kernel.  Expert 1's range reaches past M: it is
    flagged and skipped, so its row must keep what the caller put there (the reduction must not
    fill it from partial sums nobody wrote), while expert 0's row is computed normally."""
    M, K, N = 2, 7168, 512
    a, w_q, w_s = synth.gemm_operands(5, M, K, N)
    w_q2, w_s2 = np.concatenate([w_q, w_q]), np.concatenate([w_s, w_s])
    off = np.array([0, 1, 5], np.int32)
    out = torch.full((M, N), 7.0, dtype=torch.float32, device="cuda")
    moe.moe_get_device_status()
    moe.moe_w4a16_gemm(dev(a, torch.bfloat16), dev(w_q2), dev(w_s2, torch.bfloat16), dev(off), out=out,
                       out_fp32=True)
    assert moe.moe_get_device_status() == moe.MOE_ERR_DEVICE_CHECK
    got = out.cpu().numpy()
    assert np.all(got[1] == 7.0)
    ref = oracle.w4a16_gemm(a[:1], True, w_q, w_s, np.array([0, 1], np.int32))
    check_tol(got[:1], ref, what="expert 0 row")
