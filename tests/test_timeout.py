"""Bounded device waits: a wait that nothing completes runs out, the kernel
records a timeout and returns, and the context stays usable."""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu


def test_wait_runs_out_and_reports_timeout(cuda_device):
    import w8a8_int8_linear_channel_b200 as sq
    assert sq.sq_poll_status() == 0
    sq.sq_selftest_wait_timeout(2_000_000)  # 2 ms budget
    assert sq.sq_poll_status() == 8  # SQ_ERR_TIMEOUT, cleared by the poll
    assert sq.sq_poll_status() == 0
    # the next call works
    rng = np.random.default_rng(0)
    xq = rng.integers(-127, 128, (8, 64)).astype(np.int8)
    wq = rng.integers(-127, 128, (40, 64)).astype(np.int8)
    acc = torch.empty((8, 40), dtype=torch.int32, device="cuda")
    ws = sq.new_workspace(8, 40, 64)
    sq.sq_w8a8_gemm_s32(torch.from_numpy(xq).cuda(), torch.from_numpy(wq).cuda(), acc, workspace=ws)
    assert sq.sq_poll_status() == 0
    assert np.array_equal(acc.cpu().numpy(), oracle.int_gemm(xq, wq))


def test_layer_reset_after_timed_out_decode_forward(cuda_device):
    """A decode-sized forward whose bounded waits run out may leave the layer's stream-K
    counters raised; reset_workspaces puts them back to zero and the next forward is exact."""
    import w8a8_int8_linear_channel_b200 as sq
    rng = np.random.default_rng(5)
    N, K, M = 2048, 8192, 8
    w = torch.from_numpy((rng.standard_normal((N, K)) * 0.02).astype(np.float16)).cuda()
    calib = torch.from_numpy(rng.standard_normal((64, K)).astype(np.float16)).cuda()
    h = torch.from_numpy(rng.standard_normal((M, K)).astype(np.float16)).cuda()
    layer = sq.SmoothQuantLinear.from_float(w, calib, 0.5)
    y_ref = layer(h).clone()
    assert sq.sq_poll_status() == 0
    try:
        sq.sq_set_wait_budget_ns(1000)
        layer(h)
        assert sq.sq_poll_status() == 8
    finally:
        sq.sq_set_wait_budget_ns(2_000_000_000)
    layer.reset_workspaces()
    for _ in range(2):
        assert torch.equal(layer(h), y_ref)
    assert sq.sq_poll_status() == 0
