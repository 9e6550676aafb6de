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


@pytest.mark.parametrize("K", [4096, 12288])
def test_activation_rows_time_out_and_recover(cuda_device, K):
    """The bulk-copy activation kernel (rows of four warps at K = 4096, the one-row-deep
    LayerNorm loop of eight warps at K = 12288): with a 1 us wait budget and the L2 flushed,
    the first rows' copies land after the budget, the kernel records a time-out, drains its
    copies in flight and returns; the next call with the normal budget is bit-identical."""
    import w8a8_int8_linear_channel_b200 as sq
    rng = np.random.default_rng(K)
    M = 4096
    h = torch.from_numpy(rng.standard_normal((M, K)).astype(np.float16)).cuda()
    g = torch.from_numpy(rng.uniform(0.5, 2.0, K).astype(np.float32)).cuda()
    b = torch.from_numpy((rng.standard_normal(K) * 0.01).astype(np.float32)).cuda()
    q_ref = torch.empty((M, K), dtype=torch.int8, device="cuda")
    s_ref = torch.empty(M, dtype=torch.float32, device="cuda")
    sq.sq_ln_quant_act(h, q_ref, s_ref, g, b)
    assert sq.sq_poll_status() == 0
    q = torch.empty_like(q_ref)
    s = torch.empty_like(s_ref)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    try:
        flush.zero_()
        sq.sq_set_wait_budget_ns(1000)
        sq.sq_ln_quant_act(h, q, s, g, b)
        torch.cuda.synchronize()
        assert sq.sq_poll_status() == 8  # SQ_ERR_TIMEOUT
    finally:
        sq.sq_set_wait_budget_ns(2_000_000_000)
    q.fill_(0)
    sq.sq_ln_quant_act(h, q, s, g, b)
    assert sq.sq_poll_status() == 0
    assert torch.equal(q, q_ref) and torch.equal(s, s_ref)
