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
