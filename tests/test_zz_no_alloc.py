"""The allocation-free decode linear, sq_w8a8_linear_noalloc.

Callers such as a plug-in inside another runtime (which owns every device
allocation and hands over only inputs and outputs) or a latency-critical path
(where cudaMalloc may synchronize the device) cannot provide a workspace.
This entry point uses the library's own fixed scratch array instead; its
output must match the regular entry point, which uses a caller workspace, on
consecutive calls (the array keeps the previous call's contents, so every call
must start from cleared counters).  This file is collected last so that a run
stopping at the first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from gpu_util import bits_equal, f16_within

pytestmark = pytest.mark.gpu


def _inputs(rng, M, N, K, with_bias):
    xq = torch.from_numpy(rng.integers(-127, 128, (M, K)).astype(np.int8)).cuda()
    wq = torch.from_numpy(rng.integers(-127, 128, (N, K)).astype(np.int8)).cuda()
    sx = torch.from_numpy(rng.uniform(1e-4, 0.1, M).astype(np.float32)).cuda()
    sw = torch.from_numpy(rng.uniform(1e-4, 0.1, N).astype(np.float32)).cuda()
    bias = torch.from_numpy((rng.standard_normal(N) * 0.5).astype(np.float16)).cuda() if with_bias else None
    return xq, sx, wq, sw, bias


def _noalloc_via_c_abi(lib, xq, sx, wq, sw, bias, y):
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    M, K = xq.shape
    N = wq.shape[0]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.sq_w8a8_linear_noalloc(p(xq), p(sx), p(wq), p(sw), p(bias), p(y), M, N, K, stream)


def test_noalloc_matches_workspace_entry_point_on_consecutive_calls(cuda_device):
    import w8a8_int8_linear_channel_b200 as sq
    lib = sq._L
    rng = np.random.default_rng(20261202)
    # two calls in a row with different shapes: the second one runs on the
    # scratch array exactly as the first left it
    for (M, N, K, with_bias) in [(8, 1000, 4112, True), (20, 256, 16384, False)]:
        xq, sx, wq, sw, bias = _inputs(rng, M, N, K, with_bias)
        y_ref = torch.empty((M, N), dtype=torch.float16, device="cuda")
        ws = sq.new_workspace(M, N, K)
        sq.sq_w8a8_linear(xq, sx, wq, sw, y_ref, bias, workspace=ws)
        y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
        assert _noalloc_via_c_abi(lib, xq, sx, wq, sw, bias, y) == 0
        assert sq.sq_poll_status() == 0
        got, ref = y.cpu().numpy(), y_ref.cpu().numpy()
        assert f16_within(got, ref)
        assert bits_equal(got, ref)


def test_noalloc_rejects_shapes_beyond_its_scratch(cuda_device):
    import w8a8_int8_linear_channel_b200 as sq
    lib = sq._L
    fake = ctypes.c_void_p(0x10000)
    # too many tokens for the decode kernel
    assert lib.sq_w8a8_linear_noalloc(fake, fake, fake, fake, None, fake, 33, 128, 128, None) == 3
    # more output channels than the fixed array has counters for (4096 tiles of 128)
    assert lib.sq_w8a8_linear_noalloc(fake, fake, fake, fake, None, fake, 8, 4096 * 128 + 1, 128, None) == 5


def test_noalloc_calls_allocate_no_device_memory(cuda_device):
    """The defining property: once the library is loaded and the call has run once per shape
    (module and scratch-address set-up), further calls change neither the device's free memory
    nor torch's allocations."""
    import w8a8_int8_linear_channel_b200 as sq
    lib = sq._L
    rng = np.random.default_rng(7)
    cases = []
    for (M, N, K) in [(1, 4096, 4096), (16, 1000, 2064), (32, 12288, 512)]:
        xq, sx, wq, sw, bias = _inputs(rng, M, N, K, True)
        y = torch.empty((M, N), dtype=torch.float16, device="cuda")
        cases.append((xq, sx, wq, sw, bias, y))
        assert _noalloc_via_c_abi(lib, xq, sx, wq, sw, bias, y) == 0  # warm-up of this shape
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    alloc0 = torch.cuda.memory_allocated()
    for _ in range(3):
        for xq, sx, wq, sw, bias, y in cases:
            assert _noalloc_via_c_abi(lib, xq, sx, wq, sw, bias, y) == 0
    torch.cuda.synchronize()
    assert sq.sq_poll_status() == 0
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
    assert torch.cuda.memory_allocated() == alloc0


def test_noalloc_clears_counters_left_by_a_timed_out_call(cuda_device):
    """A call whose bounded waits run out (a 1 us budget: the first weight boxes are still in
    flight) can leave arrival counters raised in the shared array; the next call clears them
    before its GEMM, so it is exact again.  The kernel drains what it issued before returning,
    so the device stays usable."""
    import w8a8_int8_linear_channel_b200 as sq
    lib = sq._L
    rng = np.random.default_rng(11)
    M, N, K = 16, 4096, 8192
    xq, sx, wq, sw, bias = _inputs(rng, M, N, K, True)
    y_ref = torch.empty((M, N), dtype=torch.float16, device="cuda")
    sq.sq_w8a8_linear(xq, sx, wq, sw, y_ref, bias, workspace=sq.new_workspace(M, N, K))
    assert sq.sq_poll_status() == 0
    y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    try:
        sq.sq_set_wait_budget_ns(1000)
        assert _noalloc_via_c_abi(lib, xq, sx, wq, sw, bias, y) == 0
        assert sq.sq_poll_status() == 8  # SQ_ERR_TIMEOUT
    finally:
        sq.sq_set_wait_budget_ns(2_000_000_000)
    for _ in range(2):
        y.fill_(float("nan"))
        assert _noalloc_via_c_abi(lib, xq, sx, wq, sw, bias, y) == 0
        assert sq.sq_poll_status() == 0
        assert bits_equal(y.cpu().numpy(), y_ref.cpu().numpy())
