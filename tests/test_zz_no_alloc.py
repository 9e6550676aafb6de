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
