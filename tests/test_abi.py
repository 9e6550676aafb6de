"""The C-ABI library without a GPU: it loads, exports every entry point the
header declares, and rejects bad arguments on the host before touching a
device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sq.h")


def _lib():
    import w8a8_int8_linear_channel_b200 as sq
    return sq._L


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sq_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_five_stage_entry_points():
    names = declared_functions()
    for n in ["sq_calibrate_absmax", "sq_smooth_fold", "sq_quantize_weight", "sq_ln_quant_act",
              "sq_w8a8_linear"]:
        assert n in names


def test_library_exports_every_declared_symbol():
    L = ctypes.CDLL(os.path.join(ROOT, "w8a8_int8_linear_channel_b200", "libsq.so"))
    missing = [n for n in declared_functions() if not hasattr(L, n)]
    assert not missing, missing


def test_status_strings():
    L = _lib()
    assert L.sq_status_string(0) == b"SQ_OK"
    assert L.sq_status_string(8) == b"SQ_ERR_TIMEOUT"
    assert L.sq_status_string(99) == b"SQ_ERR_UNKNOWN"
    assert L.sq_abi_version() == 200


FAKE = ctypes.c_void_p(0x10000)      # 16-byte aligned, never dereferenced
FAKE_ODD = ctypes.c_void_p(0x10004)  # misaligned


def test_linear_rejects_bad_arguments_on_the_host():
    L = _lib()
    f = L.sq_w8a8_linear
    ok = dict(M=64, N=64, K=64)
    # null operand
    assert f(None, FAKE, FAKE, FAKE, None, FAKE, 64, 64, 64, None, 0, None) == 1
    # non-positive sizes
    assert f(FAKE, FAKE, FAKE, FAKE, None, FAKE, 0, 64, 64, None, 0, None) == 1
    assert f(FAKE, FAKE, FAKE, FAKE, None, FAKE, 64, -1, 64, None, 0, None) == 1
    # K must be a multiple of 16 and at most 133144
    assert f(FAKE, FAKE, FAKE, FAKE, None, FAKE, 64, 64, 40, None, 0, None) == 3
    assert f(FAKE, FAKE, FAKE, FAKE, None, FAKE, 64, 64, 133152, None, 0, None) == 4
    # misaligned pointer
    assert f(FAKE_ODD, FAKE, FAKE, FAKE, None, FAKE, 64, 64, 64, None, 0, None) == 2
    # forced stream-K path for too many tokens
    assert L.sq_w8a8_linear_path(FAKE, FAKE, FAKE, FAKE, None, FAKE, 129, 64, 64, FAKE, 1 << 20, 2, None) == 3
    # unknown path (4 named single-CTA 256 x 256 tiles before ABI 2.0)
    assert L.sq_w8a8_linear_path(FAKE, FAKE, FAKE, FAKE, None, FAKE, 8, 64, 64, FAKE, 1 << 20, 7, None) == 1
    assert L.sq_w8a8_linear_path(FAKE, FAKE, FAKE, FAKE, None, FAKE, 300, 64, 64, None, 0, 4, None) == 1
    del ok


def test_dynamic_producer_rejects_bad_arguments_on_the_host():
    L = _lib()
    f = L.sq_w8a8_linear_quant_dyn
    big = 1 << 30
    # no workspace / null operand
    assert f(FAKE, FAKE, FAKE, FAKE, None, 0, None, FAKE, FAKE, 64, 64, 64, None, big, None) == 1
    assert f(None, FAKE, FAKE, FAKE, None, 0, None, FAKE, FAKE, 64, 64, 64, FAKE, big, None) == 1
    # N (the next linear's K) must be a multiple of 16; K as everywhere
    assert f(FAKE, FAKE, FAKE, FAKE, None, 0, None, FAKE, FAKE, 64, 40, 64, FAKE, big, None) == 3
    assert f(FAKE, FAKE, FAKE, FAKE, None, 0, None, FAKE, FAKE, 64, 64, 40, FAKE, big, None) == 3
    # misaligned workspace or 1/s
    assert f(FAKE, FAKE, FAKE, FAKE, None, 0, None, FAKE, FAKE, 64, 64, 64, FAKE_ODD, big, None) == 2
    assert f(FAKE, FAKE, FAKE, FAKE, None, 0, FAKE_ODD, FAKE, FAKE, 64, 64, 64, FAKE, big, None) == 2
    # the workspace query: a fp16 copy of the output and the row-group maxima (more for decode)
    ws = L.sq_w8a8_linear_quant_dyn_workspace_bytes
    assert ws(300, 4096, 4096) >= 300 * 4096 * 2 + 300 * 32 * 4
    assert ws(16, 4096, 4096) > 16 * 4096 * 2 + 16 * 128 * 4
    assert ws(0, 64, 64) == 0 and ws(4, 64, -1) == 0


def test_other_entry_points_reject_bad_arguments():
    L = _lib()
    assert L.sq_calibrate_absmax(None, 4, 64, 64, None, None, 1e-5, FAKE, None) == 1
    assert L.sq_calibrate_absmax(FAKE, 4, 64, 60, None, None, 1e-5, FAKE, None) == 1   # ld < K
    assert L.sq_calibrate_absmax(FAKE, 4, 64, 68, None, None, 1e-5, FAKE, None) == 2   # ld % 8
    assert L.sq_calibrate_absmax(FAKE, 4, 64, 64, None, FAKE, 1e-5, FAKE, None) == 1   # beta w/o gamma
    assert L.sq_smooth_fold(FAKE, FAKE, 64, ctypes.c_float(1.5), FAKE, FAKE, None, None, None, None,
                            None, None, 0, None) == 1  # alpha out of [0, 1]
    assert L.sq_smooth_fold(FAKE, FAKE, 64, ctypes.c_float(0.5), FAKE, FAKE, FAKE, None, None, None,
                            None, None, 0, None) == 1  # gamma without gamma_out
    assert L.sq_quantize_weight(FAKE, 0, 64, None, FAKE, FAKE, None) == 1
    assert L.sq_quantize_weight(FAKE, 8, 24, None, FAKE, FAKE, None) == 3
    assert L.sq_ln_quant_act(FAKE, 8, 64, 64, None, None, FAKE_ODD, 1e-5, FAKE, FAKE, None) == 2
    assert L.sq_w8a8_gemm_s32(FAKE, FAKE, None, 8, 8, 64, None, 0, 0, None) == 1


def test_remaining_entry_points_reject_bad_arguments_on_the_host():
    """Every other entry point: null or non-positive arguments (1), misaligned
    pointers or leading dimensions (2), K or N outside the shape rules (3), K
    past SQ_MAX_K (4), a shape beyond the fixed scratch (5) -- each returned
    before any device is touched."""
    L = _lib()
    big = 1 << 30
    # the range reset
    assert L.sq_calibrate_reset(None, 16, None) == 1
    assert L.sq_calibrate_reset(FAKE, 0, None) == 1
    assert L.sq_calibrate_reset(FAKE_ODD, 16, None) == 2
    # per-tensor weight scale (O1-O3): the range output is required
    f = L.sq_quantize_weight_tensor
    assert f(FAKE, 8, 64, None, FAKE, FAKE, None, None) == 1
    assert f(FAKE, 8, 24, None, FAKE, FAKE, FAKE, None) == 3
    assert f(FAKE, 8, 133152, None, FAKE, FAKE, FAKE, None) == 4
    assert f(FAKE, 8, 64, None, FAKE, FAKE, FAKE_ODD, None) == 2
    assert f(FAKE, 8, 64, FAKE_ODD, FAKE, FAKE, FAKE, None) == 2
    # per-tensor dynamic (O2) and static (O3) activation scales
    for g in (L.sq_ln_quant_act_tensor, L.sq_ln_quant_act_static):
        assert g(FAKE, 8, 64, 64, None, None, None, 1e-5, FAKE, FAKE, None, None) == 1   # no range
        assert g(FAKE, 0, 64, 64, None, None, None, 1e-5, FAKE, FAKE, FAKE, None) == 1   # M = 0
        assert g(FAKE, 8, 64, 64, None, FAKE, None, 1e-5, FAKE, FAKE, FAKE, None) == 1   # beta w/o gamma
        assert g(FAKE, 8, 64, 56, None, None, None, 1e-5, FAKE, FAKE, FAKE, None) == 1   # ld < K
        assert g(FAKE, 8, 64, 68, None, None, None, 1e-5, FAKE, FAKE, FAKE, None) == 2   # ld % 8
        assert g(FAKE, 8, 64, 64, None, None, None, 1e-5, FAKE, FAKE, FAKE_ODD, None) == 2
        assert g(FAKE, 8, 40, 40, None, None, None, 1e-5, FAKE, FAKE, FAKE, None) == 3
    # the tensor range from calibrated column maxima (any K up to SQ_MAX_K)
    assert L.sq_tensor_range(None, None, 64, FAKE, None) == 1
    assert L.sq_tensor_range(FAKE, None, 0, FAKE, None) == 1
    assert L.sq_tensor_range(FAKE, None, 133152, FAKE, None) == 4
    assert L.sq_tensor_range(FAKE, FAKE_ODD, 64, FAKE, None) == 2
    # per-row ranges and quantization against them: the weight fold (s_fold)
    # excludes the activation transform (LayerNorm, 1/s)
    f = L.sq_row_ranges
    assert f(FAKE, 8, 64, 64, FAKE, None, None, FAKE, 1e-5, FAKE, None) == 1
    assert f(FAKE, 8, 64, 64, None, None, FAKE, FAKE, 1e-5, FAKE, None) == 1
    assert f(FAKE, 8, 64, 64, None, None, None, None, 1e-5, None, None) == 1
    assert f(FAKE, 8, 64, 64, None, None, None, None, 1e-5, FAKE_ODD, None) == 2
    assert f(FAKE, 8, 40, 40, None, None, None, None, 1e-5, FAKE, None) == 3
    f = L.sq_quantize_rows_ranged
    assert f(FAKE, 8, 64, 64, None, None, None, None, 1e-5, None, FAKE, FAKE, None) == 1
    assert f(FAKE, 8, 64, 64, None, None, None, None, 1e-5, FAKE, FAKE_ODD, FAKE, None) == 2
    # the row-parallel layer's dequantization: N % 4 == 0
    assert L.sq_dequant(None, FAKE, FAKE, None, FAKE, 8, 8, None) == 1
    assert L.sq_dequant(FAKE, FAKE, FAKE, None, FAKE, 0, 8, None) == 1
    assert L.sq_dequant(FAKE, FAKE, FAKE, None, FAKE, 8, 6, None) == 3
    assert L.sq_dequant(FAKE, FAKE, FAKE, FAKE_ODD, FAKE, 8, 8, None) == 2
    # the static producer-side quantization: N is the next linear's K
    f = L.sq_w8a8_linear_quant
    assert f(FAKE, FAKE, FAKE, FAKE, None, 0, None, None, FAKE, FAKE, 64, 64, 64, FAKE, big, None) == 1
    assert f(FAKE, FAKE, FAKE, FAKE, None, 0, None, FAKE, FAKE, FAKE, 64, 40, 64, FAKE, big, None) == 3
    assert f(FAKE, FAKE, FAKE, FAKE, None, 0, None, FAKE, FAKE, FAKE, 64, 64, 40, FAKE, big, None) == 3
    assert f(FAKE, FAKE, FAKE, FAKE, None, 0, None, FAKE, FAKE_ODD, FAKE, 64, 64, 64, FAKE, big, None) == 2
    # the INT8 BMM
    f = L.sq_w8a8_bmm
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 0, 64, 64, 64, None) == 1
    assert f(FAKE, FAKE, FAKE, FAKE, None, 2, 64, 64, 64, None) == 1
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 2, 64, 64, 40, None) == 3
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 2, 64, 64, 133152, None) == 4
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE_ODD, 2, 64, 64, 64, None) == 2
    # the allocation-free decode entry: M <= 32, at most 4096 tiles of 128 channels
    f = L.sq_w8a8_linear_noalloc
    assert f(None, FAKE, FAKE, FAKE, None, FAKE, 8, 64, 64, None) == 1
    assert f(FAKE, FAKE, FAKE, FAKE, None, FAKE, 33, 64, 64, None) == 3
    assert f(FAKE, FAKE, FAKE, FAKE, None, FAKE, 8, 64, 40, None) == 3
    assert f(FAKE, FAKE, FAKE, FAKE, None, FAKE, 8, 64, 133152, None) == 4
    assert f(FAKE, FAKE, FAKE, FAKE, None, FAKE, 8, 128 * 4096 + 1, 64, None) == 5
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE_ODD, FAKE, 8, 64, 64, None) == 2


def test_workspace_size_formula():
    L = _lib()
    assert L.sq_w8a8_workspace_bytes(129, 4096, 4096) == 0      # beyond stream-K: none
    assert L.sq_w8a8_workspace_bytes(0, 4096, 4096) == 0
    n = L.sq_w8a8_workspace_bytes(32, 49152, 12288)
    # counters for 384 channel tiles (rounded to 256 B) + 2 int32 [128 x 32] slots per SM
    assert n >= 1536 + 2 * 148 * 128 * 32 * 4
    # 33-64 tokens take the 64-token tile, 65-128 the 128-token tile
    assert L.sq_w8a8_workspace_bytes(64, 4096, 4096) >= 256 + 2 * 148 * 128 * 64 * 4
    assert L.sq_w8a8_workspace_bytes(65, 4096, 4096) >= 256 + 2 * 148 * 128 * 128 * 4


def _has_gpu():
    import torch
    return torch.cuda.is_available()


@pytest.mark.skipif(_has_gpu(), reason="a GPU is present")
def test_valid_call_without_a_device_reports_cuda_error():
    L = _lib()
    r = L.sq_w8a8_linear(FAKE, FAKE, FAKE, FAKE, None, FAKE, 64, 64, 64, None, 0, None)
    assert r == 7  # SQ_ERR_CUDA: no device; nothing was launched


def test_binding_refuses_host_tensors():
    # a host tensor must never reach a kernel as a device address: the binding refuses it
    # before calling the library
    import torch

    import w8a8_int8_linear_channel_b200 as sq
    xq = torch.zeros((4, 16), dtype=torch.int8)
    wq = torch.zeros((8, 16), dtype=torch.int8)
    sx, sw = torch.zeros(4), torch.zeros(8)
    y = torch.empty((4, 8), dtype=torch.float16)
    with pytest.raises(ValueError, match="CUDA tensors"):
        sq.sq_w8a8_linear(xq, sx, wq, sw, y)
    h = torch.zeros((4, 16), dtype=torch.float16)
    with pytest.raises(ValueError, match="CUDA tensors"):
        sq.sq_ln_quant_act(h, xq, sx)
    with pytest.raises(ValueError, match="CUDA tensors"):
        sq.sq_calibrate_absmax(h, torch.zeros(16))
    with pytest.raises(ValueError, match="CUDA tensors"):
        sq.sq_w8a8_bmm(xq[None], sx[None], wq[None], sw[None], y[None])


def test_layer_forward_refuses_a_host_input():
    # SmoothQuantLinear.forward on a host tensor must fail before any kernel is launched
    import torch

    import w8a8_int8_linear_channel_b200 as sq
    K, N = 16, 8
    layer = sq.SmoothQuantLinear(torch.zeros((N, K), dtype=torch.int8), torch.zeros(N), None, None, None,
                                 torch.ones(K), torch.ones(K), 1e-5)
    with pytest.raises(ValueError, match="CUDA tensors"):
        layer(torch.zeros((3, K), dtype=torch.float16))
