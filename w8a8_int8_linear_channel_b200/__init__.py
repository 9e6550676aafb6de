"""SmoothQuant W8A8 linear layer for NVIDIA B200 (sm_100a).

A thin ctypes binding over ``libsq.so`` (C ABI in ``include/sq.h``).  The
functions below carry the C names and only marshal arguments: every step of
the method runs in the library's CUDA kernels; PyTorch provides device memory
and the current stream.  There is no CPU path: importing this package fails
if the library has not been built (``python
w8a8_int8_linear_channel_b200/build.py``).

The method ("SmoothQuant: Accurate and Efficient Post-Training Quantization
for Large Language Models", abeam.tech explainer):
  calibrate  a_j = max|X_j| over calibration tokens, b_j = max|W_j|
  smooth     s_j = a_j^alpha / b_j^(1-alpha), folded into LayerNorm and W
  run        per-token INT8 activations x per-channel INT8 weights -> int32
             -> fp16 with the scales multiplied back.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

__all__ = [
    "SQError", "sq_calibrate_absmax", "sq_calibrate_reset", "sq_smooth_fold", "sq_quantize_weight", "sq_ln_quant_act",
    "sq_w8a8_workspace_bytes", "sq_w8a8_linear", "sq_w8a8_linear_path", "sq_w8a8_gemm_s32",
    "sq_poll_status", "sq_set_wait_budget_ns", "sq_selftest_wait_timeout", "SmoothQuantLinear",
    "sq_quantize_weight_tensor", "sq_ln_quant_act_tensor", "sq_ln_quant_act_static", "sq_tensor_range",
    "LEVELS", "sq_w8a8_linear_quant", "sq_w8a8_linear_quant_dyn", "sq_w8a8_linear_quant_dyn_workspace_bytes",
    "new_quant_dyn_workspace", "sq_w8a8_bmm", "sq_row_ranges", "sq_quantize_rows_ranged",
    "sq_dequant",
    "PATH_AUTO", "PATH_TILED", "PATH_SPLITK", "PATH_PAIR", "SPLITK_MAX_M", "DECODE_MAX_M", "MAX_K", "library_path",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libsq.so")

PATH_AUTO, PATH_TILED, PATH_SPLITK, PATH_PAIR = 0, 1, 2, 3
SPLITK_MAX_M = 128  # the stream-K kernel's largest token count
DECODE_MAX_M = 32   # sq_w8a8_linear always streams the weight up to here
MAX_K = 133144

STATUS = {0: "SQ_OK", 1: "SQ_ERR_INVALID_ARG", 2: "SQ_ERR_MISALIGNED", 3: "SQ_ERR_UNSUPPORTED_SHAPE",
          4: "SQ_ERR_K_OVERFLOW", 5: "SQ_ERR_WORKSPACE", 6: "SQ_ERR_ARCH", 7: "SQ_ERR_CUDA",
          8: "SQ_ERR_TIMEOUT"}


def library_path() -> str:
    return _LIB_PATH


def _load() -> ctypes.CDLL:
    if not os.path.exists(_LIB_PATH):
        raise ImportError(
            f"{_LIB_PATH} is missing: build it with `python w8a8_int8_linear_channel_b200/build.py` "
            "(nvcc, sm_100a).  There is no CPU fallback.")
    L = ctypes.CDLL(_LIB_PATH)
    P, I, F, Z, S = ctypes.c_void_p, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t, ctypes.c_int
    sigs = {
        "sq_status_string": ([S], ctypes.c_char_p),
        "sq_abi_version": ([], S),
        "sq_calibrate_absmax": ([P, I, I, I, P, P, F, P, P], S),
        "sq_calibrate_reset": ([P, I, P], S),
        "sq_smooth_fold": ([P, P, I, F, P, P, P, P, P, P, P, P, I, P], S),
        "sq_quantize_weight": ([P, I, I, P, P, P, P], S),
        "sq_ln_quant_act": ([P, I, I, I, P, P, P, F, P, P, P], S),
        "sq_quantize_weight_tensor": ([P, I, I, P, P, P, P, P], S),
        "sq_ln_quant_act_tensor": ([P, I, I, I, P, P, P, F, P, P, P, P], S),
        "sq_ln_quant_act_static": ([P, I, I, I, P, P, P, F, P, P, P, P], S),
        "sq_tensor_range": ([P, P, I, P, P], S),
        "sq_w8a8_workspace_bytes": ([I, I, I], Z),
        "sq_w8a8_linear": ([P, P, P, P, P, P, I, I, I, P, Z, P], S),
        "sq_w8a8_linear_path": ([P, P, P, P, P, P, I, I, I, P, Z, S, P], S),
        "sq_w8a8_gemm_s32": ([P, P, P, I, I, I, P, Z, S, P], S),
        "sq_w8a8_linear_noalloc": ([P, P, P, P, P, P, I, I, I, P], S),
        "sq_w8a8_linear_quant": ([P, P, P, P, P, S, P, P, P, P, I, I, I, P, Z, P], S),
        "sq_w8a8_linear_quant_dyn_workspace_bytes": ([I, I, I], Z),
        "sq_w8a8_linear_quant_dyn": ([P, P, P, P, P, S, P, P, P, I, I, I, P, Z, P], S),
        "sq_w8a8_bmm": ([P, P, P, P, P, I, I, I, I, P], S),
        "sq_row_ranges": ([P, I, I, I, P, P, P, P, F, P, P], S),
        "sq_quantize_rows_ranged": ([P, I, I, I, P, P, P, P, F, P, P, P, P], S),
        "sq_dequant": ([P, P, P, P, P, I, I, P], S),
        "sq_poll_status": ([P], S),
        "sq_set_wait_budget_ns": ([ctypes.c_uint64], None),
        "sq_selftest_wait_timeout": ([ctypes.c_uint64, P], S),
    }
    for name, (args, res) in sigs.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = res
    return L


_L = _load()


class SQError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}")


def _check(status: int, where: str) -> None:
    if status != 0:
        raise SQError(status, where)


def _p(t: Optional[torch.Tensor]):
    """Device address of a tensor argument.  The C ABI takes pointers on the
    current CUDA device: a host tensor, or one on another GPU, is refused here
    with an error instead of reaching a kernel as a wrong address."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"libsq takes CUDA tensors on the current device; got a tensor on {t.device}")
    cur = torch.cuda.current_device()
    if t.device.index != cur:
        raise ValueError(f"a tensor on {t.device} while the current device is cuda:{cur} "
                         "(libsq runs on the current device: call torch.cuda.set_device first)")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _rows(t: torch.Tensor, dtype, name: str):
    if t.dtype != dtype or t.dim() != 2 or t.stride(1) != 1:
        raise ValueError(f"{name}: need a 2-D {dtype} tensor with unit inner stride")
    return t.shape[0], t.shape[1], t.stride(0)


def _vec(t: Optional[torch.Tensor], n: int, dtype, name: str):
    if t is None:
        return
    if t.dtype != dtype or t.numel() != n or not t.is_contiguous():
        raise ValueError(f"{name}: need a contiguous {dtype} vector of {n} elements")


# --------------------------------------------------------------- C names ----
def sq_calibrate_absmax(x: torch.Tensor, amax: torch.Tensor, gamma=None, beta=None,
                        eps: float = 1e-5, stream=None) -> torch.Tensor:
    """Running per-column absmax of x (or of its LayerNorm with gamma/beta) into amax (fp32 [K])."""
    rows, K, ld = _rows(x, torch.float16, "x")
    _vec(amax, K, torch.float32, "amax")
    _vec(gamma, K, torch.float32, "gamma")
    _vec(beta, K, torch.float32, "beta")
    _check(_L.sq_calibrate_absmax(_p(x), rows, K, ld, _p(gamma), _p(beta), eps, _p(amax),
                                  _stream(stream)), "sq_calibrate_absmax")
    return amax


def sq_calibrate_reset(amax: torch.Tensor, stream=None) -> torch.Tensor:
    """Start a calibration run: every running maximum in amax (fp32, contiguous) back to 0."""
    if amax.dtype != torch.float32 or not amax.is_contiguous() or amax.numel() < 1:
        raise ValueError("amax: need a contiguous fp32 tensor")
    _check(_L.sq_calibrate_reset(_p(amax), amax.numel(), _stream(stream)), "sq_calibrate_reset")
    return amax


def sq_smooth_fold(amax_x, amax_w, alpha: float, s_out, inv_s_out, gamma=None, beta=None,
                   gamma_out=None, beta_out=None, w=None, w_out=None, stream=None):
    """s = a^alpha / b^(1-alpha), inv_s = 1/s; optional fold into gamma/beta and W."""
    K = amax_x.numel()
    for t, n in ((amax_x, "amax_x"), (amax_w, "amax_w"), (s_out, "s_out"), (inv_s_out, "inv_s_out"),
                 (gamma, "gamma"), (beta, "beta"), (gamma_out, "gamma_out"), (beta_out, "beta_out")):
        _vec(t, K, torch.float32, n)
    N = 0
    if w is not None:
        N, Kw, ld = _rows(w, torch.float16, "w")
        if Kw != K or ld != K or w_out is None or w_out.shape != w.shape or not w_out.is_contiguous():
            raise ValueError("w / w_out: need contiguous fp16 [N, K] tensors")
    _check(_L.sq_smooth_fold(_p(amax_x), _p(amax_w), K, alpha, _p(s_out), _p(inv_s_out), _p(gamma),
                             _p(beta), _p(gamma_out), _p(beta_out), _p(w), _p(w_out), N,
                             _stream(stream)), "sq_smooth_fold")


def sq_quantize_weight(w: torch.Tensor, wq: torch.Tensor, w_scale: torch.Tensor, s=None,
                       stream=None):
    """Per-output-channel INT8 of w (folded by s on the fly when given)."""
    N, K, ld = _rows(w, torch.float16, "w")
    if ld != K:
        raise ValueError("w must be contiguous")
    if wq.dtype != torch.int8 or wq.shape != w.shape or not wq.is_contiguous():
        raise ValueError("wq: need a contiguous int8 [N, K] tensor")
    _vec(w_scale, N, torch.float32, "w_scale")
    _vec(s, K, torch.float32, "s")
    _check(_L.sq_quantize_weight(_p(w), N, K, _p(s), _p(wq), _p(w_scale), _stream(stream)),
           "sq_quantize_weight")


def sq_quantize_weight_tensor(w: torch.Tensor, wq: torch.Tensor, w_scale: torch.Tensor,
                              range_out: torch.Tensor, s=None, stream=None):
    """One INT8 scale for the whole (optionally folded) weight; w_scale [N] all equal,
    range_out fp32 [1] receives max |w'|."""
    N, K, ld = _rows(w, torch.float16, "w")
    if ld != K:
        raise ValueError("w must be contiguous")
    if wq.dtype != torch.int8 or wq.shape != w.shape or not wq.is_contiguous():
        raise ValueError("wq: need a contiguous int8 [N, K] tensor")
    _vec(w_scale, N, torch.float32, "w_scale")
    _vec(range_out, 1, torch.float32, "range_out")
    _vec(s, K, torch.float32, "s")
    _check(_L.sq_quantize_weight_tensor(_p(w), N, K, _p(s), _p(wq), _p(w_scale), _p(range_out),
                                        _stream(stream)), "sq_quantize_weight_tensor")


def _act_check(h, xq, x_scale, gamma, beta, inv_s):
    M, K, ld = _rows(h, torch.float16, "h")
    if xq.dtype != torch.int8 or tuple(xq.shape) != (M, K) or not xq.is_contiguous():
        raise ValueError("xq: need a contiguous int8 [M, K] tensor")
    _vec(x_scale, M, torch.float32, "x_scale")
    for t, n in ((gamma, "gamma"), (beta, "beta"), (inv_s, "inv_s")):
        _vec(t, K, torch.float32, n)
    return M, K, ld


def sq_ln_quant_act_tensor(h, xq, x_scale, range_out, gamma=None, beta=None, inv_s=None,
                           eps: float = 1e-5, stream=None):
    """Level O2: one dynamic INT8 scale for the whole batch (range_out fp32 [1] receives it x 127)."""
    M, K, ld = _act_check(h, xq, x_scale, gamma, beta, inv_s)
    _vec(range_out, 1, torch.float32, "range_out")
    _check(_L.sq_ln_quant_act_tensor(_p(h), M, K, ld, _p(gamma), _p(beta), _p(inv_s), eps, _p(xq),
                                     _p(x_scale), _p(range_out), _stream(stream)),
           "sq_ln_quant_act_tensor")


def sq_ln_quant_act_static(h, xq, x_scale, range_in, gamma=None, beta=None, inv_s=None,
                           eps: float = 1e-5, stream=None):
    """Level O3: INT8 with the static scale range_in / 127 (values beyond it saturate)."""
    M, K, ld = _act_check(h, xq, x_scale, gamma, beta, inv_s)
    _vec(range_in, 1, torch.float32, "range_in")
    _check(_L.sq_ln_quant_act_static(_p(h), M, K, ld, _p(gamma), _p(beta), _p(inv_s), eps,
                                     _p(range_in), _p(xq), _p(x_scale), _stream(stream)),
           "sq_ln_quant_act_static")


def sq_tensor_range(amax: torch.Tensor, range_out: torch.Tensor, inv_s=None, stream=None):
    """range_out[0] = max_j amax[j] (* inv_s[j] when given): the static range of level O3."""
    K = amax.numel()
    _vec(amax, K, torch.float32, "amax")
    _vec(inv_s, K, torch.float32, "inv_s")
    _vec(range_out, 1, torch.float32, "range_out")
    _check(_L.sq_tensor_range(_p(amax), _p(inv_s), K, _p(range_out), _stream(stream)), "sq_tensor_range")
    return range_out


def sq_ln_quant_act(h: torch.Tensor, xq: torch.Tensor, x_scale: torch.Tensor, gamma=None,
                    beta=None, inv_s=None, eps: float = 1e-5, stream=None):
    """Optional LayerNorm and smoothing, then per-token INT8 of h."""
    M, K, ld = _rows(h, torch.float16, "h")
    if xq.dtype != torch.int8 or tuple(xq.shape) != (M, K) or not xq.is_contiguous():
        raise ValueError("xq: need a contiguous int8 [M, K] tensor")
    _vec(x_scale, M, torch.float32, "x_scale")
    for t, n in ((gamma, "gamma"), (beta, "beta"), (inv_s, "inv_s")):
        _vec(t, K, torch.float32, n)
    _check(_L.sq_ln_quant_act(_p(h), M, K, ld, _p(gamma), _p(beta), _p(inv_s), eps, _p(xq),
                              _p(x_scale), _stream(stream)), "sq_ln_quant_act")


def sq_w8a8_workspace_bytes(M: int, N: int, K: int) -> int:
    return int(_L.sq_w8a8_workspace_bytes(M, N, K))


def _gemm_shapes(xq, wq):
    M, K, ldx = _rows(xq, torch.int8, "xq")
    N, Kw, ldw = _rows(wq, torch.int8, "wq")
    if Kw != K or ldx != K or ldw != K:
        raise ValueError("xq / wq: need contiguous int8 [M, K] and [N, K]")
    return M, N, K


def sq_w8a8_linear(xq, x_scale, wq, w_scale, y, bias=None, workspace=None, path: int = PATH_AUTO,
                   stream=None):
    """y fp16 [M, N] = fp16((xq @ wq^T) * x_scale[:, None] * w_scale[None, :] + bias)."""
    M, N, K = _gemm_shapes(xq, wq)
    _vec(x_scale, M, torch.float32, "x_scale")
    _vec(w_scale, N, torch.float32, "w_scale")
    _vec(bias, N, torch.float16, "bias")
    if y.dtype != torch.float16 or tuple(y.shape) != (M, N) or not y.is_contiguous():
        raise ValueError("y: need a contiguous fp16 [M, N] tensor")
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_L.sq_w8a8_linear_path(_p(xq), _p(x_scale), _p(wq), _p(w_scale), _p(bias), _p(y), M, N, K,
                                  _p(workspace), ws_bytes, path, _stream(stream)), "sq_w8a8_linear")
    return y


sq_w8a8_linear_path = sq_w8a8_linear


def sq_w8a8_gemm_s32(xq, wq, acc, workspace=None, path: int = PATH_AUTO, stream=None):
    """acc int32 [M, N] = xq @ wq^T (the accumulators, no epilogue)."""
    M, N, K = _gemm_shapes(xq, wq)
    if acc.dtype != torch.int32 or tuple(acc.shape) != (M, N) or not acc.is_contiguous():
        raise ValueError("acc: need a contiguous int32 [M, N] tensor")
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_L.sq_w8a8_gemm_s32(_p(xq), _p(wq), _p(acc), M, N, K, _p(workspace), ws_bytes, path,
                               _stream(stream)), "sq_w8a8_gemm_s32")
    return acc


def sq_w8a8_linear_quant(xq, x_scale, wq, w_scale, range_next, xq_next, x_scale_next, bias=None,
                         relu: bool = False, inv_s_next=None, workspace=None, stream=None):
    """The linear with the next linear's static (level O3) input quantization
    fused into its epilogue: optional ReLU, times inv_s_next, INT8 codes
    xq_next [M, N] with x_scale_next [M] = range_next / 127."""
    M, N, K = _gemm_shapes(xq, wq)
    _vec(x_scale, M, torch.float32, "x_scale")
    _vec(w_scale, N, torch.float32, "w_scale")
    _vec(bias, N, torch.float16, "bias")
    _vec(inv_s_next, N, torch.float32, "inv_s_next")
    _vec(range_next, 1, torch.float32, "range_next")
    _vec(x_scale_next, M, torch.float32, "x_scale_next")
    if xq_next.dtype != torch.int8 or tuple(xq_next.shape) != (M, N) or not xq_next.is_contiguous():
        raise ValueError("xq_next: need a contiguous int8 [M, N] tensor")
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_L.sq_w8a8_linear_quant(_p(xq), _p(x_scale), _p(wq), _p(w_scale), _p(bias), int(bool(relu)),
                                   _p(inv_s_next), _p(range_next), _p(xq_next), _p(x_scale_next), M, N, K,
                                   _p(workspace), ws_bytes, _stream(stream)), "sq_w8a8_linear_quant")
    return xq_next, x_scale_next


def sq_w8a8_linear_quant_dyn_workspace_bytes(M: int, N: int, K: int) -> int:
    return int(_L.sq_w8a8_linear_quant_dyn_workspace_bytes(M, N, K))


def new_quant_dyn_workspace(M: int, N: int, K: int, device=None) -> torch.Tensor:
    """A zero-filled workspace for sq_w8a8_linear_quant_dyn."""
    return torch.zeros(sq_w8a8_linear_quant_dyn_workspace_bytes(M, N, K), dtype=torch.uint8,
                       device=device or "cuda")


def sq_w8a8_linear_quant_dyn(xq, x_scale, wq, w_scale, xq_next, x_scale_next, bias=None, relu: bool = False,
                             inv_s_next=None, workspace=None, stream=None):
    """The linear with the next linear's per-token dynamic input quantization: optional ReLU,
    times inv_s_next, per-token scale x_scale_next [M] = max |x| / 127 and INT8 codes
    xq_next [M, N] (two launches: the GEMM with a row-maximum epilogue, then the codes)."""
    M, N, K = _gemm_shapes(xq, wq)
    _vec(x_scale, M, torch.float32, "x_scale")
    _vec(w_scale, N, torch.float32, "w_scale")
    _vec(bias, N, torch.float16, "bias")
    _vec(inv_s_next, N, torch.float32, "inv_s_next")
    _vec(x_scale_next, M, torch.float32, "x_scale_next")
    if xq_next.dtype != torch.int8 or tuple(xq_next.shape) != (M, N) or not xq_next.is_contiguous():
        raise ValueError("xq_next: need a contiguous int8 [M, N] tensor")
    if workspace is None:
        workspace = new_quant_dyn_workspace(M, N, K, device=xq.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(_L.sq_w8a8_linear_quant_dyn(_p(xq), _p(x_scale), _p(wq), _p(w_scale), _p(bias), int(bool(relu)),
                                       _p(inv_s_next), _p(xq_next), _p(x_scale_next), M, N, K, _p(workspace),
                                       ws_bytes, _stream(stream)), "sq_w8a8_linear_quant_dyn")
    return xq_next, x_scale_next


def sq_row_ranges(x, range_out, gamma=None, beta=None, inv_s=None, s_fold=None, eps: float = 1e-5,
                  stream=None):
    """range_out[r] = max |x_hat[r, :]| over this slice's columns (activation transform, or the
    folded weight when s_fold is given): a tensor-parallel shard's row ranges."""
    rows, K, ld = _rows(x, torch.float16, "x")
    _vec(range_out, rows, torch.float32, "range_out")
    for t, n in ((gamma, "gamma"), (beta, "beta"), (inv_s, "inv_s"), (s_fold, "s_fold")):
        _vec(t, K, torch.float32, n)
    _check(_L.sq_row_ranges(_p(x), rows, K, ld, _p(gamma), _p(beta), _p(inv_s), _p(s_fold), eps,
                            _p(range_out), _stream(stream)), "sq_row_ranges")
    return range_out


def sq_quantize_rows_ranged(x, range_in, q, scale, gamma=None, beta=None, inv_s=None, s_fold=None,
                            eps: float = 1e-5, stream=None):
    """INT8 codes of the rows with given per-row ranges (scale = range / 127, codes clamped)."""
    rows, K, ld = _rows(x, torch.float16, "x")
    _vec(range_in, rows, torch.float32, "range_in")
    _vec(scale, rows, torch.float32, "scale")
    if q.dtype != torch.int8 or tuple(q.shape) != (rows, K) or not q.is_contiguous():
        raise ValueError("q: need a contiguous int8 [rows, K] tensor")
    for t, n in ((gamma, "gamma"), (beta, "beta"), (inv_s, "inv_s"), (s_fold, "s_fold")):
        _vec(t, K, torch.float32, n)
    _check(_L.sq_quantize_rows_ranged(_p(x), rows, K, ld, _p(gamma), _p(beta), _p(inv_s), _p(s_fold), eps,
                                      _p(range_in), _p(q), _p(scale), _stream(stream)), "sq_quantize_rows_ranged")
    return q, scale


def sq_dequant(acc, x_scale, w_scale, y, bias=None, stream=None):
    """y = fp16((acc * x_scale[:, None]) * w_scale[None, :] + bias) from int32 accumulators."""
    if acc.dtype != torch.int32 or acc.dim() != 2 or not acc.is_contiguous():
        raise ValueError("acc: need a contiguous int32 [M, N] tensor")
    M, N = acc.shape
    _vec(x_scale, M, torch.float32, "x_scale")
    _vec(w_scale, N, torch.float32, "w_scale")
    _vec(bias, N, torch.float16, "bias")
    if y.dtype != torch.float16 or tuple(y.shape) != (M, N) or not y.is_contiguous():
        raise ValueError("y: need a contiguous fp16 [M, N] tensor")
    _check(_L.sq_dequant(_p(acc), _p(x_scale), _p(w_scale), _p(bias), _p(y), M, N, _stream(stream)), "sq_dequant")
    return y


def sq_w8a8_bmm(a, a_scale, b, b_scale, y, stream=None):
    """INT8 BMM: y[i] = fp16((a[i] @ b[i]^T) * a_scale[i][:, None] * b_scale[i][None, :]) for every
    batch item i; a int8 [B, M, K], b int8 [B, N, K], scales fp32 [B, M] / [B, N], y fp16 [B, M, N]."""
    for t, n in ((a, "a"), (b, "b")):
        if t.dtype != torch.int8 or t.dim() != 3 or not t.is_contiguous():
            raise ValueError(f"{n}: need a contiguous int8 [batch, rows, K] tensor")
    B, M, K = a.shape
    if b.shape[0] != B or b.shape[2] != K:
        raise ValueError("b: need [batch, N, K] with the same batch and K as a")
    N = b.shape[1]
    for t, n, r in ((a_scale, "a_scale", M), (b_scale, "b_scale", N)):
        if t.dtype != torch.float32 or tuple(t.shape) != (B, r) or not t.is_contiguous():
            raise ValueError(f"{n}: need a contiguous fp32 [batch, {r}] tensor")
    if y.dtype != torch.float16 or tuple(y.shape) != (B, M, N) or not y.is_contiguous():
        raise ValueError("y: need a contiguous fp16 [batch, M, N] tensor")
    _check(_L.sq_w8a8_bmm(_p(a), _p(a_scale), _p(b), _p(b_scale), _p(y), B, M, N, K, _stream(stream)),
           "sq_w8a8_bmm")
    return y


def sq_w8a8_linear_noalloc(xq, x_scale, wq, w_scale, y, bias=None, stream=None):
    """sq_w8a8_linear for M <= 32 without a workspace: for callers that cannot
    allocate device memory (the library's own fixed scratch array is used;
    overlapping calls race on it)."""
    M, N, K = _gemm_shapes(xq, wq)
    _vec(x_scale, M, torch.float32, "x_scale")
    _vec(w_scale, N, torch.float32, "w_scale")
    _vec(bias, N, torch.float16, "bias")
    if y.dtype != torch.float16 or tuple(y.shape) != (M, N) or not y.is_contiguous():
        raise ValueError("y: need a contiguous fp16 [M, N] tensor")
    _check(_L.sq_w8a8_linear_noalloc(_p(xq), _p(x_scale), _p(wq), _p(w_scale), _p(bias), _p(y),
                                     M, N, K, _stream(stream)), "sq_w8a8_linear_noalloc")
    return y


def sq_poll_status(stream=None) -> int:
    """Synchronize the stream; return the status code of the device's bounded waits (and clear it).
    After SQ_ERR_TIMEOUT (8), zero-fill the stream-K workspaces used by the timed-out calls
    (SmoothQuantLinear.reset_workspaces for a layer's own)."""
    return int(_L.sq_poll_status(_stream(stream)))


def sq_set_wait_budget_ns(ns: int) -> None:
    _L.sq_set_wait_budget_ns(int(ns))


def sq_selftest_wait_timeout(budget_ns: int, stream=None) -> None:
    _check(_L.sq_selftest_wait_timeout(int(budget_ns), _stream(stream)), "sq_selftest_wait_timeout")


def new_workspace(M: int, N: int, K: int, device=None) -> Optional[torch.Tensor]:
    """A zero-filled workspace tensor for sq_w8a8_linear (None if the shape needs none)."""
    n = sq_w8a8_workspace_bytes(M, N, K)
    if n == 0:
        return None
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")


# ------------------------------------------------------------- layer API ----
# (activation granularity, weight granularity) of each quantization level:
# "channel" is this library's default (per-token activations, per-output-channel
# weights); O1-O3 are the explainer's efficiency levels (section "inference").
LEVELS = {
    "channel": ("token", "channel"),
    "O1": ("token", "tensor"),
    "O2": ("tensor", "tensor"),
    "O3": ("static", "tensor"),
}


class SmoothQuantLinear:
    """A quantized nn.Linear with its smoothing folded in.

    Built from an fp16 weight, its input's calibration tokens and (optionally)
    the LayerNorm that precedes it; ``forward`` runs the per-token quantization
    and the INT8 GEMM.  All work happens in libsq kernels on the current
    stream."""

    def __init__(self, wq, w_scale, bias, gamma_f, beta_f, inv_s, s, eps, smooth_inv=None,
                 level: str = "channel", act_range=None):
        self.wq, self.w_scale, self.bias = wq, w_scale, bias
        self.gamma_f, self.beta_f, self.inv_s, self.s = gamma_f, beta_f, inv_s, s
        self.smooth_inv = smooth_inv if smooth_inv is not None else inv_s  # 1/s, always kept
        self.eps = eps
        self.level = level
        self.act_mode = LEVELS[level][0]
        # fp32 [1]: the static range (O3) or the per-batch range written by O2
        self.act_range = act_range
        if self.act_mode == "tensor" and act_range is None:
            self.act_range = torch.zeros(1, dtype=torch.float32, device=wq.device)
        self._ws = {}

    @classmethod
    def from_float(cls, w: torch.Tensor, calib: torch.Tensor, alpha: float = 0.5, gamma=None,
                   beta=None, bias=None, eps: float = 1e-5, amax_x: Optional[torch.Tensor] = None,
                   process_group=None, level: str = "channel"):
        """Calibrate on ``calib`` (the LayerNorm input when gamma is given, else the
        linear's input), smooth with ``alpha`` and quantize ``w`` [N, K].  With a
        process group, the activation ranges are max-reduced over its ranks so
        every rank derives the same smoothing (data-parallel calibration).
        ``level`` picks the scale granularities (see LEVELS)."""
        if level not in LEVELS:
            raise ValueError(f"level: one of {sorted(LEVELS)}")
        act_mode, w_mode = LEVELS[level]
        N, K = w.shape
        dev = w.device
        if amax_x is None:
            amax_x = torch.zeros(K, dtype=torch.float32, device=dev)
            sq_calibrate_absmax(calib, amax_x, gamma, beta, eps)
        if process_group is not None:
            import torch.distributed as dist
            dist.all_reduce(amax_x, op=dist.ReduceOp.MAX, group=process_group)
        amax_w = torch.zeros(K, dtype=torch.float32, device=dev)
        sq_calibrate_absmax(w, amax_w)
        s = torch.empty(K, dtype=torch.float32, device=dev)
        inv_s = torch.empty_like(s)
        gamma_f = torch.empty_like(s) if gamma is not None else None
        beta_f = torch.empty_like(s) if beta is not None else None
        sq_smooth_fold(amax_x, amax_w, alpha, s, inv_s, gamma, beta, gamma_f, beta_f)
        wq = torch.empty((N, K), dtype=torch.int8, device=dev)
        w_scale = torch.empty(N, dtype=torch.float32, device=dev)
        if w_mode == "tensor":
            w_range = torch.zeros(1, dtype=torch.float32, device=dev)
            sq_quantize_weight_tensor(w, wq, w_scale, w_range, s=s)
        else:
            sq_quantize_weight(w, wq, w_scale, s=s)
        runtime_inv_s = None if gamma is not None else inv_s
        act_range = None
        if act_mode == "static":
            # the static range of the runtime transform over the calibration set
            act_range = torch.zeros(1, dtype=torch.float32, device=dev)
            if gamma is not None:
                amax_hat = torch.zeros(K, dtype=torch.float32, device=dev)
                sq_calibrate_absmax(calib, amax_hat, gamma_f, beta_f, eps)
                sq_tensor_range(amax_hat, act_range)
            else:
                sq_tensor_range(amax_x, act_range, inv_s=inv_s)
            if process_group is not None:
                import torch.distributed as dist
                dist.all_reduce(act_range, op=dist.ReduceOp.MAX, group=process_group)
        return cls(wq, w_scale, bias, gamma_f, beta_f, runtime_inv_s, s, eps, inv_s, level=level,
                   act_range=act_range)

    def workspace(self, M: int) -> Optional[torch.Tensor]:
        """The stream-K workspace for M tokens (None where no kernel needs one).  Calls that share
        a workspace must not overlap on the GPU, so the layer keeps one per stream.  (At level O2
        every forward also writes the layer's one batch-range buffer, ``act_range``, so O2
        forwards on different streams must still not overlap.)"""
        N, K = self.wq.shape
        need = sq_w8a8_workspace_bytes(M, N, K)
        if need == 0:
            return None
        key = torch.cuda.current_stream(self.wq.device).cuda_stream
        ws = self._ws.get(key)
        if ws is None or ws.numel() < need:
            ws = torch.zeros(need, dtype=torch.uint8, device=self.wq.device)
            self._ws[key] = ws
        return ws

    def reset_workspaces(self) -> None:
        """Zero-fill every stream-K workspace the layer holds.  Needed after a forward whose
        bounded device wait ran out (sq_poll_status returned SQ_ERR_TIMEOUT): that call may
        leave per-tile arrival counters non-zero, and a later decode-sized forward on the same
        stream would then elect the wrong last contributor."""
        for ws in self._ws.values():
            ws.zero_()

    def quantize_input(self, h: torch.Tensor, xq=None, x_scale=None):
        M, K = h.shape
        xq = torch.empty((M, K), dtype=torch.int8, device=h.device) if xq is None else xq
        x_scale = torch.empty(M, dtype=torch.float32, device=h.device) if x_scale is None else x_scale
        if self.act_mode == "tensor":
            sq_ln_quant_act_tensor(h, xq, x_scale, self.act_range, self.gamma_f, self.beta_f,
                                   self.inv_s, self.eps)
        elif self.act_mode == "static":
            sq_ln_quant_act_static(h, xq, x_scale, self.act_range, self.gamma_f, self.beta_f,
                                   self.inv_s, self.eps)
        else:
            sq_ln_quant_act(h, xq, x_scale, self.gamma_f, self.beta_f, self.inv_s, self.eps)
        return xq, x_scale

    def forward(self, h: torch.Tensor, y: Optional[torch.Tensor] = None) -> torch.Tensor:
        """h fp16 [..., K] (the LayerNorm input if a LayerNorm was folded) -> y fp16 [..., N].
        Leading dimensions are flattened into tokens; an empty batch launches nothing."""
        N, K = self.wq.shape
        if h.dim() < 1 or h.shape[-1] != K:
            raise ValueError(f"h: need [..., {K}], got {tuple(h.shape)}")
        lead = tuple(h.shape[:-1])
        h2 = h if h.dim() == 2 else h.reshape(-1, K)
        M = h2.shape[0]
        if y is None:
            y = torch.empty(lead + (N,), dtype=torch.float16, device=h.device)
        elif tuple(y.shape) not in (lead + (N,), (M, N)) or not y.is_contiguous():
            raise ValueError(f"y: need a contiguous fp16 {lead + (N,)} tensor")
        if M == 0:
            return y
        xq, x_scale = self.quantize_input(h2)
        sq_w8a8_linear(xq, x_scale, self.wq, self.w_scale, y.view(M, N), self.bias, self.workspace(M))
        return y

    __call__ = forward
