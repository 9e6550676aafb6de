"""CPU oracle for the SmoothQuant W8A8 linear layer -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
leg of ``bench.py`` may import this package.  The product path (the CUDA
library in ``w8a8_int8_linear_channel_b200``) never imports it, and this
package never imports the product.  The two share only the seeded input
generator ``sq_inputs``.

Two layers:

* ``liboracle.so`` (``sq_oracle.c``): the method in the exact fp32 / int32
  operation order that decides the INT8 codes, the int32 accumulators and the
  fp16 outputs.  Plain loops, ``-ffp-contract=off``.
* fp64 numpy helpers below: the mathematics the pages state without any
  rounding (the smoothing factor, the equivalence Y = (X diag(s)^-1)(diag(s)W),
  the unquantized product), used by the pins and by the quality check.

Sources, cited by page title and section:
  [SQ] "SmoothQuant: Accurate and Efficient Post-Training Quantization for
       Large Language Models", abeam.tech explainer -- glossary
       "Calibration" / "INT8 GEMM", "what it does mathematically", "why
       activations are hard to quantize", "how is the smoothing factor
       chosen", "inference" (O1/O2/O3).
  [Q]  itmedia LLM quantization tutorial, section 3 (range -> scale -> round,
       the 53 -> 5 -> 50 example).

Beyond the per-token / per-channel layer: the explainer's quantization
levels O1-O3 (``quantize_weight_tensor``, ``ln_quant_act_tensor``,
``ln_quant_act_static``, ``tensor_range``), producer-side quantization at a
static scale (``w8a8_linear_quant_static``) and at the per-token dynamic
scale (``w8a8_linear_quant_dynamic``), and the INT8 BMM (``w8a8_bmm``).

Parity status: every function here is pinned by ``tests/test_oracle.py``,
including the two unsmoothed quality references (``naive_per_tensor_w8a8``,
``per_token_per_channel_w8a8``: a hand-worked fixture and the case where
both coincide).  The ranking those references feed (naive error above the
smoothed error on outlier inputs) is a qualitative prediction of the pages,
checked as such, not a pinned value.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_HERE = os.path.dirname(os.path.abspath(__file__))

_lib = None


def lib() -> ctypes.CDLL:
    """Load (building first if needed) liboracle.so."""
    global _lib
    if _lib is None:
        # SQ_ORACLE_LIB lets the mutation test load a deliberately broken copy.
        path = os.environ.get("SQ_ORACLE_LIB") or _build.build()
        _lib = ctypes.CDLL(path)
        _declare(_lib)
    return _lib


_P = ctypes.c_void_p
_I = ctypes.c_int64
_F = ctypes.c_float


def _declare(L):
    sig = {
        "oracle_half_to_float": [_P, _P, _I],
        "oracle_float_to_half": [_P, _P, _I],
        "oracle_quantize_with_scale": [_P, _I, _F, _P],
        "oracle_ln_stats": [_P, _I, _I, _I, _F, _P, _P],
        "oracle_act_rows": [_P, _I, _I, _I, _P, _P, _P, _F, _P],
        "oracle_calibrate_absmax": [_P, _I, _I, _I, _P, _P, _F, _P, _P],
        "oracle_smooth": [_P, _P, _I, _F, _P, _P],
        "oracle_fold_ln": [_P, _P, _P, _I, _P, _P],
        "oracle_fold_weight": [_P, _I, _I, _P, _P],
        "oracle_quantize_weight": [_P, _I, _I, _P, _P],
        "oracle_ln_quant_act": [_P, _I, _I, _I, _P, _P, _P, _F, _P, _P, _P],
        "oracle_quantize_weight_tensor": [_P, _I, _I, _P, _P, _P],
        "oracle_ln_quant_act_tensor": [_P, _I, _I, _I, _P, _P, _P, _F, _P, _P, _P, _P],
        "oracle_ln_quant_act_static": [_P, _I, _I, _I, _P, _P, _P, _F, _F, _P, _P, _P],
        "oracle_tensor_range": [_P, _P, _I],
        "oracle_int_gemm": [_P, _P, _I, _I, _I, _P],
        "oracle_int_gemm64": [_P, _P, _I, _I, _I, _P],
        "oracle_dequant": [_P, _P, _P, _P, _I, _I, _P],
        "oracle_w8a8_linear": [_P, _P, _P, _P, _P, _I, _I, _I, _P],
        "oracle_w8a8_linear_quant_static": [_P, _P, _P, _P, _P, ctypes.c_int, _P, _F, _I, _I, _I, _P, _P],
        "oracle_w8a8_bmm": [_P, _P, _P, _P, _I, _I, _I, _I, _P],
        "oracle_num_threads": [],
        "oracle_set_num_threads": [ctypes.c_int],
    }
    for name, args in sig.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = (ctypes.c_int if name == "oracle_num_threads" else
                      ctypes.c_float if name == "oracle_tensor_range" else None)


def _ptr(a):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data


def _f16(a):
    a = np.ascontiguousarray(a)
    assert a.dtype == np.float16, a.dtype
    return a


def _f32(a):
    if a is None:
        return None
    return np.ascontiguousarray(a, dtype=np.float32)


def num_threads() -> int:
    return lib().oracle_num_threads()


def set_num_threads(n: int) -> None:
    lib().oracle_set_num_threads(int(n))


# --------------------------------------------------------------- fp16 helpers
def half_to_float(h: np.ndarray) -> np.ndarray:
    h = _f16(h)
    out = np.empty(h.shape, np.float32)
    lib().oracle_half_to_float(_ptr(h), _ptr(out), h.size)
    return out


def float_to_half(f: np.ndarray) -> np.ndarray:
    f = _f32(f)
    out = np.empty(f.shape, np.float16)
    lib().oracle_float_to_half(_ptr(f), _ptr(out), f.size)
    return out


# ----------------------------------------------------------- the method (fp32)
def quantize_with_scale(x: np.ndarray, scale: float) -> np.ndarray:
    """[Q] section 3: codes of x for one explicit scale."""
    x = _f32(x)
    q = np.empty(x.shape, np.int8)
    lib().oracle_quantize_with_scale(_ptr(x), x.size, float(scale), _ptr(q))
    return q


def ln_stats(h: np.ndarray, eps: float = 1e-5):
    """Exact-sum LayerNorm statistics (mu, rstd) of each row, as float32."""
    h = _f16(h)
    rows, K = h.shape
    mu = np.empty(rows, np.float32)
    rstd = np.empty(rows, np.float32)
    lib().oracle_ln_stats(_ptr(h), rows, K, K, eps, _ptr(mu), _ptr(rstd))
    return mu, rstd


def act_rows(h, gamma=None, beta=None, inv_s=None, eps: float = 1e-5) -> np.ndarray:
    """The fp32 smoothed activation rows x_hat before quantization."""
    h = _f16(h)
    rows, K = h.shape
    gamma, beta, inv_s = _f32(gamma), _f32(beta), _f32(inv_s)
    out = np.empty((rows, K), np.float32)
    lib().oracle_act_rows(_ptr(h), rows, K, K, _ptr(gamma), _ptr(beta), _ptr(inv_s), eps, _ptr(out))
    return out


def calibrate_absmax(x, amax=None, gamma=None, beta=None, eps: float = 1e-5) -> np.ndarray:
    """[SQ] "Calibration": running per-column max of |x| (or of |LN(x)|)."""
    x = _f16(x)
    rows, K = x.shape
    amax = np.zeros(K, np.float32) if amax is None else _f32(amax).copy()
    gamma, beta = _f32(gamma), _f32(beta)
    scratch = np.empty(K, np.float32)
    lib().oracle_calibrate_absmax(_ptr(x), rows, K, K, _ptr(gamma), _ptr(beta), eps, _ptr(amax), _ptr(scratch))
    return amax


def smooth(amax_x, amax_w, alpha: float):
    """[SQ] smoothing factor: s = a^alpha / b^(1-alpha) (fp64, rounded to fp32), inv_s = 1/s."""
    a, b = _f32(amax_x), _f32(amax_w)
    s = np.empty(a.size, np.float32)
    inv_s = np.empty(a.size, np.float32)
    lib().oracle_smooth(_ptr(a), _ptr(b), a.size, float(alpha), _ptr(s), _ptr(inv_s))
    return s, inv_s


def fold_ln(gamma, beta, inv_s):
    """[SQ] fold into the LayerNorm: gamma' = gamma * inv_s, beta' = beta * inv_s."""
    gamma, beta, inv_s = _f32(gamma), _f32(beta), _f32(inv_s)
    K = inv_s.size
    g = np.empty(K, np.float32) if gamma is not None else None
    b = np.empty(K, np.float32) if beta is not None else None
    lib().oracle_fold_ln(_ptr(gamma), _ptr(beta), _ptr(inv_s), K, _ptr(g), _ptr(b))
    return g, b


def fold_weight(w, s) -> np.ndarray:
    """[SQ] fold into the weight: W'[n, j] = fp16(W[n, j] * s_j)."""
    w = _f16(w)
    s = _f32(s)
    N, K = w.shape
    out = np.empty((N, K), np.float16)
    lib().oracle_fold_weight(_ptr(w), N, K, _ptr(s), _ptr(out))
    return out


def quantize_weight(w):
    """Per-output-channel symmetric INT8: (wq [N,K] int8, sw [N] fp32)."""
    w = _f16(w)
    N, K = w.shape
    wq = np.empty((N, K), np.int8)
    sw = np.empty(N, np.float32)
    lib().oracle_quantize_weight(_ptr(w), N, K, _ptr(wq), _ptr(sw))
    return wq, sw


def ln_quant_act(h, gamma=None, beta=None, inv_s=None, eps: float = 1e-5):
    """[SQ] O1 per-token dynamic quantization of x_hat: (xq [M,K] int8, sx [M] fp32)."""
    h = _f16(h)
    M, K = h.shape
    gamma, beta, inv_s = _f32(gamma), _f32(beta), _f32(inv_s)
    xq = np.empty((M, K), np.int8)
    sx = np.empty(M, np.float32)
    scratch = np.empty((max(num_threads(), 1), K), np.float32)
    lib().oracle_ln_quant_act(_ptr(h), M, K, K, _ptr(gamma), _ptr(beta), _ptr(inv_s), eps,
                              _ptr(xq), _ptr(sx), _ptr(scratch))
    return xq, sx


def quantize_weight_tensor(w):
    """[SQ] "inference" levels O1-O3: one scale for the whole weight.
    Returns (wq [N,K] int8, sw [N] fp32 all equal, range fp32)."""
    w = _f16(w)
    N, K = w.shape
    wq = np.empty((N, K), np.int8)
    sw = np.empty(N, np.float32)
    rng = np.zeros(1, np.float32)
    lib().oracle_quantize_weight_tensor(_ptr(w), N, K, _ptr(wq), _ptr(sw), _ptr(rng))
    return wq, sw, rng[0]


def ln_quant_act_tensor(h, gamma=None, beta=None, inv_s=None, eps: float = 1e-5):
    """[SQ] level O2: per-tensor dynamic activation scale over the whole batch.
    Returns (xq [M,K] int8, sx [M] fp32 all equal, range fp32)."""
    h = _f16(h)
    M, K = h.shape
    gamma, beta, inv_s = _f32(gamma), _f32(beta), _f32(inv_s)
    xq = np.empty((M, K), np.int8)
    sx = np.empty(M, np.float32)
    rng = np.zeros(1, np.float32)
    scratch = np.empty(K, np.float32)
    lib().oracle_ln_quant_act_tensor(_ptr(h), M, K, K, _ptr(gamma), _ptr(beta), _ptr(inv_s), eps,
                                     _ptr(xq), _ptr(sx), _ptr(rng), _ptr(scratch))
    return xq, sx, rng[0]


def ln_quant_act_static(h, range_, gamma=None, beta=None, inv_s=None, eps: float = 1e-5):
    """[SQ] level O3: per-tensor static activation scale range_/127 fixed
    offline; values beyond the range saturate.  Returns (xq, sx all equal)."""
    h = _f16(h)
    M, K = h.shape
    gamma, beta, inv_s = _f32(gamma), _f32(beta), _f32(inv_s)
    xq = np.empty((M, K), np.int8)
    sx = np.empty(M, np.float32)
    scratch = np.empty(K, np.float32)
    lib().oracle_ln_quant_act_static(_ptr(h), M, K, K, _ptr(gamma), _ptr(beta), _ptr(inv_s), eps,
                                     float(np.float32(range_)), _ptr(xq), _ptr(sx), _ptr(scratch))
    return xq, sx


def tensor_range(amax, inv_s=None) -> np.float32:
    """Static per-tensor range from calibrated per-channel ranges (level O3)."""
    amax, inv_s = _f32(amax), _f32(inv_s)
    return np.float32(lib().oracle_tensor_range(_ptr(amax), _ptr(inv_s), amax.size))


def int_gemm(xq, wq) -> np.ndarray:
    """[SQ] "INT8 GEMM": acc = xq @ wq^T in int32."""
    xq = np.ascontiguousarray(xq, np.int8)
    wq = np.ascontiguousarray(wq, np.int8)
    M, K = xq.shape
    N = wq.shape[0]
    acc = np.empty((M, N), np.int32)
    lib().oracle_int_gemm(_ptr(xq), _ptr(wq), M, N, K, _ptr(acc))
    return acc


def int_gemm64(xq, wq) -> np.ndarray:
    xq = np.ascontiguousarray(xq, np.int8)
    wq = np.ascontiguousarray(wq, np.int8)
    M, K = xq.shape
    N = wq.shape[0]
    acc = np.empty((M, N), np.int64)
    lib().oracle_int_gemm64(_ptr(xq), _ptr(wq), M, N, K, _ptr(acc))
    return acc


def dequant(acc, sx, sw, bias=None) -> np.ndarray:
    """[Q] multiply the scales back: y = fp16(((float)acc*sx)*sw + bias)."""
    acc = np.ascontiguousarray(acc, np.int32)
    M, N = acc.shape
    sx, sw = _f32(sx), _f32(sw)
    bias = _f16(bias) if bias is not None else None
    y = np.empty((M, N), np.float16)
    lib().oracle_dequant(_ptr(acc), _ptr(sx), _ptr(sw), _ptr(bias), M, N, _ptr(y))
    return y


def w8a8_linear(xq, sx, wq, sw, bias=None) -> np.ndarray:
    """The runtime linear: INT8 GEMM plus dequant epilogue, fp16 [M, N]."""
    xq = np.ascontiguousarray(xq, np.int8)
    wq = np.ascontiguousarray(wq, np.int8)
    M, K = xq.shape
    N = wq.shape[0]
    sx, sw = _f32(sx), _f32(sw)
    bias = _f16(bias) if bias is not None else None
    y = np.empty((M, N), np.float16)
    lib().oracle_w8a8_linear(_ptr(xq), _ptr(sx), _ptr(wq), _ptr(sw), _ptr(bias), M, N, K, _ptr(y))
    return y


def w8a8_linear_quant_static(xq, sx, wq, sw, bias=None, relu=False, inv_s_next=None,
                             range_next=1.0):
    """[SQ] producer-side quantization: the linear, an optional ReLU, the next
    linear's 1/s and its static (level O3) quantization, composed.  Returns
    (q_next [M,N] int8, sx_next [M] fp32 all equal)."""
    xq = np.ascontiguousarray(xq, np.int8)
    wq = np.ascontiguousarray(wq, np.int8)
    M, K = xq.shape
    N = wq.shape[0]
    sx, sw, inv_s_next = _f32(sx), _f32(sw), _f32(inv_s_next)
    bias = _f16(bias) if bias is not None else None
    q = np.empty((M, N), np.int8)
    s_next = np.empty(M, np.float32)
    lib().oracle_w8a8_linear_quant_static(_ptr(xq), _ptr(sx), _ptr(wq), _ptr(sw), _ptr(bias), int(bool(relu)),
                                          _ptr(inv_s_next), float(np.float32(range_next)), M, N, K,
                                          _ptr(q), _ptr(s_next))
    return q, s_next


def w8a8_linear_quant_dynamic(xq, sx, wq, sw, bias=None, relu=False, inv_s_next=None):
    """[SQ] producer-side quantization at the next linear's default level (per-token dynamic
    scale, "inference" O1): the linear, an optional ReLU, the next linear's 1/s, then the
    per-token quantizer -- written as the composition of the pinned steps, so it is exactly
    w8a8_linear, then max(a, 0) on the fp16 values (a NaN becomes 0, as ``y > 0 ? y : 0``),
    then ln_quant_act with inv_s only.  Returns (q_next [M, N] int8, sx_next [M] fp32)."""
    y = w8a8_linear(xq, sx, wq, sw, bias)
    if relu:
        y = np.where(y > 0, y, np.float16(0)).astype(np.float16)
    return ln_quant_act(y, None, None, inv_s_next)


def w8a8_bmm(a, a_scale, b, b_scale) -> np.ndarray:
    """[SQ] INT8 BMM: y[i] = fp16((a[i] @ b[i]^T) * a_scale[i][:, None] * b_scale[i][None, :])."""
    a = np.ascontiguousarray(a, np.int8)
    b = np.ascontiguousarray(b, np.int8)
    B, M, K = a.shape
    N = b.shape[1]
    a_scale, b_scale = _f32(a_scale), _f32(b_scale)
    y = np.empty((B, M, N), np.float16)
    lib().oracle_w8a8_bmm(_ptr(a), _ptr(a_scale), _ptr(b), _ptr(b_scale), B, M, N, K, _ptr(y))
    return y


# ------------------------------------------------------- fp64 mathematics ----
def smooth_fp64(amax_x, amax_w, alpha: float, floor: float = 1e-5) -> np.ndarray:
    """[SQ] s_j = max|X_j|^alpha / max|W_j|^(1-alpha) in exact-as-possible fp64."""
    a = np.maximum(np.asarray(amax_x, np.float64), floor)
    b = np.maximum(np.asarray(amax_w, np.float64), floor)
    return a ** alpha / b ** (1.0 - alpha)


def linear_fp64(x, w, bias=None) -> np.ndarray:
    """Unquantized Y = X W^T (+ b) in fp64; x [M,K], w [N,K]."""
    y = np.asarray(x, np.float64) @ np.asarray(w, np.float64).T
    if bias is not None:
        y = y + np.asarray(bias, np.float64)[None, :]
    return y


def smoothed_linear_fp64(x, w, s) -> np.ndarray:
    """[SQ] (X diag(s)^-1)(diag(s) W^T): mathematically equal to X W^T."""
    s = np.asarray(s, np.float64)
    return (np.asarray(x, np.float64) / s[None, :]) @ (np.asarray(w, np.float64) * s[None, :]).T


def layernorm_fp64(h, gamma, beta, eps: float = 1e-5) -> np.ndarray:
    """Biased-variance LayerNorm in fp64 (for pins of the exact-sum statistics)."""
    h = np.asarray(h, np.float64)
    mu = h.mean(axis=1, keepdims=True)
    var = ((h - mu) ** 2).mean(axis=1, keepdims=True)
    y = (h - mu) / np.sqrt(var + eps)
    if gamma is not None:
        y = y * np.asarray(gamma, np.float64)[None, :]
    if beta is not None:
        y = y + np.asarray(beta, np.float64)[None, :]
    return y


def naive_per_tensor_w8a8(x, w, bias=None) -> np.ndarray:
    """Naive W8A8 with no smoothing: one absmax scale for all of X and one for
    all of W ([SQ] "challenge": the baseline that collapses on large models).
    Quantization in fp64, round half to even; returns the fp64 dequantized
    product.  Quality reference; pinned by the hand-worked
    ``tests/golden/quality_refs_2x3.txt``."""
    x = np.asarray(x, np.float64)
    w = np.asarray(w, np.float64)
    sx = np.abs(x).max() / 127.0
    sw = np.abs(w).max() / 127.0
    qx = np.clip(np.rint(x / sx if sx > 0 else 0 * x), -127, 127)
    qw = np.clip(np.rint(w / sw if sw > 0 else 0 * w), -127, 127)
    y = (qx @ qw.T) * (sx * sw)
    if bias is not None:
        y = y + np.asarray(bias, np.float64)[None, :]
    return y


def per_token_per_channel_w8a8(x, w, bias=None) -> np.ndarray:
    """W8A8 with per-token X scales and per-channel W scales but no smoothing
    (fp64 quantization).  Quality reference; pinned by the hand-worked
    ``tests/golden/quality_refs_2x3.txt`` and by agreeing with the naive
    reference when every row has the same range."""
    x = np.asarray(x, np.float64)
    w = np.asarray(w, np.float64)
    sx = np.abs(x).max(axis=1, keepdims=True) / 127.0
    sw = np.abs(w).max(axis=1, keepdims=True) / 127.0
    with np.errstate(divide="ignore", invalid="ignore"):
        qx = np.clip(np.rint(np.where(sx > 0, x / sx, 0.0)), -127, 127)
        qw = np.clip(np.rint(np.where(sw > 0, w / sw, 0.0)), -127, 127)
    y = (qx @ qw.T) * sx * sw.T
    if bias is not None:
        y = y + np.asarray(bias, np.float64)[None, :]
    return y


# ------------------------------------------------------------ whole step ----
def run_step(calib, w, h, gamma=None, beta=None, bias=None, alpha=0.5, eps=1e-5, amax_x=None):
    """One pass of the whole method, in the pages' order ([SQ] "training
    method" and "inference"): calibrate -> smoothing factor -> fold -> quantize
    the weight -> per-token quantize the activations -> INT8 GEMM + dequant.

    calib, h: fp16 token rows (the LayerNorm input when gamma is given, else
    the linear's input X); w: fp16 [N, K].  With gamma the smoothing is folded
    into the LayerNorm; without it the runtime multiplies by inv_s.
    ``amax_x`` may be passed in to use an already-reduced activation range
    (data-parallel calibration).  Returns every intermediate."""
    out = {}
    out["amax_x"] = calibrate_absmax(calib, gamma=gamma, beta=beta, eps=eps) if amax_x is None else amax_x
    out["amax_w"] = calibrate_absmax(w)
    s, inv_s = smooth(out["amax_x"], out["amax_w"], alpha)
    out["s"], out["inv_s"] = s, inv_s
    if gamma is not None:
        out["gamma_f"], out["beta_f"] = fold_ln(gamma, beta, inv_s)
    else:
        out["gamma_f"], out["beta_f"] = None, None
    out["w_f"] = fold_weight(w, s)
    out["wq"], out["sw"] = quantize_weight(out["w_f"])
    out["xq"], out["sx"] = ln_quant_act(h, out["gamma_f"], out["beta_f"],
                                        None if gamma is not None else inv_s, eps)
    out["y"] = w8a8_linear(out["xq"], out["sx"], out["wq"], out["sw"], bias)
    return out
