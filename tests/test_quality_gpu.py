"""Reconstruction quality of the CUDA path on the four OPT-shaped outlier workloads, full
layers (every output channel), on sampled token rows.

The SmoothQuant explainer ("challenge", "why activations are hard to quantize") predicts that
naive per-tensor W8A8 collapses on persistent activation outliers while the smoothed layer
does not.  The pages give no numbers for one layer, so only that ordering is asserted; the
values are unpinned.  The smoothed layer runs through the public API
(SmoothQuantLinear.from_float + forward); the two unsmoothed baselines through the library's
own entry points (per-tensor: level O2 activations and a per-tensor weight; per token / per
channel: sq_ln_quant_act and sq_quantize_weight, both without smoothing).  The reference is
the unquantized fp64 X W^T (+ b), with X the fp64 LayerNorm of h where the workload has one.
"""
import numpy as np
import pytest
import torch

import oracle
import sq_inputs
from gpu_util import dev, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sq(cuda_device):
    import w8a8_int8_linear_channel_b200 as m
    return m


def _y64(wl, h, w, b16):
    X = (oracle.layernorm_fp64(h, sq_inputs.gamma(wl), sq_inputs.beta(wl), eps=float(np.float32(1e-5)))
         if wl.ln else h.astype(np.float64))
    Y = np.empty((h.shape[0], w.shape[0]), np.float64)
    for n0 in range(0, w.shape[0], 2048):  # fp64 copies of 2048 weight rows at a time
        Y[:, n0:n0 + 2048] = oracle.linear_fp64(X, w[n0:n0 + 2048])
    if b16 is not None:
        Y += b16.astype(np.float64)[None, :]
    return Y


def _unsmoothed(sq, h, w, g, b, bias, per_tensor):
    m, K = h.shape
    N = w.shape[0]
    xq = torch.empty((m, K), dtype=torch.int8, device="cuda")
    sx = torch.empty(m, dtype=torch.float32, device="cuda")
    wq = torch.empty((N, K), dtype=torch.int8, device="cuda")
    sw = torch.empty(N, dtype=torch.float32, device="cuda")
    if per_tensor:
        r = torch.zeros(8, dtype=torch.float32, device="cuda")
        sq.sq_ln_quant_act_tensor(h, xq, sx, r[:1], g, b)
        sq.sq_quantize_weight_tensor(w, wq, sw, r[4:5])
    else:
        sq.sq_ln_quant_act(h, xq, sx, g, b)
        sq.sq_quantize_weight(w, wq, sw)
    y = torch.empty((m, N), dtype=torch.float16, device="cuda")
    sq.sq_w8a8_linear(xq, sx, wq, sw, y, bias, workspace=sq.new_workspace(m, N, K))
    return host(y)


def _rel(y, Y):
    return float(np.linalg.norm(y.astype(np.float64) - Y) / np.linalg.norm(Y))


@pytest.mark.parametrize("name,m", [("attn", 64), ("ffn_up", 32), ("decode", 32), ("ffn_down", 16)])
def test_quality_full_layer(sq, name, m):
    wl = sq_inputs.WORKLOADS[name]
    w = sq_inputs.weight(wl)
    calib = sq_inputs.calib_rows(wl)
    h = sq_inputs.run_rows(wl, 0, min(m, wl.M))
    b16 = sq_inputs.bias(wl)
    g, b = sq_inputs.gamma(wl), sq_inputs.beta(wl)
    wt, ht = dev(w), dev(h)
    layer = sq.SmoothQuantLinear.from_float(wt, dev(calib), wl.alpha, dev(g), dev(b), dev(b16))
    y_sq = host(layer(ht))
    y_naive = _unsmoothed(sq, ht, wt, dev(g), dev(b), dev(b16), True)
    y_tok = _unsmoothed(sq, ht, wt, dev(g), dev(b), dev(b16), False)
    assert sq.sq_poll_status() == 0
    Y = _y64(wl, h, w, b16)
    e_sq, e_naive, e_tok = _rel(y_sq, Y), _rel(y_naive, Y), _rel(y_tok, Y)
    print(f"{name}: e_sq {e_sq:.4g}  e_naive_per_tensor {e_naive:.4g}  e_per_token_per_channel {e_tok:.4g}")
    assert e_sq < e_naive, (name, e_sq, e_naive)
