"""Reconstruction quality of the oracle's SmoothQuant W8A8 against the
unquantized fp64 product, compared with naive per-tensor W8A8.

The explainer's "challenge" section says naive W8A8 collapses on models with
activation outliers and SmoothQuant does not; it gives no numbers for a single
layer, so the values here are parity unpinned -- only the ordering is checked.
"""
import numpy as np
import pytest

import oracle
import sq_inputs


def _x_fp64(wl, h):
    if wl.ln:
        return oracle.layernorm_fp64(h.astype(np.float64), sq_inputs.gamma(wl), sq_inputs.beta(wl),
                                     eps=float(np.float32(1e-5)))
    return h.astype(np.float64)


def _rel(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


@pytest.mark.parametrize("name", ["tiny", "tiny_ln"])
def test_smoothquant_beats_naive_per_tensor(name):
    wl = sq_inputs.WORKLOADS[name]
    calib, h, w = sq_inputs.calib_rows(wl), sq_inputs.run_rows(wl), sq_inputs.weight(wl)
    b16 = sq_inputs.bias(wl)
    r = oracle.run_step(calib, w, h, sq_inputs.gamma(wl), sq_inputs.beta(wl), b16, wl.alpha)
    X = _x_fp64(wl, h)
    bias = None if b16 is None else b16.astype(np.float64)
    y64 = oracle.linear_fp64(X, w.astype(np.float64), bias)
    e_sq = _rel(r["y"].astype(np.float64), y64)
    e_naive = _rel(oracle.naive_per_tensor_w8a8(X, w.astype(np.float64), bias), y64)
    e_tok = _rel(oracle.per_token_per_channel_w8a8(X, w.astype(np.float64), bias), y64)
    assert e_sq < e_naive, (e_sq, e_naive)
    assert e_sq < e_tok, (e_sq, e_tok)
    assert e_sq < 0.05


def test_alpha_moves_difficulty_to_weights():
    # "smoothing factor": a larger alpha flattens activations more and loads the weights more.
    wl = sq_inputs.WORKLOADS["tiny"]
    calib, w = sq_inputs.calib_rows(wl), sq_inputs.weight(wl)
    ax = oracle.calibrate_absmax(calib)
    aw = oracle.calibrate_absmax(w)
    spread_x, spread_w = [], []
    for alpha in (0.0, 0.25, 0.5, 0.75, 1.0):
        s, inv_s = oracle.smooth(ax, aw, alpha)
        xm = ax.astype(np.float64) * inv_s
        wm = np.abs(oracle.fold_weight(w, s).astype(np.float64)).max(0)
        spread_x.append(xm.max() / np.median(xm))
        spread_w.append(wm.max() / np.median(wm))
    assert all(a > b for a, b in zip(spread_x, spread_x[1:]))
    assert all(a < b for a, b in zip(spread_w, spread_w[1:]))
