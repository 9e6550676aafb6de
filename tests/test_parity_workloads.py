"""The whole path at the full workload sizes, in the launch configuration the
benchmark times, checked against the oracle on sampled outputs.

Stagewise: each oracle stage takes the GPU's previous-stage output, so the
calibration ranges, folded LayerNorm vectors, weight codes and scales,
activation codes and scales, int32 accumulators and fp16 outputs are all
compared bit for bit (the smoothing factor, which goes through pow, within
1 fp32 ulp).  The samples are whole rows: token rows of X/Y and weight rows
spread over every 128-row tile.
"""
import numpy as np
import pytest
import torch

import oracle
import sq_inputs
from gpu_util import bits_equal, f16_within, ulps32

pytestmark = pytest.mark.gpu


def _T(a):
    return None if a is None else torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _run_path(sq, wl, M, alpha):
    """The benchmark's step through the binding; returns host copies of every stage."""
    w = sq_inputs.weight(wl)
    calib = sq_inputs.calib_rows(wl)
    h = sq_inputs.run_rows(wl, 0, M)
    g, b, bias = sq_inputs.gamma(wl), sq_inputs.beta(wl), sq_inputs.bias(wl)
    K, N = wl.K, wl.N
    dw, dcal, dh, dg, db, dbias = _T(w), _T(calib), _T(h), _T(g), _T(b), _T(bias)
    ax = torch.zeros(K, dtype=torch.float32, device="cuda")
    aw = torch.zeros(K, dtype=torch.float32, device="cuda")
    sq.sq_calibrate_absmax(dcal, ax, dg, db)
    sq.sq_calibrate_absmax(dw, aw)
    s = torch.empty(K, device="cuda")
    inv_s = torch.empty(K, device="cuda")
    gf = torch.empty(K, device="cuda") if g is not None else None
    bf = torch.empty(K, device="cuda") if b is not None else None
    sq.sq_smooth_fold(ax, aw, alpha, s, inv_s, dg, db, gf, bf)
    wq = torch.empty((N, K), dtype=torch.int8, device="cuda")
    sw = torch.empty(N, device="cuda")
    sq.sq_quantize_weight(dw, wq, sw, s=s)
    xq = torch.empty((M, K), dtype=torch.int8, device="cuda")
    sx = torch.empty(M, device="cuda")
    sq.sq_ln_quant_act(dh, xq, sx, gf, bf, None if g is not None else inv_s)
    y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    ws = sq.new_workspace(M, N, K)
    sq.sq_w8a8_linear(xq, sx, wq, sw, y, dbias, workspace=ws)
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    sq.sq_w8a8_gemm_s32(xq, wq, acc, workspace=ws)
    torch.cuda.synchronize()
    assert sq.sq_poll_status() == 0
    out = {k: (None if v is None else v.cpu().numpy()) for k, v in dict(
        ax=ax, aw=aw, s=s, inv_s=inv_s, gf=gf, bf=bf, wq=wq, sw=sw, xq=xq, sx=sx, y=y, acc=acc).items()}
    out.update(w=w, calib=calib, h=h, g=g, b=b, bias=bias)
    return out


def _weight_sample(N, per_tile=4, seed=0):
    rng = np.random.default_rng(seed)
    rows = []
    for t in range(0, N, 128):
        hi = min(N, t + 128)
        rows += [t, hi - 1] + list(rng.integers(t, hi, per_tile - 2))
    return np.unique(np.asarray(rows))


def _check(r, wl, M, alpha, token_rows, weight_rows):
    # calibration: exact over the whole calibration set and the whole weight
    assert bits_equal(r["ax"], oracle.calibrate_absmax(r["calib"], gamma=r["g"], beta=r["b"]))
    assert bits_equal(r["aw"], oracle.calibrate_absmax(r["w"]))
    s_ref, _ = oracle.smooth(r["ax"], r["aw"], alpha)
    assert ulps32(r["s"], s_ref).max() <= 1
    assert bits_equal(r["inv_s"], (np.float32(1) / r["s"]).astype(np.float32))
    if r["g"] is not None:
        gf, bf = oracle.fold_ln(r["g"], r["b"], r["inv_s"])
        assert bits_equal(r["gf"], gf) and bits_equal(r["bf"], bf)
    # weight codes on sampled rows of every tile
    wq_ref, sw_ref = oracle.quantize_weight(oracle.fold_weight(r["w"][weight_rows], r["s"]))
    assert bits_equal(r["wq"][weight_rows], wq_ref)
    assert bits_equal(r["sw"][weight_rows], sw_ref)
    # activation codes on sampled tokens
    h = r["h"][token_rows]
    if r["g"] is not None:
        xq_ref, sx_ref = oracle.ln_quant_act(h, r["gf"], r["bf"])
    else:
        xq_ref, sx_ref = oracle.ln_quant_act(h, inv_s=r["inv_s"])
    assert bits_equal(r["xq"][token_rows], xq_ref)
    assert bits_equal(r["sx"][token_rows], sx_ref)
    # accumulators and outputs of the sampled tokens against every channel
    xq_s, sx_s = r["xq"][token_rows], r["sx"][token_rows]
    acc_ref = oracle.int_gemm(xq_s, r["wq"])
    assert np.array_equal(r["acc"][token_rows], acc_ref)
    y_ref = oracle.w8a8_linear(xq_s, sx_s, r["wq"], r["sw"], r["bias"])
    assert f16_within(r["y"][token_rows], y_ref)
    assert bits_equal(r["y"][token_rows], y_ref)


@pytest.fixture(scope="module")
def sq(cuda_device):
    import w8a8_int8_linear_channel_b200 as m
    return m


@pytest.mark.parametrize("name", ["attn", "ffn_up"])
def test_full_size_large_m(sq, name):
    wl = sq_inputs.WORKLOADS[name]
    r = _run_path(sq, wl, wl.M, wl.alpha)
    tokens = np.unique(np.r_[0, 1, 127, 128, 255, 256, wl.M - 1, np.random.default_rng(1).integers(0, wl.M, 5)])
    _check(r, wl, wl.M, wl.alpha, tokens, _weight_sample(wl.N, per_tile=2))


@pytest.mark.parametrize("M", sq_inputs.DECODE_M)
def test_full_size_decode(sq, M):
    wl = sq_inputs.WORKLOADS["decode"]
    r = _run_path(sq, wl, M, wl.alpha)
    # every token against sampled channels of every tile: y and acc columns
    cols = _weight_sample(wl.N, per_tile=3, seed=M)
    _check_decode(r, wl, M, cols)


def _check_decode(r, wl, M, cols):
    assert bits_equal(r["ax"], oracle.calibrate_absmax(r["calib"], gamma=r["g"], beta=r["b"]))
    assert bits_equal(r["aw"], oracle.calibrate_absmax(r["w"]))
    s_ref, _ = oracle.smooth(r["ax"], r["aw"], wl.alpha)
    assert ulps32(r["s"], s_ref).max() <= 1
    wq_ref, sw_ref = oracle.quantize_weight(oracle.fold_weight(r["w"][cols], r["s"]))
    assert bits_equal(r["wq"][cols], wq_ref) and bits_equal(r["sw"][cols], sw_ref)
    xq_ref, sx_ref = oracle.ln_quant_act(r["h"], r["gf"], r["bf"])
    assert bits_equal(r["xq"], xq_ref) and bits_equal(r["sx"], sx_ref)
    acc_ref = oracle.int_gemm(r["xq"], r["wq"][cols])
    assert np.array_equal(r["acc"][:, cols], acc_ref)
    y_ref = oracle.w8a8_linear(r["xq"], r["sx"], r["wq"][cols], r["sw"][cols], None)
    assert bits_equal(r["y"][:, cols], y_ref)


@pytest.mark.parametrize("alpha", sq_inputs.FFN_DOWN_ALPHAS)
def test_full_size_ffn_down(sq, alpha):
    wl = sq_inputs.WORKLOADS["ffn_down"]
    r = _run_path(sq, wl, wl.M, alpha)
    tokens = np.array([0, 4095, wl.M - 1])
    _check(r, wl, wl.M, alpha, tokens, _weight_sample(wl.N, per_tile=2, seed=3))


@pytest.mark.parametrize("path", ["auto", "pair"])
def test_persistent_gemm_more_tiles_than_sms(sq, path):
    # 6 x 26 = 156 tiles of 256 x 256 on 148 SMs (74 CTA pairs), ragged M, N and K
    p = {"auto": sq.PATH_AUTO, "pair": sq.PATH_PAIR}[path]
    rng = np.random.default_rng(99)
    M, N, K = 1300, 6500, 272
    xq = rng.integers(-127, 128, (M, K)).astype(np.int8)
    wq = rng.integers(-127, 128, (N, K)).astype(np.int8)
    sx = rng.uniform(1e-4, 1e-2, M).astype(np.float32)
    sw = rng.uniform(1e-4, 1e-2, N).astype(np.float32)
    bias = (rng.standard_normal(N) * 0.1).astype(np.float16)
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    sq.sq_w8a8_gemm_s32(_T(xq), _T(wq), acc, path=p)
    assert np.array_equal(acc.cpu().numpy(), oracle.int_gemm(xq, wq))
    y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    sq.sq_w8a8_linear(_T(xq), _T(sx), _T(wq), _T(sw), y, _T(bias), path=p)
    assert bits_equal(y.cpu().numpy(), oracle.w8a8_linear(xq, sx, wq, sw, bias))
