"""The quantization levels of the explainer (section "inference": O1 per-token
activations and per-tensor weights, O2 per-tensor dynamic, O3 per-tensor
static) on the GPU against the oracle, bit for bit: per-tensor weight
quantization (with the fold), the O2 two-pass activation quantization, the O3
one-pass static quantization with saturation, the static range from
calibrated channel ranges, and the whole layer at each level.  Shapes cover
every row-kernel shape (warp per row, register-resident CTA rows, CTA rows
re-read from global) with ragged row counts."""
import numpy as np
import pytest
import torch

import oracle
import sq_inputs
from gpu_util import bits_equal, dev, f16_within, host

pytestmark = pytest.mark.gpu

ACT_SHAPES = [(1, 16, "plain"), (37, 256, "inv_s"), (19, 1024, "ln"), (33, 4096, "ln"),
              (9, 20480, "inv_s"), (5, 49152, "ln_inv_s"), (3, 65536, "inv_s")]


@pytest.fixture(scope="module")
def sq(cuda_device):
    import w8a8_int8_linear_channel_b200 as m
    return m


def _act_inputs(M, K, mode, seed):
    rng = np.random.default_rng(seed)
    h = (rng.standard_normal((M, K)) + 0.2).astype(np.float32)
    h[:, [2, K - 3]] *= 60.0
    h = h.astype(np.float16)
    g = b = inv = None
    if "ln" in mode:
        g = rng.uniform(0.5, 2.0, K).astype(np.float32)
        g[[2, K - 3]] = 70.0
        b = (rng.standard_normal(K) * 0.01).astype(np.float32)
    if "inv_s" in mode:
        inv = rng.uniform(0.02, 2.0, K).astype(np.float32)
    return h, g, b, inv


def _f32(n=1):
    return torch.zeros(n, dtype=torch.float32, device="cuda")


@pytest.mark.parametrize("M,K,mode", ACT_SHAPES)
def test_o2_per_tensor_dynamic(sq, M, K, mode):
    h, g, b, inv = _act_inputs(M, K, mode, M * 7 + K)
    xq = torch.empty((M, K), dtype=torch.int8, device="cuda")
    sx = torch.empty(M, dtype=torch.float32, device="cuda")
    rng_ = _f32()
    rng_.fill_(1e30)  # the entry point clears it itself
    sq.sq_ln_quant_act_tensor(dev(h), xq, sx, rng_, dev(g), dev(b), dev(inv))
    q_ref, s_ref, r_ref = oracle.ln_quant_act_tensor(h, g, b, inv)
    assert bits_equal(host(rng_), np.float32(r_ref).reshape(1))
    assert bits_equal(host(sx), s_ref)
    assert bits_equal(host(xq), q_ref)
    assert sq.sq_poll_status() == 0


@pytest.mark.parametrize("M,K,mode", ACT_SHAPES)
def test_o3_per_tensor_static_saturates(sq, M, K, mode):
    h, g, b, inv = _act_inputs(M, K, mode, M * 11 + K)
    x = oracle.act_rows(h, g, b, inv)
    r = np.float32(np.abs(x).max() * 0.4)  # calibration saw less than this batch: saturation
    xq = torch.empty((M, K), dtype=torch.int8, device="cuda")
    sx = torch.empty(M, dtype=torch.float32, device="cuda")
    sq.sq_ln_quant_act_static(dev(h), xq, sx, dev(np.array([r], np.float32)), dev(g), dev(b), dev(inv))
    q_ref, s_ref = oracle.ln_quant_act_static(h, r, g, b, inv)
    assert (np.abs(q_ref) == 127).sum() >= 1
    assert bits_equal(host(sx), s_ref)
    assert bits_equal(host(xq), q_ref)


@pytest.mark.parametrize("N,K,fold", [(1, 16, False), (77, 48, True), (300, 4112, True),
                                      (40, 16400, True), (13, 49152, True), (6, 65536, False)])
def test_per_tensor_weight(sq, N, K, fold):
    rng = np.random.default_rng(N * 3 + K)
    w = (rng.standard_normal((N, K)) * 0.02).astype(np.float16)
    w[min(3, N - 1)] = 0
    s = rng.uniform(0.05, 20, K).astype(np.float32) if fold else None
    wq = torch.empty((N, K), dtype=torch.int8, device="cuda")
    sw = torch.empty(N, dtype=torch.float32, device="cuda")
    r = _f32()
    sq.sq_quantize_weight_tensor(dev(w), wq, sw, r, s=dev(s))
    w_ref = oracle.fold_weight(w, s) if fold else w
    wq_ref, sw_ref, r_ref = oracle.quantize_weight_tensor(w_ref)
    assert bits_equal(host(r), np.float32(r_ref).reshape(1))
    assert bits_equal(host(sw), sw_ref)
    assert bits_equal(host(wq), wq_ref)


@pytest.mark.parametrize("K", [16, 4096, 133136])
@pytest.mark.parametrize("with_inv_s", [False, True])
def test_tensor_range(sq, K, with_inv_s):
    rng = np.random.default_rng(K + with_inv_s)
    amax = rng.uniform(0, 50, K).astype(np.float32)
    inv = rng.uniform(0.01, 3, K).astype(np.float32) if with_inv_s else None
    r = _f32()
    sq.sq_tensor_range(dev(amax), r, inv_s=dev(inv))
    assert bits_equal(host(r), np.float32(oracle.tensor_range(amax, inv)).reshape(1))


@pytest.mark.parametrize("level", ["channel", "O1", "O2", "O3"])
@pytest.mark.parametrize("wl_name", ["tiny", "tiny_ln"])
def test_layer_at_each_level(sq, level, wl_name):
    """SmoothQuantLinear at each level against the oracle chain of the same
    level (stagewise on the GPU's smoothing factor, which goes through pow)."""
    wl = sq_inputs.WORKLOADS[wl_name]
    w, calib = sq_inputs.weight(wl), sq_inputs.calib_rows(wl)
    h = sq_inputs.run_rows(wl, 0, wl.M)
    g, b, bias = sq_inputs.gamma(wl), sq_inputs.beta(wl), sq_inputs.bias(wl)
    layer = sq.SmoothQuantLinear.from_float(dev(w), dev(calib), alpha=wl.alpha, gamma=dev(g),
                                            beta=dev(b), bias=dev(bias), level=level)
    y = host(layer(dev(h)))
    act_mode, w_mode = sq.LEVELS[level]
    s = host(layer.s)  # the GPU's smoothing factor (checked against the oracle elsewhere)
    inv_s = (np.float32(1) / s).astype(np.float32)
    assert bits_equal(host(layer.smooth_inv), inv_s)
    gf, bf = oracle.fold_ln(g, b, inv_s) if g is not None else (None, None)
    rt_inv = None if g is not None else inv_s
    w_f = oracle.fold_weight(w, s)
    if w_mode == "tensor":
        wq_ref, sw_ref, _ = oracle.quantize_weight_tensor(w_f)
    else:
        wq_ref, sw_ref = oracle.quantize_weight(w_f)
    assert bits_equal(host(layer.wq), wq_ref) and bits_equal(host(layer.w_scale), sw_ref)
    if act_mode == "token":
        xq_ref, sx_ref = oracle.ln_quant_act(h, gf, bf, rt_inv)
    elif act_mode == "tensor":
        xq_ref, sx_ref, _ = oracle.ln_quant_act_tensor(h, gf, bf, rt_inv)
    else:
        if g is not None:
            r = oracle.tensor_range(oracle.calibrate_absmax(calib, gamma=gf, beta=bf))
        else:
            r = oracle.tensor_range(oracle.calibrate_absmax(calib), inv_s)
        assert bits_equal(host(layer.act_range), np.float32(r).reshape(1))
        xq_ref, sx_ref = oracle.ln_quant_act_static(h, r, gf, bf, rt_inv)
    y_ref = oracle.w8a8_linear(xq_ref, sx_ref, wq_ref, sw_ref, bias)
    assert f16_within(y, y_ref)
    assert bits_equal(y, y_ref)


def test_o2_full_size_attention_batch(sq):
    """O2 at the attention-projection size (2048 x 4096, LayerNorm folded)."""
    wl = sq_inputs.WORKLOADS["attn"]
    h = sq_inputs.run_rows(wl, 0, wl.M)
    g, b = sq_inputs.gamma(wl), sq_inputs.beta(wl)
    xq = torch.empty((wl.M, wl.K), dtype=torch.int8, device="cuda")
    sx = torch.empty(wl.M, dtype=torch.float32, device="cuda")
    r = _f32()
    sq.sq_ln_quant_act_tensor(dev(h), xq, sx, r, dev(g), dev(b))
    q_ref, s_ref, r_ref = oracle.ln_quant_act_tensor(h, g, b)
    assert bits_equal(host(r), np.float32(r_ref).reshape(1))
    assert bits_equal(host(sx), s_ref)
    assert bits_equal(host(xq), q_ref)


def test_layer_batch_shapes(sq):
    """Leading dimensions are flattened into tokens (same bits as the 2-D call);
    an empty batch returns an empty output and launches nothing."""
    wl = sq_inputs.WORKLOADS["tiny_ln"]
    w, calib = sq_inputs.weight(wl), sq_inputs.calib_rows(wl)
    g, b, bias = sq_inputs.gamma(wl), sq_inputs.beta(wl), sq_inputs.bias(wl)
    layer = sq.SmoothQuantLinear.from_float(dev(w), dev(calib), alpha=wl.alpha, gamma=dev(g), beta=dev(b),
                                            bias=dev(bias))
    h = sq_inputs.run_rows(wl, 0, 12)
    y2 = host(layer(dev(h)))
    y3 = layer(dev(h).view(3, 4, wl.K))
    assert tuple(y3.shape) == (3, 4, wl.N) and bits_equal(host(y3).reshape(12, wl.N), y2)
    out = torch.empty((3, 4, wl.N), dtype=torch.float16, device="cuda")
    assert layer(dev(h).view(3, 4, wl.K), out) is out and bits_equal(host(out).reshape(12, wl.N), y2)
    for shape in [(0, wl.K), (2, 0, wl.K)]:
        e = layer(torch.empty(shape, dtype=torch.float16, device="cuda"))
        assert tuple(e.shape) == shape[:-1] + (wl.N,)
    with pytest.raises(ValueError):
        layer(dev(h)[:, :16])
    assert sq.sq_poll_status() == 0
