"""Non-finite inputs on the GPU against the oracle, bit for bit.

IEEE arithmetic decides every case: a LayerNorm row holding an Inf or a NaN
has NaN statistics, so its whole output is NaN; a NaN never wins a maximum;
a NaN product is quantized to 0; an infinite range gives an infinite scale,
a zero reciprocal and therefore codes 0.  Every row-kernel shape is covered
(warp per row, register-resident CTA rows, CTA rows held in registers beyond
eight chunks, CTA rows re-read from global, and at 300 x 12288 the bulk-copy
rows of eight warps, where CTAs take two rows each and the LayerNorm loop runs
one row deep, a non-finite row next to a finite one), with calibration, weight
quantization (with and without the fold), the per-tensor levels, the fused
producer-side quantization and the dequant epilogue."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import bits_equal, dev, host

pytestmark = pytest.mark.gpu

SHAPES = [(6, 256), (5, 1024), (7, 4096), (300, 12288), (5, 20480), (5, 65536)]


@pytest.fixture(scope="module")
def sq(cuda_device):
    import w8a8_int8_linear_channel_b200 as m
    return m


def _rows(M, K, seed):
    """fp16 rows: row 1 +Inf, row 2 NaN, row 3 -Inf, row 4 both (when present);
    the others finite, with a few large channels."""
    rng = np.random.default_rng(seed)
    h = (rng.standard_normal((M, K)) + 0.1).astype(np.float32)
    h[:, [1, K - 2]] *= 50.0
    h = h.astype(np.float16)
    cols = rng.integers(0, K, 4)
    if M > 1:
        h[1, cols[0]] = np.inf
    if M > 2:
        h[2, cols[1]] = np.nan
    if M > 3:
        h[3, cols[2]] = -np.inf
    if M > 4:
        h[4, cols[3]] = np.inf
        h[4, (cols[3] + 7) % K] = np.nan
    return h


def _vecs(K, mode, seed):
    rng = np.random.default_rng(seed)
    g = b = inv = None
    if "ln" in mode:
        g = rng.uniform(0.5, 2.0, K).astype(np.float32)
        b = (rng.standard_normal(K) * 0.05).astype(np.float32)
    if "inv_s" in mode:
        inv = rng.uniform(0.05, 2.0, K).astype(np.float32)
    return g, b, inv


@pytest.mark.parametrize("M,K", SHAPES)
@pytest.mark.parametrize("mode", ["plain", "inv_s", "ln", "ln_inv_s"])
def test_activation_quantization(sq, M, K, mode):
    h = _rows(M, K, M + K)
    g, b, inv = _vecs(K, mode, K)
    xq = torch.empty((M, K), dtype=torch.int8, device="cuda")
    sx = torch.empty(M, dtype=torch.float32, device="cuda")
    sq.sq_ln_quant_act(dev(h), xq, sx, dev(g), dev(b), dev(inv))
    q_ref, s_ref = oracle.ln_quant_act(h, g, b, inv)
    if "ln" in mode:  # the non-finite rows: scale 0, codes 0
        bad = slice(1, min(M, 5))
        assert (s_ref[bad] == 0).all() and not q_ref[bad].any()
    assert bits_equal(host(sx), s_ref)
    assert bits_equal(host(xq), q_ref)
    assert sq.sq_poll_status() == 0


@pytest.mark.parametrize("M,K", SHAPES)
@pytest.mark.parametrize("ln", [False, True])
def test_calibration(sq, M, K, ln):
    h = _rows(M, K, 3 * M + K)
    g, b, _ = _vecs(K, "ln" if ln else "plain", 2 * K)
    a0 = np.abs(np.random.default_rng(K).standard_normal(K)).astype(np.float32)  # running maxima
    amax = dev(a0.copy())
    sq.sq_calibrate_absmax(dev(h), amax, dev(g), dev(b))
    ref = oracle.calibrate_absmax(h, a0, g, b)
    assert bits_equal(host(amax), ref)


@pytest.mark.parametrize("N,K", SHAPES)
@pytest.mark.parametrize("fold", [False, True])
def test_weight_quantization(sq, N, K, fold):
    w = _rows(N, K, 5 * N + K)
    s = np.random.default_rng(N).uniform(0.1, 8.0, K).astype(np.float32) if fold else None
    wq = torch.empty((N, K), dtype=torch.int8, device="cuda")
    sw = torch.empty(N, dtype=torch.float32, device="cuda")
    sq.sq_quantize_weight(dev(w), wq, sw, s=dev(s))
    wq_ref, sw_ref = oracle.quantize_weight(oracle.fold_weight(w, s) if fold else w)
    assert bits_equal(host(sw), sw_ref)
    assert bits_equal(host(wq), wq_ref)


@pytest.mark.parametrize("M,K", [(5, 1024), (7, 4096), (5, 20480)])
@pytest.mark.parametrize("mode", ["plain", "ln"])
def test_per_tensor_levels(sq, M, K, mode):
    h = _rows(M, K, 7 * M + K)
    h_nan = h.copy()
    h_nan[1] = 0.5  # O2 with a NaN but no Inf: a finite range
    h_nan[3] = -0.25
    h_nan[4] = 0.125
    g, b, inv = _vecs(K, mode, 3 * K)
    for rows in (h, h_nan):
        xq = torch.empty((M, K), dtype=torch.int8, device="cuda")
        sx = torch.empty(M, dtype=torch.float32, device="cuda")
        r = torch.zeros(1, dtype=torch.float32, device="cuda")
        sq.sq_ln_quant_act_tensor(dev(rows), xq, sx, r, dev(g), dev(b), dev(inv))
        q_ref, s_ref, r_ref = oracle.ln_quant_act_tensor(rows, g, b, inv)
        assert bits_equal(host(r), np.float32(r_ref).reshape(1))
        assert bits_equal(host(sx), s_ref) and bits_equal(host(xq), q_ref)
    # O3: a static range, so +-Inf saturate and NaN codes 0
    r3 = np.float32(3.0)
    xq = torch.empty((M, K), dtype=torch.int8, device="cuda")
    sx = torch.empty(M, dtype=torch.float32, device="cuda")
    sq.sq_ln_quant_act_static(dev(h), xq, sx, dev(np.array([r3], np.float32)), dev(g), dev(b), dev(inv))
    q_ref, s_ref = oracle.ln_quant_act_static(h, r3, g, b, inv)
    assert bits_equal(host(sx), s_ref) and bits_equal(host(xq), q_ref)
    # per-tensor weight (no LayerNorm on a weight)
    wq = torch.empty((M, K), dtype=torch.int8, device="cuda")
    sw = torch.empty(M, dtype=torch.float32, device="cuda")
    rw = torch.zeros(1, dtype=torch.float32, device="cuda")
    sq.sq_quantize_weight_tensor(dev(h_nan), wq, sw, rw)
    wq_ref, sw_ref, rw_ref = oracle.quantize_weight_tensor(h_nan)
    assert bits_equal(host(rw), np.float32(rw_ref).reshape(1))
    assert bits_equal(host(sw), sw_ref) and bits_equal(host(wq), wq_ref)


def _gemm_inputs(M, N, K, seed):
    rng = np.random.default_rng(seed)
    xq = rng.integers(-127, 128, (M, K)).astype(np.int8)
    wq = rng.integers(-127, 128, (N, K)).astype(np.int8)
    xq[M // 2] = 0  # a zero row: 0 * Inf below gives NaN
    sx = rng.uniform(1e-4, 1e-3, M).astype(np.float32)
    sw = rng.uniform(1e-4, 1e-3, N).astype(np.float32)
    sw[[1, N - 2]] = np.nan
    sw[N // 2] = np.inf
    sx[M - 1] = np.inf
    bias = (rng.standard_normal(N) * 0.1).astype(np.float16)
    return xq, sx, wq, sw, bias


@pytest.mark.parametrize("M", [16, 300])
@pytest.mark.parametrize("relu", [False, True])
def test_producer_quantization_of_non_finite_outputs(sq, M, relu):
    N, K = 272, 512  # N: the next linear's K, a multiple of 16
    xq, sx, wq, sw, bias = _gemm_inputs(M, N, K, M + relu)
    inv = np.random.default_rng(M).uniform(0.2, 3.0, N).astype(np.float32)
    r = np.float32(2.0)
    q = torch.empty((M, N), dtype=torch.int8, device="cuda")
    s = torch.empty(M, dtype=torch.float32, device="cuda")
    sq.sq_w8a8_linear_quant(dev(xq), dev(sx), dev(wq), dev(sw), dev(np.array([r], np.float32)), q, s,
                            bias=dev(bias), relu=relu, inv_s_next=dev(inv), workspace=sq.new_workspace(M, N, K))
    q_ref, s_ref = oracle.w8a8_linear_quant_static(xq, sx, wq, sw, bias, relu=relu, inv_s_next=inv,
                                                   range_next=r)
    assert bits_equal(host(s), s_ref)
    assert bits_equal(host(q), q_ref)
    assert sq.sq_poll_status() == 0


@pytest.mark.parametrize("M,path", [(16, "splitk"), (100, "tiled"), (300, "pair")])
def test_dequant_of_non_finite_scales(sq, M, path):
    N, K = 264, 512
    xq, sx, wq, sw, bias = _gemm_inputs(M, N, K, 11 * M)
    p = {"splitk": sq.PATH_SPLITK, "tiled": sq.PATH_TILED, "pair": sq.PATH_PAIR}[path]
    y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    sq.sq_w8a8_linear(dev(xq), dev(sx), dev(wq), dev(sw), y, dev(bias), workspace=sq.new_workspace(M, N, K),
                      path=p)
    ref = oracle.w8a8_linear(xq, sx, wq, sw, bias)
    got = host(y)
    nan = np.isnan(ref)
    assert nan.any() and np.isinf(ref).any()
    # NaN payloads are not part of the contract; every other value is bit-exact
    assert np.array_equal(np.isnan(got), nan)
    assert bits_equal(got[~nan], ref[~nan])
