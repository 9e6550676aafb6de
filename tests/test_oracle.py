"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: a worked
example printed on a page, a hand-worked example whose every value is exact,
a closed form, a library routine on a special case, or brute force.
"""
import numpy as np
import pytest

import oracle
from golden_io import load

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def f16(a):
    return np.asarray(a, np.float64).astype(np.float16)


def ulp32(x):
    x = np.abs(np.asarray(x, np.float32))
    return np.spacing(x)


# ------------------------------------------------------------------ fp16 ----
def test_half_to_float_all_bit_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    h = bits.view(np.float16)
    got = oracle.half_to_float(h)
    want = h.astype(np.float32)
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), want[~nan].view(np.uint32))


def test_float_to_half_round_to_nearest_even():
    rng = np.random.default_rng(1)
    f = np.concatenate([
        rng.standard_normal(200000).astype(np.float32) * np.float32(1000),
        rng.standard_normal(20000).astype(np.float32) * np.float32(1e-5),
        # exact midpoints between neighbouring fp16 values: ties must go to even
        ((np.arange(1, 4000, dtype=np.float32) + np.float32(0.5)) * np.float32(2.0 ** -3)),
        np.array([65504, 65519.99, 65520, 1e9, -1e9, 2 ** -25, 3 * 2 ** -26], np.float32),
    ])
    got = oracle.float_to_half(f)
    want = f.astype(np.float16)
    assert np.array_equal(got.view(np.uint16), want.view(np.uint16))


# --------------------------------------------------- the page's example ----
def test_itmedia_worked_example_53():
    g = load("itmedia_53.txt")
    q = oracle.quantize_with_scale(np.array([g["x"]], np.float32), float(g["scale"]))
    assert q[0] == g["q"]
    assert q[0] * g["scale"] == g["dequant"]
    assert g["x"] - q[0] * g["scale"] == g["error"]
    # the same numbers through the absmax rule of a token row
    xq, sx = oracle.ln_quant_act(f16([g["row"]]))
    assert sx[0] == np.float32(g["scale"])
    assert list(xq[0]) == list(g["row_q"])


# ---------------------------------------------------------- hand examples ----
def test_hand_example_quant_gemm_dequant():
    g = load("quant_gemm_3x2.txt")
    xq, sx = oracle.ln_quant_act(f16(g["A"]))
    assert np.array_equal(sx, g["sx"].astype(np.float32))
    assert np.array_equal(xq, g["qx"].astype(np.int8))
    wq, sw = oracle.quantize_weight(f16(g["Wt"]))
    assert np.array_equal(sw, g["sw"].astype(np.float32))
    assert np.array_equal(wq, g["qw"].astype(np.int8))
    acc = oracle.int_gemm(xq, wq)
    assert np.array_equal(acc, g["acc"].astype(np.int32))
    y = oracle.dequant(acc, sx, sw)
    assert np.array_equal(y.astype(np.float64), g["y"])
    y2 = oracle.w8a8_linear(xq, sx, wq, sw)
    assert np.array_equal(y2.view(np.uint16), y.view(np.uint16))
    assert np.allclose(oracle.linear_fp64(g["A"], g["Wt"]), g["Y64"], rtol=0, atol=1e-9)


def test_hand_example_smoothing():
    g = load("smoothing_4x4.txt")
    X, W = g["X"], g["W"]
    ax = oracle.calibrate_absmax(f16(X))
    aw = oracle.calibrate_absmax(f16(W))
    assert np.array_equal(ax, g["amax_x"].astype(np.float32))
    assert np.array_equal(aw, g["amax_w"].astype(np.float32))

    s, inv_s = oracle.smooth(ax, aw, 0.5)
    assert np.array_equal(s, g["s_half"].astype(np.float32))
    xhat = oracle.act_rows(f16(X), inv_s=inv_s)
    assert np.array_equal(xhat, g["Xhat_half"].astype(np.float32))
    what = oracle.fold_weight(f16(W), s)
    assert np.array_equal(what.astype(np.float64), g["What_half"])
    assert np.array_equal(np.abs(xhat).max(0), g["colmax_Xhat_half"].astype(np.float32))
    assert np.array_equal(np.abs(what.astype(np.float32)).max(0), g["colmax_What_half"].astype(np.float32))
    # the product is unchanged by the transform
    assert np.array_equal(oracle.linear_fp64(xhat, what), g["Y"])
    assert np.array_equal(oracle.linear_fp64(X, W), g["Y"])

    s1, inv1 = oracle.smooth(ax, aw, 1.0)
    assert np.array_equal(s1, g["s_one"].astype(np.float32))
    assert np.array_equal(np.abs(oracle.act_rows(f16(X), inv_s=inv1)).max(0),
                          g["colmax_Xhat_one"].astype(np.float32))
    s0, _ = oracle.smooth(ax, aw, 0.0)
    assert np.array_equal(s0, g["s_zero"].astype(np.float32))


# ------------------------------------------------------------ invariants ----
def _outlier_data(seed, T=64, K=96, N=40, gain=80.0):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((T, K))
    ch = rng.choice(K, 4, replace=False)
    X[:, ch] *= gain
    W = rng.standard_normal((N, K)) * 0.02
    return X, W


@pytest.mark.parametrize("alpha", [0.0, 0.25, 0.5, 0.75, 0.85, 1.0])
def test_equivalence_fp64(alpha):
    X, W = _outlier_data(2)
    a = np.abs(X).max(0)
    b = np.abs(W).max(0)
    s = oracle.smooth_fp64(a, b, alpha)
    Y = oracle.linear_fp64(X, W)
    Ys = oracle.smoothed_linear_fp64(X, W, s)
    assert np.linalg.norm(Ys - Y) / np.linalg.norm(Y) <= 1e-12


@pytest.mark.parametrize("alpha", [0.0, 0.25, 0.5, 0.75, 0.85, 1.0])
def test_alpha_closed_forms(alpha):
    rng = np.random.default_rng(3)
    K = 4096
    a = np.exp(rng.uniform(np.log(1e-3), np.log(300.0), K)).astype(np.float32)
    b = np.exp(rng.uniform(np.log(1e-3), np.log(3.0), K)).astype(np.float32)
    a64, b64 = a.astype(np.float64), b.astype(np.float64)
    s, inv_s = oracle.smooth(a, b, alpha)
    alpha = float(np.float32(alpha))  # the exponent is passed as an fp32 number
    # fp32 s is the rounding of a^alpha / b^(1-alpha): within one fp32 ulp of the fp64 value
    s64 = a64 ** alpha / b64 ** (1.0 - alpha)
    assert np.all(np.abs(s.astype(np.float64) - s64) <= ulp32(s))
    assert np.array_equal(inv_s, (np.float32(1) / s).astype(np.float32))
    # closed forms of the smoothed maxima: max|Xhat_j| = (a b)^(1-alpha), max|What_j| = (a b)^alpha
    xmax = a64 / s.astype(np.float64)
    wmax = b64 * s.astype(np.float64)
    assert np.allclose(xmax, (a64 * b64) ** (1 - alpha), rtol=2e-7, atol=0)
    assert np.allclose(wmax, (a64 * b64) ** alpha, rtol=2e-7, atol=0)
    assert np.allclose(xmax * wmax, a64 * b64, rtol=3e-7, atol=0)
    if alpha == 1.0:  # activation channel maxima equalised to 1
        assert np.allclose(a64 * inv_s.astype(np.float64), 1.0, rtol=2.5e-7)
    if alpha == 0.0:  # weight-only scaling: s = 1/b, weight channel maxima become 1
        assert np.allclose(wmax, 1.0, rtol=2e-7)
    if alpha == 0.5:
        assert np.allclose(s64, np.sqrt(a64) / np.sqrt(b64), rtol=1e-15)
        assert np.allclose(xmax, wmax, rtol=3e-7)


def test_smooth_floors_dead_channels():
    a = np.array([0.0, 0.0, 2.0], np.float32)
    b = np.array([0.0, 4.0, 0.0], np.float32)
    s, inv_s = oracle.smooth(a, b, 0.5)
    want = np.array([1.0, np.sqrt(1e-5) / 2.0, np.sqrt(2.0) / np.sqrt(1e-5)])
    # the floor is the fp32 number nearest 1e-5
    want = oracle.smooth_fp64(a, b, 0.5, floor=float(np.float32(1e-5)))
    assert np.all(np.abs(s - want) <= ulp32(s))
    assert np.all(np.isfinite(inv_s))


# -------------------------------------------------- library special cases ----
def test_calibration_max_is_numpy_abs_max():
    rng = np.random.default_rng(4)
    x1 = f16(rng.standard_normal((37, 200)) * 5)
    x2 = f16(rng.standard_normal((11, 200)) * 9)
    a = oracle.calibrate_absmax(x1)
    assert np.array_equal(a, np.abs(x1.astype(np.float32)).max(0))
    a = oracle.calibrate_absmax(x2, amax=a)  # running max across batches
    both = np.concatenate([x1, x2]).astype(np.float32)
    assert np.array_equal(a, np.abs(both).max(0))


@pytest.mark.parametrize("M,N,K", [(1, 1, 16), (7, 5, 48), (33, 17, 256), (16, 33, 144)])
def test_int_gemm_brute_force(M, N, K):
    rng = np.random.default_rng(M * 1000 + N * 10 + K)
    xq = rng.integers(-127, 128, (M, K)).astype(np.int8)
    wq = rng.integers(-127, 128, (N, K)).astype(np.int8)
    want = xq.astype(np.int64) @ wq.astype(np.int64).T
    assert np.array_equal(oracle.int_gemm(xq, wq).astype(np.int64), want)
    assert np.array_equal(oracle.int_gemm64(xq, wq), want)


def test_int32_accumulator_bound_at_max_k():
    K = 133144
    assert K * 127 * 127 <= 2 ** 31 - 1 < (K + 1) * 127 * 127 + 127 * 127
    xq = np.full((2, K), 127, np.int8)
    xq[1] = -127
    wq = np.full((1, K), 127, np.int8)
    acc = oracle.int_gemm(xq, wq)
    assert acc[0, 0] == K * 16129 == 2147479576
    assert acc[1, 0] == -K * 16129
    assert np.array_equal(acc.astype(np.int64), oracle.int_gemm64(xq, wq))


def test_unit_smoothing_reduces_to_plain_w8a8():
    rng = np.random.default_rng(5)
    h = f16(rng.standard_normal((9, 64)) * 3)
    a = oracle.ln_quant_act(h)
    b = oracle.ln_quant_act(h, inv_s=np.ones(64, np.float32))
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_per_tensor_weight_scale_is_equal_channel_scales():
    # O1 of the explainer ("inference"): one weight scale for the whole tensor.
    rng = np.random.default_rng(6)
    w = rng.standard_normal((8, 32))
    w[np.arange(8), rng.integers(0, 32, 8)] = 4.0  # every row has the same absmax
    wq, sw = oracle.quantize_weight(f16(w))
    assert np.all(sw == sw[0])


# ------------------------------------------------------ quantize properties --
def test_per_token_quantization_properties():
    rng = np.random.default_rng(7)
    h = rng.standard_normal((50, 128)) * rng.uniform(0.01, 100, (50, 1))
    h[3] = 0.0
    h16 = f16(h)
    xq, sx = oracle.ln_quant_act(h16)
    x = h16.astype(np.float32)
    amax = np.abs(x).max(1)
    assert np.array_equal(sx, (amax / np.float32(127)).astype(np.float32))
    assert sx[3] == 0 and not xq[3].any()
    nz = amax > 0
    assert np.all(np.abs(xq[nz]).max(1) == 127)
    err = np.abs(xq.astype(np.float64) * sx[:, None].astype(np.float64) - x.astype(np.float64))
    assert np.all(err <= 0.5 * sx[:, None] * (1 + 1e-5) + 1e-30)
    # numpy round-half-to-even on the same fp32 products gives the same codes
    inv = np.where(sx > 0, np.float32(1) / np.where(sx > 0, sx, 1), 0).astype(np.float32)
    p = (x * inv[:, None]).astype(np.float32)
    assert np.array_equal(xq, np.clip(np.rint(p), -127, 127).astype(np.int8))


def test_dequant_zero_row_gives_bias():
    xq = np.zeros((2, 32), np.int8)
    xq[1, 0] = 5
    sx = np.array([0.0, 0.5], np.float32)
    wq = np.ones((3, 32), np.int8)
    sw = np.array([1.0, 2.0, 4.0], np.float32)
    bias = f16([0.25, -1.5, 3.0])
    y = oracle.w8a8_linear(xq, sx, wq, sw, bias)
    assert np.array_equal(y[0], bias)
    assert np.array_equal(y[1].astype(np.float64), [2.75, 3.5, 13.0])


def test_dequant_matches_fp64_within_one_fp16_rounding():
    rng = np.random.default_rng(8)
    acc = rng.integers(-2 ** 24, 2 ** 24, (20, 30)).astype(np.int32)
    sx = rng.uniform(1e-4, 1e-2, 20).astype(np.float32)
    sw = rng.uniform(1e-4, 1e-2, 30).astype(np.float32)
    bias = f16(rng.standard_normal(30))
    y = oracle.dequant(acc, sx, sw, bias).astype(np.float64)
    exact = acc * sx[:, None].astype(np.float64) * sw[None, :].astype(np.float64) + bias.astype(np.float64)
    # three fp32 roundings then one fp16 rounding
    tol = np.spacing(np.abs(exact).astype(np.float16)).astype(np.float64) * 0.5 + np.abs(exact) * 4e-7
    assert np.all(np.abs(y - exact) <= tol)


# -------------------------------------------------------------- LayerNorm ----
def test_ln_stats_exact_sums_match_fp64():
    rng = np.random.default_rng(9)
    rows = [rng.standard_normal(4096), rng.standard_normal(4096) * 0.01 + 50.0,
            rng.standard_normal(1000) * 300, np.concatenate([rng.standard_normal(511), [4000.0]])]
    for r in rows:
        h = f16(r)[None, :]
        mu, rstd = oracle.ln_stats(h)
        v = h.astype(np.float64)[0]
        m64 = v.mean()
        r64 = 1.0 / np.sqrt(((v - m64) ** 2).mean() + float(np.float32(1e-5)))
        assert abs(mu[0] - m64) <= ulp32(mu[0]) + abs(m64) * 1e-12
        assert abs(rstd[0] - r64) <= ulp32(rstd[0]) * 1.0 + r64 * 1e-9


def test_ln_stats_closed_form_row():
    h = f16(np.tile([1.0, -1.0], 64))[None, :]
    mu, rstd = oracle.ln_stats(h)
    assert mu[0] == 0.0
    assert rstd[0] == np.float32(1.0 / np.sqrt(1.0 + float(np.float32(1e-5))))
    h = f16(np.full(100, 3.25))[None, :]  # constant row: var 0, output = beta
    mu, rstd = oracle.ln_stats(h)
    assert mu[0] == np.float32(3.25)
    assert rstd[0] == np.float32(1.0 / np.sqrt(float(np.float32(1e-5))))
    beta = np.linspace(-1, 1, 100).astype(np.float32)
    x = oracle.act_rows(h, gamma=np.full(100, 7.0, np.float32), beta=beta)
    assert np.array_equal(x[0], beta)


def test_ln_output_matches_fp64_layernorm():
    rng = np.random.default_rng(10)
    K = 512
    h = f16(rng.standard_normal((16, K)) * 2 + 0.5)
    g = np.ones(K, np.float32)
    g[[5, 99]] = 60.0
    b = (rng.standard_normal(K) * 0.01).astype(np.float32)
    x = oracle.act_rows(h, gamma=g, beta=b)
    hv = h.astype(np.float64)
    ref = oracle.layernorm_fp64(hv, g, b, eps=float(np.float32(1e-5)))
    # error budget of fp32 evaluation: mu and rstd each rounded once, then four
    # rounded ops; |h - mu| may cancel, so the bound scales with |mu| + |h - mu|
    mu = hv.mean(1, keepdims=True)
    rstd = 1 / np.sqrt(((hv - mu) ** 2).mean(1, keepdims=True) + 1e-5)
    budget = np.abs(g) * rstd * (np.abs(mu) + np.abs(hv - mu)) + np.abs(b) + np.abs(ref)
    assert np.all(np.abs(x - ref) <= 4 * 2.0 ** -24 * budget)


def test_ln_quant_equals_quantized_ln_rows():
    rng = np.random.default_rng(11)
    K = 256
    h = f16(rng.standard_normal((8, K)))
    g = rng.uniform(0.5, 2, K).astype(np.float32)
    b = rng.standard_normal(K).astype(np.float32) * np.float32(0.1)
    inv_s = rng.uniform(0.1, 3, K).astype(np.float32)
    xq, sx = oracle.ln_quant_act(h, gamma=g, beta=b, inv_s=inv_s)
    x = oracle.act_rows(h, gamma=g, beta=b, inv_s=inv_s)
    assert np.array_equal(sx, (np.abs(x).max(1) / np.float32(127)).astype(np.float32))
    for t in range(8):
        assert np.array_equal(xq[t], oracle.quantize_with_scale(x[t], float(sx[t])))


def test_fold_ln_is_gamma_times_inv_s():
    rng = np.random.default_rng(12)
    g = rng.standard_normal(64).astype(np.float32)
    b = rng.standard_normal(64).astype(np.float32)
    inv_s = rng.uniform(0.01, 10, 64).astype(np.float32)
    g2, b2 = oracle.fold_ln(g, b, inv_s)
    assert np.array_equal(g2, (g * inv_s).astype(np.float32))
    assert np.array_equal(b2, (b * inv_s).astype(np.float32))


def test_fold_weight_rounds_once_to_fp16():
    rng = np.random.default_rng(13)
    w = f16(rng.standard_normal((16, 48)) * 0.02)
    s = rng.uniform(0.05, 20, 48).astype(np.float32)
    got = oracle.fold_weight(w, s)
    want = (w.astype(np.float32) * s[None, :]).astype(np.float32).astype(np.float16)
    assert np.array_equal(got.view(np.uint16), want.view(np.uint16))


def test_symmetric_range_never_produces_minus_128():
    # The INT8 range is the symmetric [-127, 127]: values beyond the range clamp.
    x = np.array([-1000.0, 1000.0, -127.5, 127.5, -128.0, 126.5], np.float32)
    q = oracle.quantize_with_scale(x, 1.0)
    assert list(q) == [-127, 127, -127, 127, -127, 126]


def test_zero_scale_gives_zero_codes():
    # Reading where the pages are silent: a zero scale (all-zero range) has no
    # reciprocal; its codes are 0 and its dequantized values are exactly 0.
    q = oracle.quantize_with_scale(np.array([1.0, -2.0, 0.0], np.float32), 0.0)
    assert list(q) == [0, 0, 0]


# ------------------------------------------------- quantization levels O1-O3 --
def test_hand_example_levels():
    g = load("levels_2x4.txt")
    x = f16(g["X"])
    xq, sx = oracle.ln_quant_act(x)
    assert np.array_equal(sx, g["o1_sx"]) and np.array_equal(xq, g["o1_qx"])
    xq, sx, rng_ = oracle.ln_quant_act_tensor(x)
    assert rng_ == g["o2_range"]
    assert np.array_equal(sx, g["o2_sx"]) and np.array_equal(xq, g["o2_qx"])
    xq, sx = oracle.ln_quant_act_static(x, g["o3_range"])
    assert np.array_equal(sx, g["o3_sx"]) and np.array_equal(xq, g["o3_qx"])
    wq, sw, wr = oracle.quantize_weight_tensor(f16(g["W"]))
    assert wr == g["wt_range"]
    assert np.array_equal(sw, g["wt_sw"]) and np.array_equal(wq, g["wt_qw"])
    assert oracle.tensor_range(g["cal_amax"], g["cal_inv_s"]) == g["cal_range"]
    assert oracle.tensor_range(g["cal_amax"]) == 7.0


def _ln_batch(seed, M=12, K=96):
    rng = np.random.default_rng(seed)
    h = f16(rng.standard_normal((M, K)) * 2)
    gamma = (1 + rng.uniform(0, 3, K)).astype(np.float32)
    gamma[rng.integers(0, K, 3)] = 60.0
    beta = (rng.standard_normal(K) * 0.1).astype(np.float32)
    inv_s = rng.uniform(0.05, 2.0, K).astype(np.float32)
    return h, gamma, beta, inv_s


def _np_codes(x, range_):
    """Independent restatement: the same quantizer in numpy float32 arithmetic."""
    sc = np.float32(range_) / np.float32(127)
    inv = np.float32(1) / sc if sc > 0 else np.float32(0)
    p = (np.asarray(x, np.float32) * inv).astype(np.float32)
    return np.clip(np.rint(p), -127, 127).astype(np.int8), sc


@pytest.mark.parametrize("path", ["ln", "inv_s"])
def test_o2_is_one_range_over_the_batch(path):
    h, gamma, beta, inv_s = _ln_batch(21)
    kw = dict(gamma=gamma, beta=beta) if path == "ln" else dict(inv_s=inv_s)
    xq, sx, rng_ = oracle.ln_quant_act_tensor(h, **kw)
    x = oracle.act_rows(h, **kw)
    assert rng_ == np.abs(x).max()
    codes, sc = _np_codes(x, rng_)
    assert np.all(sx == sc) and np.array_equal(xq, codes)
    # a batch of one token: O2 is O1
    q1, s1 = oracle.ln_quant_act(h[4:5], **kw)
    q2, s2, _ = oracle.ln_quant_act_tensor(h[4:5], **kw)
    assert np.array_equal(q1, q2) and np.array_equal(s1, s2)


def test_o3_static_equals_o2_when_calibrated_on_the_batch():
    h, gamma, beta, _ = _ln_batch(22)
    amax = oracle.calibrate_absmax(h, gamma=gamma, beta=beta)
    r = oracle.tensor_range(amax)
    q3, s3 = oracle.ln_quant_act_static(h, r, gamma=gamma, beta=beta)
    q2, s2, r2 = oracle.ln_quant_act_tensor(h, gamma=gamma, beta=beta)
    assert r == r2 and np.array_equal(q3, q2) and np.array_equal(s3, s2)


def test_o3_saturates_outside_the_static_range():
    h, gamma, beta, inv_s = _ln_batch(23)
    x = oracle.act_rows(h, inv_s=inv_s)
    r = np.float32(np.abs(x).max() * 0.25)  # calibration saw a quarter of this batch's range
    q, s = oracle.ln_quant_act_static(h, r, inv_s=inv_s)
    codes, sc = _np_codes(x, r)
    assert np.all(s == sc) and np.array_equal(q, codes)
    big = np.abs(x) * (np.float32(1) / sc) > 127.5
    assert big.any() and np.array_equal(q[big], np.sign(x[big]).astype(np.int8) * 127)


def test_static_range_from_inv_s_is_the_smoothed_calibration_max():
    h, _, _, inv_s = _ln_batch(24)
    amax = oracle.calibrate_absmax(h)
    r = oracle.tensor_range(amax, inv_s)
    assert r == np.abs(oracle.act_rows(h, inv_s=inv_s)).max()


def test_per_tensor_weight_quantization():
    rng = np.random.default_rng(25)
    w = f16(rng.standard_normal((20, 64)) * rng.uniform(0.1, 5, (20, 1)))
    wq, sw, r = oracle.quantize_weight_tensor(w)
    assert r == np.abs(w.astype(np.float32)).max()
    codes, sc = _np_codes(w.astype(np.float32), r)
    assert np.all(sw == sc) and np.array_equal(wq, codes)
    # equal row ranges: per-tensor and per-channel agree
    w2 = rng.standard_normal((8, 32))
    w2[np.arange(8), rng.integers(0, 32, 8)] = 4.0
    a = oracle.quantize_weight(f16(w2))
    b = oracle.quantize_weight_tensor(f16(w2))
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


# ------------------------------------------- producer-side quantization ----
def test_hand_example_producer_quant():
    g = load("producer_quant_2x3.txt")
    args = (g["xq"].astype(np.int8), g["sx"], g["wq"].astype(np.int8), g["sw"], f16(g["bias"]))
    q, s = oracle.w8a8_linear_quant_static(*args, relu=True, inv_s_next=g["inv_s"], range_next=g["range"])
    assert np.array_equal(q, g["q_relu"]) and np.array_equal(s, g["sx_next"])
    q, s = oracle.w8a8_linear_quant_static(*args, relu=False, inv_s_next=g["inv_s"], range_next=g["range"])
    assert np.array_equal(q, g["q_plain"])


@pytest.mark.parametrize("relu", [False, True])
def test_producer_quant_is_linear_then_static_quant(relu):
    """Independent restatement in numpy float32 of everything after the
    (separately pinned) fp16 linear output."""
    rng = np.random.default_rng(31 + relu)
    M, N, K = 9, 40, 64
    xq = rng.integers(-127, 128, (M, K)).astype(np.int8)
    wq = rng.integers(-127, 128, (N, K)).astype(np.int8)
    sx = rng.uniform(1e-3, 1e-2, M).astype(np.float32)
    sw = rng.uniform(1e-3, 1e-2, N).astype(np.float32)
    bias = f16(rng.standard_normal(N) * 0.1)
    inv = rng.uniform(0.1, 3.0, N).astype(np.float32)
    y = oracle.w8a8_linear(xq, sx, wq, sw, bias).astype(np.float32)
    a = np.where(y > 0, y, np.float32(0)) if relu else y
    x = (a * inv[None, :]).astype(np.float32)
    r = np.float32(np.abs(x).max() * 0.7)  # some values saturate
    codes, sc = _np_codes(x, r)
    q, s = oracle.w8a8_linear_quant_static(xq, sx, wq, sw, bias, relu=relu, inv_s_next=inv, range_next=r)
    assert np.all(s == sc) and np.array_equal(q, codes)
    assert (np.abs(q) == 127).any()


def test_hand_example_producer_dynamic():
    g = load("producer_dyn_3x3.txt")
    args = (g["xq"].astype(np.int8), g["sx"], g["wq"].astype(np.int8), g["sw"], f16(g["bias"]))
    q, s = oracle.w8a8_linear_quant_dynamic(*args, relu=True, inv_s_next=g["inv_s"])
    assert np.array_equal(q, g["q_relu"]) and np.array_equal(s, g["sx_relu"].astype(np.float32))
    q, s = oracle.w8a8_linear_quant_dynamic(*args, relu=False, inv_s_next=g["inv_s"])
    assert np.array_equal(q, g["q_plain"])
    assert np.array_equal(s[:2], g["sx_plain_rows01"].astype(np.float32))
    assert s[2] == np.float32(0.375) / np.float32(127)


@pytest.mark.parametrize("relu", [False, True])
def test_producer_dynamic_is_linear_then_per_token_quant(relu):
    """Independent restatement in numpy float32 of everything after the (separately pinned)
    fp16 linear output: ReLU, times 1/s, per-token absmax scale, round half to even."""
    rng = np.random.default_rng(77 + relu)
    M, N, K = 11, 48, 64
    xq = rng.integers(-127, 128, (M, K)).astype(np.int8)
    wq = rng.integers(-127, 128, (N, K)).astype(np.int8)
    sx = rng.uniform(1e-3, 1e-2, M).astype(np.float32)
    sx[3] = 0.0  # a zero row: y = bias
    sw = rng.uniform(1e-3, 1e-2, N).astype(np.float32)
    bias = f16(rng.standard_normal(N) * 0.1)
    inv = rng.uniform(0.1, 3.0, N).astype(np.float32)
    y = oracle.w8a8_linear(xq, sx, wq, sw, bias).astype(np.float32)
    a = np.where(y > 0, y, np.float32(0)) if relu else y
    x = (a * inv[None, :]).astype(np.float32)
    sc = (np.abs(x).max(axis=1) / np.float32(127)).astype(np.float32)
    rcp = np.where(sc > 0, np.float32(1) / np.where(sc > 0, sc, 1), 0).astype(np.float32)
    codes = np.clip(np.rint((x * rcp[:, None]).astype(np.float32)), -127, 127).astype(np.int8)
    q, s = oracle.w8a8_linear_quant_dynamic(xq, sx, wq, sw, bias, relu=relu, inv_s_next=inv)
    assert np.array_equal(s, sc) and np.array_equal(q, codes)
    # the row maxima hit 127 exactly: the dynamic scale is each row's own range
    assert np.all(np.abs(q).max(axis=1)[sc > 0] == 127)


def test_producer_dynamic_equals_static_when_rows_share_a_range():
    """When every row's range equals one static range, the per-token and the static
    (level O3) producer quantizations coincide."""
    rng = np.random.default_rng(5)
    M, N, K = 6, 32, 32
    xq = rng.integers(-20, 21, (M, K)).astype(np.int8)
    wq = rng.integers(-20, 21, (N, K)).astype(np.int8)
    xq[:, 0] = 100  # channel 0 of every output gets one large, equal value per row
    wq[:, 0] = 0
    wq[0, :] = 0
    wq[0, 0] = 127
    sx = np.full(M, 0.01, np.float32)
    sw = np.full(N, 0.01, np.float32)
    inv = np.ones(N, np.float32)
    y = oracle.w8a8_linear(xq, sx, wq, sw).astype(np.float32)
    r = np.abs(y).max(axis=1)
    assert np.all(r == r[0])  # the same range in every row (output 0 dominates)
    qd, sd = oracle.w8a8_linear_quant_dynamic(xq, sx, wq, sw, inv_s_next=inv)
    qs, ss = oracle.w8a8_linear_quant_static(xq, sx, wq, sw, inv_s_next=inv, range_next=r[0])
    assert np.array_equal(qd, qs) and np.array_equal(sd, ss)


# ------------------------------------------------------------------ INT8 BMM --
def test_hand_example_bmm():
    g = load("bmm_2x2x2.txt")
    a = np.stack([g["a0"], g["a1"]]).astype(np.int8)
    b = np.stack([g["b0"], g["b1"]]).astype(np.int8)
    y = oracle.w8a8_bmm(a, np.stack([g["as0"], g["as1"]]), b, np.stack([g["bs0"], g["bs1"]]))
    assert np.array_equal(y.astype(np.float64), np.stack([g["y0"], g["y1"]]))


def test_bmm_items_are_independent_linears():
    rng = np.random.default_rng(41)
    B, M, N, K = 3, 7, 9, 48
    a = rng.integers(-127, 128, (B, M, K)).astype(np.int8)
    b = rng.integers(-127, 128, (B, N, K)).astype(np.int8)
    sa = rng.uniform(1e-3, 1e-2, (B, M)).astype(np.float32)
    sb = rng.uniform(1e-3, 1e-2, (B, N)).astype(np.float32)
    y = oracle.w8a8_bmm(a, sa, b, sb)
    for i in range(B):
        acc = a[i].astype(np.int64) @ b[i].astype(np.int64).T  # numpy brute force
        exact = acc * sa[i][:, None].astype(np.float64) * sb[i][None, :].astype(np.float64)
        assert np.all(np.abs(y[i].astype(np.float64) - exact) <= np.spacing(np.abs(exact).astype(np.float16)))
        assert np.array_equal(y[i], oracle.w8a8_linear(a[i], sa[i], b[i], sb[i]))


# ------------------------------------------------------- non-finite inputs ----
# IEEE arithmetic fixes these: a mean or variance over a row that holds an Inf
# or a NaN is NaN, a NaN never wins a maximum taken with ">", and a NaN
# product has no nearest integer level (the quantizer gives 0 for it).
@pytest.mark.parametrize("bad", [np.inf, -np.inf, np.nan])
def test_ln_stats_of_a_non_finite_row_are_nan(bad):
    h = f16(np.linspace(-2, 2, 64)).reshape(2, 32)
    h[1, 7] = bad
    mu, rstd = oracle.ln_stats(h)
    assert np.isfinite(mu[0]) and np.isfinite(rstd[0])
    assert np.isnan(mu[1]) and np.isnan(rstd[1])
    g = np.ones(32, np.float32)
    x = oracle.act_rows(h, g, g)
    assert np.isfinite(x[0]).all() and np.isnan(x[1]).all()


@pytest.mark.parametrize("bad", [np.inf, np.nan])
def test_ln_quantization_of_a_non_finite_row(bad):
    rng = np.random.default_rng(3)
    h = f16(rng.standard_normal((3, 48)))
    h[1, 5] = bad
    g = (rng.random(48) + 0.5).astype(np.float32)
    b = rng.standard_normal(48).astype(np.float32)
    xq, sx = oracle.ln_quant_act(h, g, b)
    # the NaN row: no level wins the maximum, scale 0, every code 0
    assert sx[1] == 0.0 and not xq[1].any()
    # the finite rows are what they are alone
    for r in (0, 2):
        q1, s1 = oracle.ln_quant_act(h[r:r + 1], g, b)
        assert np.array_equal(xq[r], q1[0]) and sx[r] == s1[0]
    # calibration: the NaN row adds nothing to the running maxima
    a_all = oracle.calibrate_absmax(h, gamma=g, beta=b)
    a_fin = oracle.calibrate_absmax(h[[0, 2]], gamma=g, beta=b)
    assert np.array_equal(a_all, a_fin)


def test_nan_values_quantize_to_zero_and_inf_saturates():
    rng = np.random.default_rng(4)
    h = f16(rng.standard_normal((2, 40)))
    h[0, 3] = np.nan
    h[1, 9] = np.inf
    xq, sx = oracle.ln_quant_act(h)  # no LayerNorm: x_hat = h
    # row 0: the NaN is ignored by the maximum and gets code 0
    assert sx[0] == np.float32(np.abs(np.delete(h[0], 3).astype(np.float32)).max() / np.float32(127))
    assert xq[0, 3] == 0 and np.abs(xq[0]).max() == 127
    # row 1: an infinite range makes the scale Inf and 1/scale 0, so every
    # product is 0 (finite values) or NaN (Inf * 0): all codes 0
    assert np.isinf(sx[1]) and not xq[1].any()
    wq, sw = oracle.quantize_weight(h)
    assert np.array_equal(wq, xq) and np.array_equal(sw, sx)


# ------------------------------------------------- quality references ----
def test_hand_example_quality_references():
    # naive per-tensor W8A8 and per-token / per-channel W8A8 without smoothing, against the
    # hand-worked fixture (power-of-two scales, so the fp64 results are exact)
    g = load("quality_refs_2x3.txt")
    X, W, bias = g["X"], g["W"], g["bias"]
    assert np.array_equal(oracle.naive_per_tensor_w8a8(X, W), g["naive_y"])
    assert np.array_equal(oracle.per_token_per_channel_w8a8(X, W), g["ptpc_y"])
    assert np.array_equal(oracle.naive_per_tensor_w8a8(X, W, bias), g["naive_y"] + bias[None, :])
    assert np.array_equal(oracle.per_token_per_channel_w8a8(X, W, bias), g["ptpc_y"] + bias[None, :])
    # the fixture's own steps hang together: codes -> exact integer sums -> scaled sums
    assert np.array_equal(g["naive_qx"] @ g["naive_qw"].T, g["naive_acc"])
    assert np.array_equal(g["naive_acc"] * (2.0 * 2.0), g["naive_y"])
    assert np.array_equal(g["ptpc_qx"] @ g["ptpc_qw"].T, g["ptpc_acc"])
    sx, sw = np.array([2.0, 0.5, 0.0]), np.array([1.0, 2.0])
    assert np.array_equal(g["ptpc_acc"] * sx[:, None] * sw[None, :], g["ptpc_y"])
    assert np.array_equal(X @ W.T, g["Y"])


def test_quality_references_agree_when_every_row_has_one_range():
    # with the same absmax on every token row and every weight row, one scale per row is one
    # scale per tensor: the two references take the same codes, so they agree up to the fp64
    # rounding of their scale products (acc * (sx * sw) against (acc * sx) * sw)
    rng = np.random.default_rng(5)
    X = rng.uniform(-2.9, 2.9, (6, 16))
    W = rng.uniform(-0.49, 0.49, (5, 16))
    X[np.arange(6), rng.integers(0, 16, 6)] = 3.0 * rng.choice([-1.0, 1.0], 6)
    W[np.arange(5), rng.integers(0, 16, 5)] = 0.5 * rng.choice([-1.0, 1.0], 5)
    b = rng.standard_normal(5)
    assert np.allclose(oracle.naive_per_tensor_w8a8(X, W, b), oracle.per_token_per_channel_w8a8(X, W, b),
                       rtol=1e-14, atol=1e-14)
    # and both are the plain product within half a quantization step per operand
    err = np.abs(oracle.naive_per_tensor_w8a8(X, W) - X @ W.T)
    bound = 16 * (0.5 * 3.0 / 127 * 0.5 + 0.5 * 0.5 / 127 * 3.0 + 0.25 * (3.0 / 127) * (0.5 / 127))
    assert (err <= bound).all()
