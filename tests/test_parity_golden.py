"""The hand-worked fixtures under tests/golden/ pushed through the CUDA path
(the C ABI, through the binding), bit for bit, and tie-rich synthetic tensors
that reach every kernel shape's rounding.

The fixtures fix round-half-to-even (itmedia quantization tutorial, section
3, "round to the nearest level", read as ties-to-even), all-zero rows, the
alpha limits of the smoothing factor (SmoothQuant explainer, "how is the
smoothing factor chosen"), the efficiency levels O1-O3 ("inference"),
producer-side quantization ("what it does mathematically") and the INT8 BMM.
Their expected values are the fixtures' own, derived by hand; nothing here
depends on the oracle.

K must be a multiple of 16 at the boundary, so a fixture with a shorter K is
padded with zero columns: a zero changes no range, no code and no sum.  The
tie tensors are built so that every scale is a power of two; then
x * (1/scale) is exact in fp32 and lands on k + 0.5 for many elements, and
the expected code is numpy's rint (ties to even) of the exact quotient.
"""
import numpy as np
import pytest
import torch

from golden_io import load
from gpu_util import bits_equal, dev, host

pytestmark = pytest.mark.gpu

KP = 16


@pytest.fixture(scope="module")
def sq(cuda_device):
    import w8a8_int8_linear_channel_b200 as m
    return m


def padk(a, K=KP):
    a = np.atleast_2d(np.asarray(a))
    out = np.zeros(a.shape[:-1] + (K,), a.dtype)
    out[..., : a.shape[-1]] = a
    return out


def padv(v, K=KP, fill=0.0):
    v = np.asarray(v, np.float32).ravel()
    out = np.full(K, fill, np.float32)
    out[: v.size] = v
    return out


def i8(a):
    return np.asarray(a).astype(np.int8)


def f32(a):
    return np.asarray(a, np.float32).ravel()


PATHS = ("tiled", "splitk", "pair", "auto")


def path_id(sq, name):
    return {"tiled": sq.PATH_TILED, "splitk": sq.PATH_SPLITK, "pair": sq.PATH_PAIR,
            "auto": sq.PATH_AUTO}[name]


def act_quant(sq, h, gamma=None, beta=None, inv_s=None):
    M, K = h.shape
    xq = torch.empty((M, K), dtype=torch.int8, device="cuda")
    sx = torch.empty(M, dtype=torch.float32, device="cuda")
    sq.sq_ln_quant_act(dev(h), xq, sx, dev(gamma), dev(beta), dev(inv_s))
    return host(xq), host(sx)


def weight_quant(sq, w, s=None):
    N, K = w.shape
    wq = torch.empty((N, K), dtype=torch.int8, device="cuda")
    sw = torch.empty(N, dtype=torch.float32, device="cuda")
    sq.sq_quantize_weight(dev(w), wq, sw, s=dev(s))
    return host(wq), host(sw)


# ------------------------------------------- quantize -> GEMM -> dequant ----
G = load("quant_gemm_3x2.txt")


def test_fixture_activation_codes(sq):
    xq, sx = act_quant(sq, padk(G["A"].astype(np.float16)))
    assert bits_equal(sx, f32(G["sx"]))
    assert np.array_equal(xq, padk(i8(G["qx"])))


@pytest.mark.parametrize("fold", [False, True])
def test_fixture_weight_codes(sq, fold):
    # the fold with s = 1 goes through the fold-on-the-fly branch and changes nothing
    s = np.ones(KP, np.float32) if fold else None
    wq, sw = weight_quant(sq, padk(G["Wt"].astype(np.float16)), s)
    assert bits_equal(sw, f32(G["sw"]))
    assert np.array_equal(wq, padk(i8(G["qw"])))


@pytest.mark.parametrize("path", PATHS)
def test_fixture_gemm_and_epilogue(sq, path):
    qx, qw = padk(i8(G["qx"])), padk(i8(G["qw"]))
    M, N = qx.shape[0], qw.shape[0]
    p = path_id(sq, path)
    ws = sq.new_workspace(M, N, KP)
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    sq.sq_w8a8_gemm_s32(dev(qx), dev(qw), acc, workspace=ws, path=p)
    assert np.array_equal(host(acc), G["acc"].astype(np.int32))
    y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    sq.sq_w8a8_linear(dev(qx), dev(f32(G["sx"])), dev(qw), dev(f32(G["sw"])), y, workspace=ws, path=p)
    assert bits_equal(host(y), G["y"].astype(np.float16))
    assert sq.sq_poll_status() == 0


def test_fixture_whole_chain(sq):
    """Activations and weight quantized on the GPU, then the linear: the fixture's y."""
    xq, sx = act_quant(sq, padk(G["A"].astype(np.float16)))
    wq, sw = weight_quant(sq, padk(G["Wt"].astype(np.float16)))
    y = torch.empty((3, 2), dtype=torch.float16, device="cuda")
    sq.sq_w8a8_linear(dev(xq), dev(sx), dev(wq), dev(sw), y, workspace=sq.new_workspace(3, 2, KP))
    assert bits_equal(host(y), G["y"].astype(np.float16))


# the same rows placed anywhere in a long row: every row-kernel shape (a warp per row with 1,
# 2 or 4 chunks; CTA rows of 64-256 threads with 4-24 chunks in registers; rows re-read from
# global memory) meets the fixture's ties, in its first, middle and last chunks
ROW_KS = [16, 256, 512, 1024, 2048, 4096, 4112, 8192, 12288, 16384, 24576, 49152, 65536]


@pytest.mark.parametrize("K", ROW_KS)
def test_fixture_rows_every_row_shape(sq, K):
    rng = np.random.default_rng(K)
    pos = np.sort(rng.choice(np.arange(1, K - 1), 2, replace=False)) if K > 16 else np.array([1, 2])
    cols = np.array([0, pos[0], pos[1], K - 1])
    A = np.zeros((3, K), np.float16)
    A[:, cols] = G["A"].astype(np.float16)
    W = np.zeros((2, K), np.float16)
    W[:, cols] = G["Wt"].astype(np.float16)
    qx_want = np.zeros((3, K), np.int8)
    qx_want[:, cols] = i8(G["qx"])
    qw_want = np.zeros((2, K), np.int8)
    qw_want[:, cols] = i8(G["qw"])
    xq, sx = act_quant(sq, A)
    assert bits_equal(sx, f32(G["sx"])) and np.array_equal(xq, qx_want)
    wq, sw = weight_quant(sq, W)
    assert bits_equal(sw, f32(G["sw"])) and np.array_equal(wq, qw_want)
    y = torch.empty((3, 2), dtype=torch.float16, device="cuda")
    sq.sq_w8a8_linear(dev(xq), dev(sx), dev(wq), dev(sw), y, workspace=sq.new_workspace(3, 2, K))
    assert bits_equal(host(y), G["y"].astype(np.float16))


# ------------------------------------------------------------- smoothing ----
S = load("smoothing_4x4.txt")


@pytest.mark.parametrize("alpha,key", [(0.5, "s_half"), (1.0, "s_one"), (0.0, "s_zero")])
def test_fixture_smoothing(sq, alpha, key):
    X = padk(S["X"].astype(np.float16))
    W = padk(S["W"].astype(np.float16))
    ax = torch.zeros(KP, dtype=torch.float32, device="cuda")
    aw = torch.zeros(KP, dtype=torch.float32, device="cuda")
    sq.sq_calibrate_absmax(dev(X), ax)
    sq.sq_calibrate_absmax(dev(W), aw)
    assert bits_equal(host(ax), padv(S["amax_x"]))
    assert bits_equal(host(aw), padv(S["amax_w"]))
    s, inv_s = torch.empty(KP, device="cuda"), torch.empty(KP, device="cuda")
    w_out = torch.empty((4, KP), dtype=torch.float16, device="cuda")
    sq.sq_smooth_fold(ax, aw, alpha, s, inv_s, w=dev(W), w_out=w_out)
    s_h = host(s)
    assert bits_equal(s_h[:4], f32(S[key]))
    # the padded channels are dead on both sides: both floors, s = 1e-5^alpha / 1e-5^(1-alpha)
    assert np.all(np.isfinite(s_h[4:])) and np.all(s_h[4:] > 0)
    inv_h = host(inv_s)
    assert bits_equal(inv_h[:4], (np.float32(1) / f32(S[key])).astype(np.float32))
    if key == "s_half":
        assert bits_equal(host(w_out)[:, :4], S["What_half"].astype(np.float16))
        # the smoothed activations X diag(s)^-1, quantized per token on the GPU, give the codes
        # of the fixture's X-hat (its per-token scale is max|X-hat row| / 127)
        xq, sx = act_quant(sq, X, inv_s=inv_h)
        xhat = S["Xhat_half"]
        want_sx = np.abs(xhat).max(1).astype(np.float32) / np.float32(127)
        assert bits_equal(sx, want_sx)
        q = np.rint(xhat.astype(np.float32) * (np.float32(1) / want_sx)[:, None])
        assert np.array_equal(xq[:, :4], q.astype(np.int8))
    # column maxima of X diag(s)^-1: max over channels = the static range of the smoothed input
    rng_out = torch.zeros(4, dtype=torch.float32, device="cuda")
    sq.sq_tensor_range(ax[:4].contiguous(), rng_out[:1], inv_s=inv_s[:4].contiguous())
    col = {"s_half": S["colmax_Xhat_half"], "s_one": S["colmax_Xhat_one"], "s_zero": S["amax_x"]}[key]
    assert host(rng_out)[0] == np.float32(np.max(col))
    if key == "s_one":  # alpha = 1: every activation channel maximum becomes exactly 1
        assert np.array_equal(host(ax)[:4] * inv_h[:4], np.ones(4, np.float32))
    if key == "s_zero":  # alpha = 0: weight-only scaling, W' = W here (its maxima are 1)
        assert bits_equal(host(w_out)[:, :4], S["W"].astype(np.float16))


# --------------------------------------------------------------- levels ----
L = load("levels_2x4.txt")


def test_fixture_levels_activations(sq):
    X = padk(L["X"].astype(np.float16))
    # O1: per token
    xq, sx = act_quant(sq, X)
    assert bits_equal(sx, f32(L["o1_sx"])) and np.array_equal(xq, padk(i8(L["o1_qx"])))
    # O2: one dynamic range for the batch
    q = torch.empty((2, KP), dtype=torch.int8, device="cuda")
    s = torch.empty(2, dtype=torch.float32, device="cuda")
    rng_out = torch.zeros(4, dtype=torch.float32, device="cuda")
    sq.sq_ln_quant_act_tensor(dev(X), q, s, rng_out[:1])
    assert host(rng_out)[0] == np.float32(L["o2_range"])
    assert bits_equal(host(s), f32(L["o2_sx"])) and np.array_equal(host(q), padk(i8(L["o2_qx"])))
    # O3: a static range, values beyond it saturate
    rin = dev(np.array([L["o3_range"], 0, 0, 0], np.float32))
    sq.sq_ln_quant_act_static(dev(X), q, s, rin[:1])
    assert bits_equal(host(s), f32(L["o3_sx"])) and np.array_equal(host(q), padk(i8(L["o3_qx"])))


def test_fixture_levels_weight_and_range(sq):
    W = padk(L["W"].astype(np.float16))
    wq = torch.empty((2, KP), dtype=torch.int8, device="cuda")
    sw = torch.empty(2, dtype=torch.float32, device="cuda")
    rng_out = torch.zeros(4, dtype=torch.float32, device="cuda")
    sq.sq_quantize_weight_tensor(dev(W), wq, sw, rng_out[:1])
    assert host(rng_out)[0] == np.float32(L["wt_range"])
    assert bits_equal(host(sw), f32(L["wt_sw"])) and np.array_equal(host(wq), padk(i8(L["wt_qw"])))
    r2 = torch.zeros(4, dtype=torch.float32, device="cuda")
    sq.sq_tensor_range(dev(padv(L["cal_amax"])), r2[:1], inv_s=dev(padv(L["cal_inv_s"])))
    assert host(r2)[0] == np.float32(L["cal_range"])


# ------------------------------------------------- producer-side quantization ----
P = load("producer_quant_2x3.txt")


@pytest.mark.parametrize("relu,key", [(True, "q_relu"), (False, "q_plain")])
@pytest.mark.parametrize("rows", [2, 300])
def test_fixture_producer_quant(sq, relu, key, rows):
    # N padded to 16 (the next linear's K) with zero weight rows, zero scales and zero 1/s;
    # 300 rows (the fixture's two rows repeated) run the CTA-pair kernel's int8 epilogue
    xq = np.tile(padk(i8(P["xq"])), (rows // 2, 1))
    sx = np.tile(f32(P["sx"]), rows // 2)
    wq = np.zeros((16, KP), np.int8)
    wq[:3] = padk(i8(P["wq"]))
    sw, inv = padv(P["sw"]), padv(P["inv_s"])
    bias = padv(P["bias"]).astype(np.float16)
    q = torch.empty((rows, 16), dtype=torch.int8, device="cuda")
    s = torch.empty(rows, dtype=torch.float32, device="cuda")
    rin = dev(np.array([P["range"], 0, 0, 0], np.float32))
    sq.sq_w8a8_linear_quant(dev(xq), dev(sx), dev(wq), dev(sw), rin[:1], q, s, bias=dev(bias), relu=relu,
                            inv_s_next=dev(inv), workspace=sq.new_workspace(rows, 16, KP))
    want = np.tile(padk(i8(P[key])), (rows // 2, 1))
    assert np.array_equal(host(q), want)
    assert bits_equal(host(s), np.full(rows, P["sx_next"][0], np.float32))
    assert sq.sq_poll_status() == 0


# ------------------------------------------------------------------- BMM ----
B = load("bmm_2x2x2.txt")


def test_fixture_bmm(sq):
    a = np.stack([padk(i8(B["a0"])), padk(i8(B["a1"]))])
    b = np.stack([padk(i8(B["b0"])), padk(i8(B["b1"]))])
    sa = np.stack([f32(B["as0"]), f32(B["as1"])])
    sb = np.stack([f32(B["bs0"]), f32(B["bs1"])])
    y = torch.empty((2, 2, 2), dtype=torch.float16, device="cuda")
    sq.sq_w8a8_bmm(dev(a), dev(sa), dev(b), dev(sb), y)
    assert bits_equal(host(y), np.stack([B["y0"], B["y1"]]).astype(np.float16))


# --------------------------------------------- the tutorial's printed example ----
def test_itmedia_53_through_the_gpu(sq):
    E = load("itmedia_53.txt")
    # a row whose absmax is 1270 has scale 10; 53 becomes 5.3, rounds to 5
    xq, sx = act_quant(sq, padk(np.array([E["row"]], np.float16)))
    assert sx[0] == np.float32(E["scale"])
    assert np.array_equal(xq[0, :2], i8(E["row_q"]))
    # reading 5 back with the scale gives 50 (the linear against a one-hot weight row, scale 1)
    wq = np.zeros((1, KP), np.int8)
    wq[0, 0] = 1
    y = torch.empty((1, 1), dtype=torch.float16, device="cuda")
    sq.sq_w8a8_linear(dev(xq), dev(sx), dev(wq), dev(np.ones(1, np.float32)), y,
                      workspace=sq.new_workspace(1, 1, KP))
    assert host(y)[0, 0] == np.float16(E["dequant"])
    assert float(E["x"]) - float(host(y)[0, 0]) == E["error"]


# ------------------------------------------- unsmoothed quality references ----
Q = load("quality_refs_2x3.txt")


def test_fixture_quality_refs_through_gpu(sq):
    """The two unsmoothed W8A8 baselines run on the library's own entry points: per token /
    per channel (sq_ln_quant_act, sq_quantize_weight) and naive per tensor (levels O2 for X,
    per-tensor weight)."""
    X, W = padk(Q["X"].astype(np.float16)), padk(Q["W"].astype(np.float16))
    bias = Q["bias"].astype(np.float16)
    xq, sx = act_quant(sq, X)
    wq, sw = weight_quant(sq, W)
    assert np.array_equal(xq, padk(i8(Q["ptpc_qx"]))) and np.array_equal(wq, padk(i8(Q["ptpc_qw"])))
    acc = torch.empty((3, 2), dtype=torch.int32, device="cuda")
    sq.sq_w8a8_gemm_s32(dev(xq), dev(wq), acc, workspace=sq.new_workspace(3, 2, KP))
    assert np.array_equal(host(acc), Q["ptpc_acc"].astype(np.int32))
    y = torch.empty((3, 2), dtype=torch.float16, device="cuda")
    sq.sq_w8a8_linear(dev(xq), dev(sx), dev(wq), dev(sw), y, dev(bias), workspace=sq.new_workspace(3, 2, KP))
    # power-of-two scales keep every step exact up to the last rounding:
    # y = fp16(acc * sx * sw + bias), the fixture's acc * sx * sw plus the bias (the zero row: bias)
    assert bits_equal(sx, np.array([2, 0.5, 0], np.float32)) and bits_equal(sw, np.array([1, 2], np.float32))
    assert bits_equal(host(y), (Q["ptpc_y"] + Q["bias"][None, :]).astype(np.float16))
    q = torch.empty((3, KP), dtype=torch.int8, device="cuda")
    s = torch.empty(3, dtype=torch.float32, device="cuda")
    r = torch.zeros(4, dtype=torch.float32, device="cuda")
    sq.sq_ln_quant_act_tensor(dev(X), q, s, r[:1])
    wq2 = torch.empty((2, KP), dtype=torch.int8, device="cuda")
    sw2 = torch.empty(2, dtype=torch.float32, device="cuda")
    r2 = torch.zeros(4, dtype=torch.float32, device="cuda")
    sq.sq_quantize_weight_tensor(dev(W), wq2, sw2, r2[:1])
    assert np.array_equal(host(q), padk(i8(Q["naive_qx"]))) and np.array_equal(host(wq2), padk(i8(Q["naive_qw"])))
    sq.sq_w8a8_gemm_s32(q, wq2, acc, workspace=sq.new_workspace(3, 2, KP))
    assert np.array_equal(host(acc), Q["naive_acc"].astype(np.int32))


# ------------------------------------------------------------ tie tensors ----
def tie_rows(rng, M, K, e_lo=-14, e_hi=4):
    """Rows whose absmax is 127 * 2^e (one element, random sign and place), so the per-row
    scale is exactly 2^e; the other elements are (k + 1/2) 2^e (ties), k 2^e, or arbitrary fp16
    values below the absmax.  Returns (x fp16 [M, K], e [M])."""
    e = rng.integers(e_lo, e_hi + 1, M)
    k = rng.integers(-127, 127, (M, K)).astype(np.float64)
    kind = rng.random((M, K))
    grid = np.where(kind < 0.5, k + 0.5, k)
    free = rng.uniform(-126.9, 126.9, (M, K))
    v = np.where(kind < 0.85, grid, free) * np.exp2(e)[:, None]
    x = v.astype(np.float16)
    top = rng.integers(0, K, M)
    x[np.arange(M), top] = (rng.choice([-127.0, 127.0], M) * np.exp2(e)).astype(np.float16)
    return x, e


def want_codes(x, e):
    """x * 2^-e is exact, so rint (ties to even) of it is the definition's code."""
    q = np.rint(x.astype(np.float64) * np.exp2(-e.astype(np.float64))[:, None])
    return np.clip(q, -127, 127).astype(np.int8)


TIE_SHAPES = [(300, 256), (300, 512), (300, 1024), (300, 2048), (300, 4096), (200, 4112), (150, 8192),
              (64, 12288), (48, 16384), (24, 24576), (12, 49152), (8, 65536)]


@pytest.mark.parametrize("M,K", TIE_SHAPES)
def test_ties_activation_codes(sq, M, K):
    rng = np.random.default_rng(M * 31 + K)
    x, e = tie_rows(rng, M, K)
    xq, sx = act_quant(sq, x)
    assert bits_equal(sx, np.exp2(e).astype(np.float32))
    want = want_codes(x, e)
    assert np.mean(np.abs(np.modf(x.astype(np.float64) * np.exp2(-e)[:, None])[0]) == 0.5) > 0.3
    assert np.array_equal(xq, want)
    # the smoothing multiply on the way in: x * 1/4 keeps every quotient (scale 2^(e-2))
    xq2, sx2 = act_quant(sq, x, inv_s=np.full(K, 0.25, np.float32))
    assert bits_equal(sx2, np.exp2(e - 2).astype(np.float32))
    assert np.array_equal(xq2, want)


@pytest.mark.parametrize("M,K", [(300, 256), (300, 4096), (150, 8192), (48, 16384), (12, 49152)])
def test_ties_layernorm_path(sq, M, K):
    """gamma = 0 makes the LayerNorm output beta exactly ((h - mu) rstd is finite), so the
    LayerNorm branch's rounding sees beta's ties in every row."""
    rng = np.random.default_rng(K + 7)
    beta, e = tie_rows(rng, 1, K)
    h = rng.standard_normal((M, K)).astype(np.float16)
    xq, sx = act_quant(sq, h, gamma=np.zeros(K, np.float32), beta=beta[0].astype(np.float32))
    assert bits_equal(sx, np.full(M, np.exp2(e[0]), np.float32))
    assert np.array_equal(xq, np.repeat(want_codes(beta, e), M, axis=0))


@pytest.mark.parametrize("N,K", [(300, 256), (300, 4096), (200, 4112), (150, 8192), (48, 16384),
                                 (12, 49152), (6, 65536)])
@pytest.mark.parametrize("s", [None, 2.0, 0.5])
def test_ties_weight_codes(sq, N, K, s):
    rng = np.random.default_rng(N + 3 * K)
    w, e = tie_rows(rng, N, K, e_lo=-12, e_hi=3)
    sv = None if s is None else np.full(K, s, np.float32)
    wq, sw = weight_quant(sq, w, sv)
    shift = 0 if s is None else int(np.log2(s))
    assert bits_equal(sw, np.exp2(e + shift).astype(np.float32))
    assert np.array_equal(wq, want_codes(w, e))


@pytest.mark.parametrize("M,K", [(300, 4096), (64, 12288), (12, 49152)])
def test_ties_static_range(sq, M, K):
    """Level O3: one static range 127 * 2^e; ties, and values past the range saturate."""
    rng = np.random.default_rng(K * 5)
    e = 2
    x, _ = tie_rows(rng, M, K, e_lo=e, e_hi=e)
    x[:, ::97] = (np.float16(300.0) * np.float16(2 ** e)) * np.sign(x[:, ::97] + np.float16(0.5))
    q = torch.empty((M, K), dtype=torch.int8, device="cuda")
    s = torch.empty(M, dtype=torch.float32, device="cuda")
    rin = dev(np.array([127 * 2 ** e, 0, 0, 0], np.float32))
    sq.sq_ln_quant_act_static(dev(x), q, s, rin[:1])
    assert bits_equal(host(s), np.full(M, 2.0 ** e, np.float32))
    assert np.array_equal(host(q), want_codes(x, np.full(M, e)))


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("with_bias", [False, True])
def test_ties_epilogue(sq, path, with_bias):
    """Unit scales make y = fp16(acc (+ bias)): odd accumulators in [2048, 4096), accumulators
    2 mod 4 in [4096, 8192) and acc + 1/2 in [1024, 2048) are exact ties of the fp16 rounding."""
    M = 20 if path == "splitk" else 300
    N, K = 264, 256
    rng = np.random.default_rng(M + with_bias)
    xq = rng.integers(-20, 21, (M, K)).astype(np.int8)
    wq = rng.integers(-20, 21, (N, K)).astype(np.int8)
    acc = xq.astype(np.int64) @ wq.astype(np.int64).T
    bias = np.full(N, 0.5, np.float16) if with_bias else None
    exact = acc.astype(np.float64) + (0.5 if with_bias else 0.0)
    ulp = np.spacing(np.abs(exact).astype(np.float16)).astype(np.float64)
    assert np.mean(np.abs(np.modf(exact / ulp)[0]) == 0.5) > 0.05  # many ties
    y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    sq.sq_w8a8_linear(dev(xq), dev(np.ones(M, np.float32)), dev(wq), dev(np.ones(N, np.float32)), y,
                      dev(bias), workspace=sq.new_workspace(M, N, K), path=path_id(sq, path))
    assert bits_equal(host(y), exact.astype(np.float16))
    assert sq.sq_poll_status() == 0
