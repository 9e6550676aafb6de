"""Each CUDA stage against the oracle on the same inputs, at sizes the oracle
finishes in seconds that still span several tiles and a ragged tail.
Stagewise: the oracle of a stage takes the GPU's output of the previous
stage, so every stage is checked bit for bit (the smoothing factor, which
goes through pow, within 1 fp32 ulp)."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import bits_equal, dev, f16_within, host, ulps32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sq(cuda_device):
    import w8a8_int8_linear_channel_b200 as m
    return m


def rand_h(rng, M, K, outliers=(), gain=60.0, shift=0.0):
    h = rng.standard_normal((M, K)).astype(np.float32) + np.float32(shift)
    for c in outliers:
        h[:, c] *= gain
    return h.astype(np.float16)


# ------------------------------------------------------------ calibration ----
# (4100, 4112) and (1030, 12304): many row bands per block of 256 columns, a
# ragged last band and a partial last column block
@pytest.mark.parametrize("rows,K", [(1, 16), (7, 48), (128, 256), (300, 4112), (33, 2064), (4100, 4112),
                                    (1030, 12304)])
def test_calibrate_absmax_raw(sq, rows, K):
    rng = np.random.default_rng(rows * 7 + K)
    x = rand_h(rng, rows, K, outliers=(0, K - 1, K // 3))
    amax = torch.zeros(K, dtype=torch.float32, device="cuda")
    sq.sq_calibrate_absmax(dev(x), amax)
    sq.sq_calibrate_absmax(dev(x[: max(1, rows // 2)] * np.float16(2)), amax)  # running max
    want = oracle.calibrate_absmax(x)
    want = oracle.calibrate_absmax(x[: max(1, rows // 2)] * np.float16(2), amax=want)
    assert bits_equal(host(amax), want)


# one case per kernel shape: a warp per row with 1, 2 or 4 chunks (K <= 256, 512, 1024), CTA
# rows of 64, 128 or 256 threads (K <= 2048, 4096, 8192, 16384; 3000 and 1500 rows: several
# rows per CTA, one of them with a ragged last chunk), and above 16384 the kernel whose CTAs
# re-read each row from global memory and merge their column maxima with atomics
@pytest.mark.parametrize("rows,K", [(5, 256), (6, 512), (64, 4096), (17, 1040), (12, 8192), (9, 16384),
                                    (3, 49152), (2, 65536), (3000, 4096), (1500, 2064)])
def test_calibrate_absmax_layernorm(sq, rows, K):
    rng = np.random.default_rng(rows + K)
    h = rand_h(rng, rows, K, shift=0.3)
    g = np.ones(K, np.float32)
    g[[1, K // 2]] = 60.0
    b = (rng.standard_normal(K) * 0.01).astype(np.float32)
    amax = torch.zeros(K, dtype=torch.float32, device="cuda")
    sq.sq_calibrate_absmax(dev(h), amax, dev(g), dev(b))
    assert bits_equal(host(amax), oracle.calibrate_absmax(h, gamma=g, beta=b))


@pytest.mark.parametrize("n", [1, 300, 3 * 4096])
def test_calibrate_reset_starts_a_new_run(sq, n):
    """sq_calibrate_reset zeroes stale maxima (several ranges back to back), so the next
    calibration equals one from a zero-filled buffer."""
    rng = np.random.default_rng(n)
    amax = dev(rng.uniform(10, 100, n).astype(np.float32))
    sq.sq_calibrate_reset(amax)
    assert not host(amax).any()
    if n < 16:
        return
    K = 16 * (n // 16)
    x = rand_h(rng, 33, K)
    sq.sq_calibrate_absmax(dev(x), amax[:K])
    assert bits_equal(host(amax)[:K], oracle.calibrate_absmax(x))
    assert not host(amax)[K:].any()


def test_calibrate_strided_rows(sq):
    rng = np.random.default_rng(3)
    full = rand_h(rng, 40, 320)
    t = dev(full)[:, :256]  # ld = 320
    amax = torch.zeros(256, dtype=torch.float32, device="cuda")
    sq.sq_calibrate_absmax(t, amax)
    assert bits_equal(host(amax), oracle.calibrate_absmax(np.ascontiguousarray(full[:, :256])))


# ------------------------------------------------------------ smooth/fold ----
@pytest.mark.parametrize("alpha", [0.0, 0.25, 0.5, 0.75, 0.85, 1.0])
def test_smooth_and_fold(sq, alpha):
    rng = np.random.default_rng(int(alpha * 100))
    K, N = 4096, 72
    a = np.exp(rng.uniform(-9, 6, K)).astype(np.float32)
    b = np.exp(rng.uniform(-9, 2, K)).astype(np.float32)
    a[:3] = 0.0  # dead channels hit the 1e-5 floor
    b[3:5] = 0.0
    g = rng.standard_normal(K).astype(np.float32)
    be = rng.standard_normal(K).astype(np.float32)
    w = (rng.standard_normal((N, K)) * 0.02).astype(np.float16)
    s, inv_s = torch.empty(K, device="cuda"), torch.empty(K, device="cuda")
    g_o, b_o = torch.empty(K, device="cuda"), torch.empty(K, device="cuda")
    w_o = torch.empty((N, K), dtype=torch.float16, device="cuda")
    sq.sq_smooth_fold(dev(a), dev(b), alpha, s, inv_s, dev(g), dev(be), g_o, b_o, dev(w), w_o)
    s_ref, inv_ref = oracle.smooth(a, b, alpha)
    assert ulps32(host(s), s_ref).max() <= 1
    s_g, inv_g = host(s), host(inv_s)
    assert bits_equal(inv_g, (np.float32(1) / s_g).astype(np.float32))
    g_ref, b_ref = oracle.fold_ln(g, be, inv_g)
    assert bits_equal(host(g_o), g_ref) and bits_equal(host(b_o), b_ref)
    assert bits_equal(host(w_o), oracle.fold_weight(w, s_g))


def test_fold_weight_in_place(sq):
    rng = np.random.default_rng(5)
    K, N = 256, 40
    w = (rng.standard_normal((N, K)) * 0.02).astype(np.float16)
    a = np.abs(rng.standard_normal(K)).astype(np.float32) + 1
    b = np.abs(w.astype(np.float32)).max(0)
    s, inv_s = torch.empty(K, device="cuda"), torch.empty(K, device="cuda")
    wt = dev(w)
    sq.sq_smooth_fold(dev(a), dev(b), 0.5, s, inv_s, w=wt, w_out=wt)
    assert bits_equal(host(wt), oracle.fold_weight(w, host(s)))


# --------------------------------------------------------- weight quantize ----
@pytest.mark.parametrize("N,K,fold", [(1, 16, False), (77, 48, True), (11, 512, True), (21, 2048, True),
                                      (300, 4112, True), (256, 256, False), (5, 16384, False),
                                      (40, 16400, True), (13, 49152, True), (1100, 4096, True),
                                      (9, 12288, True), (150, 1552, False)])
def test_quantize_weight(sq, N, K, fold):
    rng = np.random.default_rng(N + K)
    w = (rng.standard_normal((N, K)) * 0.02).astype(np.float16)
    w[min(3, N - 1)] = 0  # an all-zero row
    s = rng.uniform(0.05, 20, K).astype(np.float32) if fold else None
    wq = torch.empty((N, K), dtype=torch.int8, device="cuda")
    sw = torch.empty(N, dtype=torch.float32, device="cuda")
    sq.sq_quantize_weight(dev(w), wq, sw, s=dev(s))
    w_ref = oracle.fold_weight(w, s) if fold else w
    wq_ref, sw_ref = oracle.quantize_weight(w_ref)
    assert bits_equal(host(sw), sw_ref)
    assert bits_equal(host(wq), wq_ref)


# ---------------------------------------------------------- LN + quantize ----
@pytest.mark.parametrize("M,K,mode", [(1, 16, "plain"), (16, 256, "inv_s"), (9, 512, "ln"), (33, 4096, "ln"),
                                      (129, 1040, "ln_inv_s"), (6, 8192, "inv_s"), (7, 12288, "ln"),
                                      (3, 16384, "ln_inv_s"), (5, 49152, "inv_s"), (3, 65536, "inv_s"),
                                      (2, 49152, "ln")])
def test_ln_quant_act(sq, M, K, mode):
    rng = np.random.default_rng(M * K)
    h = rand_h(rng, M, K, outliers=(2, K - 3), shift=0.2)
    h[0, :] = 0  # all-zero row (constant under LN: output beta)
    g = b = inv = None
    if "ln" in mode:
        g = rng.uniform(0.5, 2.0, K).astype(np.float32)
        g[[2, K - 3]] = 70.0
        b = (rng.standard_normal(K) * 0.01).astype(np.float32)
    if "inv_s" in mode:
        inv = rng.uniform(0.02, 2.0, K).astype(np.float32)
    xq = torch.empty((M, K), dtype=torch.int8, device="cuda")
    sx = torch.empty(M, dtype=torch.float32, device="cuda")
    sq.sq_ln_quant_act(dev(h), xq, sx, dev(g), dev(b), dev(inv))
    xq_ref, sx_ref = oracle.ln_quant_act(h, g, b, inv)
    assert bits_equal(host(sx), sx_ref)
    assert bits_equal(host(xq), xq_ref)


# ------------------------------------------------------------------ GEMM ----
# K = 496 / 512 / 528: the pair kernel's one-box ring below K = 512, two-box stages from there
# (528: the last stage's second box lies wholly past K).  33 / 64 / 127 / 128 tokens: the
# stream-K kernel's 64- and 128-token tiles; (64, 520, 8208) and (128, 1000, 4112) split
# their channel tiles between CTAs
GEMM_SHAPES = [(1, 8, 16), (5, 100, 48), (16, 256, 256), (17, 260, 144), (32, 1000, 4112),
               (33, 77, 16), (64, 520, 8208), (127, 513, 272), (128, 1000, 4112), (129, 256, 4096),
               (300, 1000, 2064), (256, 520, 528), (260, 300, 496), (513, 264, 512)]


def _rand_i8(rng, M, N, K):
    xq = rng.integers(-127, 128, (M, K)).astype(np.int8)
    wq = rng.integers(-127, 128, (N, K)).astype(np.int8)
    sx = rng.uniform(1e-4, 0.1, M).astype(np.float32)
    sw = rng.uniform(1e-4, 0.1, N).astype(np.float32)
    sx[0] = 0.0
    bias = (rng.standard_normal(N) * 0.5).astype(np.float16)
    return xq, wq, sx, sw, bias


_PATHS = {"tiled": lambda m: m.PATH_TILED, "splitk": lambda m: m.PATH_SPLITK,
          "pair": lambda m: m.PATH_PAIR}


@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
@pytest.mark.parametrize("path", ["tiled", "splitk", "pair"])
def test_gemm_accumulators_bit_exact(sq, M, N, K, path):
    if path == "splitk" and M > sq.SPLITK_MAX_M:
        pytest.skip("stream-K path serves M <= 128")
    rng = np.random.default_rng(M * 1000003 + N * 101 + K)
    xq, wq, _, _, _ = _rand_i8(rng, M, N, K)
    p = _PATHS[path](sq)
    ws = sq.new_workspace(M, N, K) if path == "splitk" else None
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    sq.sq_w8a8_gemm_s32(dev(xq), dev(wq), acc, workspace=ws, path=p)
    assert sq.sq_poll_status() == 0
    assert np.array_equal(host(acc), oracle.int_gemm(xq, wq))


@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
@pytest.mark.parametrize("path", ["tiled", "splitk", "pair"])
@pytest.mark.parametrize("with_bias", [False, True])
def test_linear_output(sq, M, N, K, path, with_bias):
    if path == "splitk" and M > sq.SPLITK_MAX_M:
        pytest.skip("stream-K path serves M <= 128")
    rng = np.random.default_rng(M * 7919 + N * 31 + K + with_bias)
    xq, wq, sx, sw, bias = _rand_i8(rng, M, N, K)
    bias = bias if with_bias else None
    p = _PATHS[path](sq)
    ws = sq.new_workspace(M, N, K) if path == "splitk" else None
    y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    sq.sq_w8a8_linear(dev(xq), dev(sx), dev(wq), dev(sw), y, dev(bias), workspace=ws, path=p)
    ref = oracle.w8a8_linear(xq, sx, wq, sw, bias)
    got = host(y)
    assert f16_within(got, ref)
    assert bits_equal(got, ref)


# The CTA-pair kernel's persistent walk: fewer tiles than pairs, a partial last wave (the
# attention shape: 128 tiles on 74 pairs), ragged N and M, and more than two waves in grouped
# order.
@pytest.mark.parametrize("M,N,K", [(512, 4160, 272), (2048, 4096, 528), (300, 2000, 1040),
                                   (2100, 8200, 272)])
@pytest.mark.parametrize("with_bias", [False, True])
def test_pair_kernel_persistent_walks(sq, M, N, K, with_bias):
    rng = np.random.default_rng(M + N + K + with_bias)
    xq, wq, sx, sw, bias = _rand_i8(rng, M, N, K)
    bias = bias if with_bias else None
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    sq.sq_w8a8_gemm_s32(dev(xq), dev(wq), acc, path=sq.PATH_PAIR)
    assert np.array_equal(host(acc), oracle.int_gemm(xq, wq))
    y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    sq.sq_w8a8_linear(dev(xq), dev(sx), dev(wq), dev(sw), y, dev(bias), path=sq.PATH_PAIR)
    assert bits_equal(host(y), oracle.w8a8_linear(xq, sx, wq, sw, bias))
    assert sq.sq_poll_status() == 0


def test_splitk_many_contributors_per_tile(sq):
    # few channel tiles, long K: every tile is shared by many CTAs
    rng = np.random.default_rng(11)
    M, N, K = 8, 256, 16384
    xq, wq, sx, sw, bias = _rand_i8(rng, M, N, K)
    ws = sq.new_workspace(M, N, K)
    for _ in range(3):  # counters must come back to zero after every call
        y = torch.empty((M, N), dtype=torch.float16, device="cuda")
        sq.sq_w8a8_linear(dev(xq), dev(sx), dev(wq), dev(sw), y, dev(bias), workspace=ws,
                          path=sq.PATH_SPLITK)
        assert bits_equal(host(y), oracle.w8a8_linear(xq, sx, wq, sw, bias))
    assert sq.sq_poll_status() == 0


@pytest.mark.parametrize("path", ["tiled", "splitk", "pair"])
def test_linear_large_accumulators(sq, path):
    # rows of +-127 codes against +-127 weight rows make |acc| = 127^2 K, far
    # above 2^22 (beyond exact conversion through 1.5 * 2^23 + acc); the other
    # rows stay small, so one tile holds both kinds of 32-value chunks
    M = 16 if path == "splitk" else 300
    N, K = 520, 8192
    rng = np.random.default_rng(17)
    xq = rng.integers(-3, 4, (M, K)).astype(np.int8)
    wq = rng.integers(-127, 128, (N, K)).astype(np.int8)
    big = rng.choice(M, M // 3, replace=False)
    xq[big] = rng.choice([-127, 127], (big.size, 1)).astype(np.int8)
    wq[::7] = rng.choice([-127, 127], (len(range(0, N, 7)), 1)).astype(np.int8)
    sx = rng.uniform(1e-7, 1e-6, M).astype(np.float32)
    sw = rng.uniform(1e-4, 1e-3, N).astype(np.float32)
    bias = (rng.standard_normal(N) * 0.5).astype(np.float16)
    acc = oracle.int_gemm(xq, wq)
    assert (np.abs(acc) >= 2 ** 22).any() and (np.abs(acc) < 2 ** 22).any()
    y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    sq.sq_w8a8_linear(dev(xq), dev(sx), dev(wq), dev(sw), y, dev(bias), workspace=sq.new_workspace(M, N, K),
                      path=_PATHS[path](sq))
    assert bits_equal(host(y), oracle.dequant(acc, sx, sw, bias))
    assert sq.sq_poll_status() == 0


def test_extreme_codes_do_not_wrap(sq):
    K = 133136  # the largest multiple of 16 <= 133144
    xq = np.full((2, K), 127, np.int8)
    xq[1] = -127
    wq = np.full((3, K), 127, np.int8)
    wq[2] = -127
    for path in (sq.PATH_TILED, sq.PATH_SPLITK, sq.PATH_PAIR):
        acc = torch.empty((2, 3), dtype=torch.int32, device="cuda")
        ws = sq.new_workspace(2, 3, K)
        sq.sq_w8a8_gemm_s32(dev(xq), dev(wq), acc, workspace=ws, path=path)
        assert np.array_equal(host(acc), oracle.int_gemm64(xq, wq))
