"""Guard bands around every buffer an entry point writes.

Each output (and the stream-K workspace) is the middle of a larger allocation
whose 4 KiB margins hold a byte pattern; after the call the pattern must be
intact on both sides.  A store past a tensor's end -- a ragged tile's tail, a
clipped TMA box, a stream-K partial slot indexed one slot too far -- changes a
margin byte even when every value inside comes out right, and on a device
without a memory checker this is how such a store shows.  The values inside
are checked against the oracle as in the stage parity tests, on ragged shapes
that end mid-tile in every dimension.  Collected after the other GPU tests and
before the allocation-free entry point's test."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import bits_equal, dev, host, ulps32

PAD = 4096
FILL = 0xA5


class Banded:
    """A tensor of `shape` / `dtype` inside PAD bytes of FILL on each side (16-byte aligned)."""

    def __init__(self, shape, dtype, device="cuda", zero=False):
        shape = tuple(shape)
        self.nbytes = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        self.buf = torch.full((PAD + self.nbytes + PAD,), FILL, dtype=torch.uint8, device=device)
        self.t = self.buf[PAD:PAD + self.nbytes].view(dtype).view(shape)
        if zero:
            self.t.zero_()

    def intact(self):
        head = self.buf[:PAD]
        tail = self.buf[PAD + self.nbytes:]
        return bool((head == FILL).all().item()) and bool((tail == FILL).all().item())


def _all_intact(*bands):
    return all(b.intact() for b in bands)


# ------------------------------------------------- the detector itself (CPU) ----
def test_bands_detect_a_store_on_either_side():
    for dtype, shape in ((torch.float16, (3, 5)), (torch.int32, (7,)), (torch.int8, (2, 9))):
        b = Banded(shape, dtype, device="cpu", zero=True)
        assert b.t.data_ptr() % 16 == 0 and b.t.shape == shape and b.t.is_contiguous()
        b.t.fill_(1)  # every value inside
        assert b.intact()
        b.buf[PAD + b.nbytes] = 0  # one byte past the end
        assert not b.intact()
        b2 = Banded(shape, dtype, device="cpu")
        b2.buf[PAD - 1] = 0  # one byte before the start
        assert not b2.intact()


# ------------------------------------------------------------ GPU fixtures ----
@pytest.fixture(scope="module")
def sq(cuda_device):
    import w8a8_int8_linear_channel_b200 as m
    return m


def _rand_i8(rng, M, N, K):
    xq = rng.integers(-127, 128, (M, K)).astype(np.int8)
    wq = rng.integers(-127, 128, (N, K)).astype(np.int8)
    sx = rng.uniform(1e-4, 0.1, M).astype(np.float32)
    sw = rng.uniform(1e-4, 0.1, N).astype(np.float32)
    bias = (rng.standard_normal(N) * 0.5).astype(np.float16)
    return xq, wq, sx, sw, bias


# ragged in M, N and K; 33-128 tokens take the stream-K kernel's 64- and 128-token tiles
LINEAR_SHAPES = [(5, 100, 48), (33, 77, 16), (64, 520, 8208), (127, 513, 272), (128, 1000, 4112),
                 (300, 1000, 2064), (256, 520, 528), (513, 264, 512)]
PATHS = {"tiled": "PATH_TILED", "splitk": "PATH_SPLITK", "pair": "PATH_PAIR"}


@pytest.mark.gpu
@pytest.mark.parametrize("M,N,K", LINEAR_SHAPES)
@pytest.mark.parametrize("path", sorted(PATHS))
def test_linear_and_accumulators_stay_in_bounds(sq, M, N, K, path):
    if path == "splitk" and M > sq.SPLITK_MAX_M:
        pytest.skip("stream-K path serves M <= 128")
    rng = np.random.default_rng(M * 131 + N * 7 + K)
    xq, wq, sx, sw, bias = _rand_i8(rng, M, N, K)
    p = getattr(sq, PATHS[path])
    need = sq.sq_w8a8_workspace_bytes(M, N, K) if path == "splitk" else 0
    ws = Banded((need,), torch.uint8, zero=True) if need else None
    y = Banded((M, N), torch.float16)
    sq.sq_w8a8_linear(dev(xq), dev(sx), dev(wq), dev(sw), y.t, dev(bias), workspace=ws.t if ws else None, path=p)
    acc = Banded((M, N), torch.int32)
    sq.sq_w8a8_gemm_s32(dev(xq), dev(wq), acc.t, workspace=ws.t if ws else None, path=p)
    assert sq.sq_poll_status() == 0
    assert _all_intact(y, acc, *([ws] if ws else []))
    assert bits_equal(host(y.t), oracle.w8a8_linear(xq, sx, wq, sw, bias))
    assert np.array_equal(host(acc.t), oracle.int_gemm(xq, wq))


@pytest.mark.gpu
@pytest.mark.parametrize("M,N,K", [(1, 16, 16), (5, 272, 48), (33, 256, 256), (300, 1008, 2064)])
def test_producer_quantization_stays_in_bounds(sq, M, N, K):
    rng = np.random.default_rng(M * 17 + N + K)
    xq, wq, sx, sw, bias = _rand_i8(rng, M, N, K)
    sx = (sx * 0.02).astype(np.float32)
    sw = (sw * 0.02).astype(np.float32)
    inv = rng.uniform(0.05, 3.0, N).astype(np.float32)
    y = oracle.w8a8_linear(xq, sx, wq, sw, bias).astype(np.float32)
    x = np.maximum(y, 0) * inv[None, :]
    r = np.float32(np.abs(x[np.isfinite(x)]).max() * 0.6)
    q = Banded((M, N), torch.int8)
    s = Banded((M,), torch.float32)
    ws = sq.new_workspace(M, N, K)
    sq.sq_w8a8_linear_quant(dev(xq), dev(sx), dev(wq), dev(sw), dev(np.array([r], np.float32)), q.t, s.t,
                            bias=dev(bias), relu=True, inv_s_next=dev(inv), workspace=ws)
    assert sq.sq_poll_status() == 0
    assert _all_intact(q, s)
    q_ref, s_ref = oracle.w8a8_linear_quant_static(xq, sx, wq, sw, bias, relu=True, inv_s_next=inv, range_next=r)
    assert bits_equal(host(s.t), s_ref)
    assert bits_equal(host(q.t), q_ref)


@pytest.mark.gpu
@pytest.mark.parametrize("B,M,N,K", [(1, 1, 16, 16), (3, 37, 40, 48), (4, 300, 272, 144), (5, 129, 513, 1040)])
def test_bmm_stays_in_bounds(sq, B, M, N, K):
    rng = np.random.default_rng(B * 7 + M + N + K)
    a = rng.integers(-127, 128, (B, M, K)).astype(np.int8)
    b = rng.integers(-127, 128, (B, N, K)).astype(np.int8)
    sa = rng.uniform(1e-3, 1e-2, (B, M)).astype(np.float32)
    sb = rng.uniform(1e-3, 1e-2, (B, N)).astype(np.float32)
    y = Banded((B, M, N), torch.float16)
    sq.sq_w8a8_bmm(dev(a), dev(sa), dev(b), dev(sb), y.t)
    assert sq.sq_poll_status() == 0
    assert y.intact()
    assert bits_equal(host(y.t), oracle.w8a8_bmm(a, sa, b, sb))


def _act_inputs(rng, M, K, mode):
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


ACT_SHAPES = [(1, 16, "plain"), (37, 256, "inv_s"), (33, 4096, "ln"), (5, 49152, "ln_inv_s"), (3, 65536, "inv_s")]


@pytest.mark.gpu
@pytest.mark.parametrize("M,K,mode", ACT_SHAPES)
def test_activation_quantization_stays_in_bounds(sq, M, K, mode):
    rng = np.random.default_rng(M * 5 + K)
    h, g, b, inv = _act_inputs(rng, M, K, mode)
    # per token (dynamic)
    xq, sx = Banded((M, K), torch.int8), Banded((M,), torch.float32)
    sq.sq_ln_quant_act(dev(h), xq.t, sx.t, dev(g), dev(b), dev(inv))
    q_ref, s_ref = oracle.ln_quant_act(h, g, b, inv)
    assert _all_intact(xq, sx)
    assert bits_equal(host(sx.t), s_ref) and bits_equal(host(xq.t), q_ref)
    # one dynamic range for the batch (O2)
    xq2, sx2, r2 = Banded((M, K), torch.int8), Banded((M,), torch.float32), Banded((1,), torch.float32)
    sq.sq_ln_quant_act_tensor(dev(h), xq2.t, sx2.t, r2.t, dev(g), dev(b), dev(inv))
    q_ref, s_ref, r_ref = oracle.ln_quant_act_tensor(h, g, b, inv)
    assert _all_intact(xq2, sx2, r2)
    assert bits_equal(host(r2.t), np.float32(r_ref).reshape(1))
    assert bits_equal(host(sx2.t), s_ref) and bits_equal(host(xq2.t), q_ref)
    # a static range (O3), part of the batch saturating
    r = np.float32(np.abs(oracle.act_rows(h, g, b, inv)).max() * 0.4)
    xq3, sx3 = Banded((M, K), torch.int8), Banded((M,), torch.float32)
    sq.sq_ln_quant_act_static(dev(h), xq3.t, sx3.t, dev(np.array([r], np.float32)), dev(g), dev(b), dev(inv))
    q_ref, s_ref = oracle.ln_quant_act_static(h, r, g, b, inv)
    assert _all_intact(xq3, sx3)
    assert bits_equal(host(sx3.t), s_ref) and bits_equal(host(xq3.t), q_ref)
    # calibration: running column maxima of the same rows (of their LayerNorm at the widths
    # the LayerNorm calibration stage tests run)
    gl, bl = (g, b) if K <= 16384 else (None, None)
    amax = Banded((K,), torch.float32, zero=True)
    sq.sq_calibrate_absmax(dev(h), amax.t, dev(gl), dev(bl))
    assert amax.intact()
    assert bits_equal(host(amax.t), oracle.calibrate_absmax(h, gamma=gl, beta=bl))
    assert sq.sq_poll_status() == 0


@pytest.mark.gpu
@pytest.mark.parametrize("N,K,fold", [(1, 16, False), (77, 48, True), (300, 4112, True), (40, 16400, True),
                                      (13, 49152, True)])
def test_weight_quantization_stays_in_bounds(sq, N, K, fold):
    rng = np.random.default_rng(N * 3 + K + 1)
    w = (rng.standard_normal((N, K)) * 0.02).astype(np.float16)
    s = rng.uniform(0.05, 20, K).astype(np.float32) if fold else None
    w_ref = oracle.fold_weight(w, s) if fold else w
    wq, sw = Banded((N, K), torch.int8), Banded((N,), torch.float32)
    sq.sq_quantize_weight(dev(w), wq.t, sw.t, s=dev(s))
    wq_ref, sw_ref = oracle.quantize_weight(w_ref)
    assert _all_intact(wq, sw)
    assert bits_equal(host(sw.t), sw_ref) and bits_equal(host(wq.t), wq_ref)
    wq2, sw2, r2 = Banded((N, K), torch.int8), Banded((N,), torch.float32), Banded((1,), torch.float32, zero=True)
    sq.sq_quantize_weight_tensor(dev(w), wq2.t, sw2.t, r2.t, s=dev(s))
    wq_ref, sw_ref, r_ref = oracle.quantize_weight_tensor(w_ref)
    assert _all_intact(wq2, sw2, r2)
    assert bits_equal(host(r2.t), np.float32(r_ref).reshape(1))
    assert bits_equal(host(sw2.t), sw_ref) and bits_equal(host(wq2.t), wq_ref)
    assert sq.sq_poll_status() == 0


@pytest.mark.gpu
@pytest.mark.parametrize("K,N", [(16, 1), (4112, 72), (49152, 3)])
def test_smoothing_and_fold_stay_in_bounds(sq, K, N):
    rng = np.random.default_rng(K + N)
    a = np.exp(rng.uniform(-9, 6, K)).astype(np.float32)
    b = np.exp(rng.uniform(-9, 2, K)).astype(np.float32)
    g = rng.standard_normal(K).astype(np.float32)
    be = rng.standard_normal(K).astype(np.float32)
    w = (rng.standard_normal((N, K)) * 0.02).astype(np.float16)
    s, inv_s, g_o, b_o = (Banded((K,), torch.float32) for _ in range(4))
    w_o = Banded((N, K), torch.float16)
    sq.sq_smooth_fold(dev(a), dev(b), 0.5, s.t, inv_s.t, dev(g), dev(be), g_o.t, b_o.t, dev(w), w_o.t)
    r = Banded((1,), torch.float32, zero=True)
    sq.sq_tensor_range(dev(a), r.t, inv_s=inv_s.t)
    assert _all_intact(s, inv_s, g_o, b_o, w_o, r)
    s_ref, _ = oracle.smooth(a, b, 0.5)
    assert ulps32(host(s.t), s_ref).max() <= 1
    s_g, inv_g = host(s.t), host(inv_s.t)
    assert bits_equal(inv_g, (np.float32(1) / s_g).astype(np.float32))
    g_ref, b_ref = oracle.fold_ln(g, be, inv_g)
    assert bits_equal(host(g_o.t), g_ref) and bits_equal(host(b_o.t), b_ref)
    assert bits_equal(host(w_o.t), oracle.fold_weight(w, s_g))
    assert bits_equal(host(r.t), np.float32(oracle.tensor_range(a, inv_g)).reshape(1))
    assert sq.sq_poll_status() == 0


@pytest.mark.gpu
@pytest.mark.parametrize("rows,K,mode", [(1, 16, "act"), (37, 256, "act_inv"), (9, 20480, "act_inv"),
                                         (19, 4096, "fold"), (5, 49152, "fold")])
def test_sharded_row_steps_stay_in_bounds(sq, rows, K, mode):
    rng = np.random.default_rng(rows * 13 + K + 1)
    x = (rng.standard_normal((rows, K)) * 2).astype(np.float16)
    vec = rng.uniform(0.05, 3.0, K).astype(np.float32)
    inv = vec if mode == "act_inv" else None
    s_fold = vec if mode == "fold" else None
    xr = oracle.fold_weight(x, s_fold).astype(np.float32) if s_fold is not None else oracle.act_rows(x, inv_s=inv)
    r = Banded((rows,), torch.float32)
    sq.sq_row_ranges(dev(x), r.t, inv_s=dev(inv), s_fold=dev(s_fold))
    given = (np.abs(xr).max(1) * rng.choice([1.0, 1.5], rows)).astype(np.float32)
    q, sc = Banded((rows, K), torch.int8), Banded((rows,), torch.float32)
    sq.sq_quantize_rows_ranged(dev(x), dev(given), q.t, sc.t, inv_s=dev(inv), s_fold=dev(s_fold))
    assert sq.sq_poll_status() == 0
    assert _all_intact(r, q, sc)
    assert bits_equal(host(r.t), np.abs(xr).max(1).astype(np.float32))
    sc_ref = (given / np.float32(127)).astype(np.float32)
    q_ref = np.stack([oracle.quantize_with_scale(xr[i], sc_ref[i]) for i in range(rows)])
    assert bits_equal(host(sc.t), sc_ref) and bits_equal(host(q.t), q_ref)


@pytest.mark.gpu
@pytest.mark.parametrize("M,N", [(1, 4), (33, 260), (300, 4096)])
def test_dequant_stays_in_bounds(sq, M, N):
    rng = np.random.default_rng(M + N + 3)
    acc = rng.integers(-2 ** 28, 2 ** 28, (M, N)).astype(np.int32)
    sx = rng.uniform(1e-5, 1e-3, M).astype(np.float32)
    sw = rng.uniform(1e-5, 1e-3, N).astype(np.float32)
    bias = rng.standard_normal(N).astype(np.float16)
    y = Banded((M, N), torch.float16)
    sq.sq_dequant(dev(acc), dev(sx), dev(sw), y.t, dev(bias))
    assert sq.sq_poll_status() == 0
    assert y.intact()
    assert bits_equal(host(y.t), oracle.dequant(acc, sx, sw, bias))


@pytest.mark.gpu
@pytest.mark.parametrize("M,N,K", [(8, 1000, 4112), (20, 256, 16384), (32, 1000, 4112)])
def test_allocation_free_linear_stays_in_bounds(sq, M, N, K):
    rng = np.random.default_rng(M + N + K)
    xq, wq, sx, sw, bias = _rand_i8(rng, M, N, K)
    y = Banded((M, N), torch.float16)
    sq.sq_w8a8_linear_noalloc(dev(xq), dev(sx), dev(wq), dev(sw), y.t, bias=dev(bias))
    assert sq.sq_poll_status() == 0
    assert y.intact()
    assert bits_equal(host(y.t), oracle.w8a8_linear(xq, sx, wq, sw, bias))
