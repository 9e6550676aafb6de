"""Producer-side quantization at the next linear's per-token dynamic scale on the GPU, bit for
bit against the oracle (the composition of the linear, the ReLU and the per-token quantizer
with 1/s): the stream-K kernel (M <= 32) and the CTA-pair kernel (larger M) with the second
launch that codes each row at its own maximum; ragged shapes, zero rows, non-finite outputs,
repeated calls on one workspace, the hand-worked fixture and the unfused GPU chain."""
import numpy as np
import pytest
import torch

import oracle
from golden_io import load
from gpu_util import bits_equal, dev, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sq(cuda_device):
    import w8a8_int8_linear_channel_b200 as m
    return m


def _case(M, N, K, seed):
    rng = np.random.default_rng(seed)
    xq = rng.integers(-127, 128, (M, K)).astype(np.int8)
    wq = rng.integers(-127, 128, (N, K)).astype(np.int8)
    sx = rng.uniform(1e-4, 2e-3, M).astype(np.float32)
    sx[min(2, M - 1)] = 0.0  # a row whose y is the bias alone
    sw = rng.uniform(1e-4, 2e-3, N).astype(np.float32)
    bias = (rng.standard_normal(N) * 0.5).astype(np.float16)
    inv = rng.uniform(0.05, 3.0, N).astype(np.float32)
    return xq, sx, wq, sw, bias, inv


def _run(sq, xq, sx, wq, sw, bias, relu, inv, ws=None):
    M, N = xq.shape[0], wq.shape[0]
    q = torch.empty((M, N), dtype=torch.int8, device="cuda")
    s = torch.empty(M, dtype=torch.float32, device="cuda")
    sq.sq_w8a8_linear_quant_dyn(dev(xq), dev(sx), dev(wq), dev(sw), q, s, bias=dev(bias), relu=relu,
                                inv_s_next=dev(inv), workspace=ws)
    return q, s


SHAPES = [(1, 16, 16), (5, 272, 48), (16, 1040, 4112), (17, 48, 256), (32, 4096, 1024), (33, 256, 256),
          (129, 1008, 2064), (300, 16, 528), (513, 4096, 1024), (600, 2064, 512)]


@pytest.mark.parametrize("M,N,K", SHAPES)
@pytest.mark.parametrize("relu", [False, True])
@pytest.mark.parametrize("variant", ["bias_inv_s", "plain"])
def test_producer_dynamic(sq, M, N, K, relu, variant):
    xq, sx, wq, sw, bias, inv = _case(M, N, K, M * 131 + N + K + relu)
    if variant == "plain":
        bias, inv = None, None
    q, s = _run(sq, xq, sx, wq, sw, bias, relu, inv)
    q_ref, s_ref = oracle.w8a8_linear_quant_dynamic(xq, sx, wq, sw, bias, relu=relu, inv_s_next=inv)
    assert sq.sq_poll_status() == 0
    assert bits_equal(host(s), s_ref)
    assert bits_equal(host(q), q_ref)


@pytest.mark.parametrize("M", [7, 300])
def test_producer_dynamic_repeated_calls_share_a_workspace(sq, M):
    N, K = 1040, 4112
    ws = sq.new_quant_dyn_workspace(M, N, K)
    for seed in range(3):  # stream-K counters back at zero and stale row maxima overwritten
        xq, sx, wq, sw, bias, inv = _case(M, N, K, 900 + seed)
        q, s = _run(sq, xq, sx, wq, sw, bias, True, inv, ws=ws)
        q_ref, s_ref = oracle.w8a8_linear_quant_dynamic(xq, sx, wq, sw, bias, relu=True, inv_s_next=inv)
        assert bits_equal(host(s), s_ref) and bits_equal(host(q), q_ref)
    assert sq.sq_poll_status() == 0


@pytest.mark.parametrize("M", [4, 260])
def test_producer_dynamic_non_finite(sq, M):
    """Outputs that overflow fp16 (Inf) and NaN scales follow the per-token quantizer's IEEE
    rules: an Inf in a row makes its scale Inf and every code 0; a NaN is coded 0 and never
    sets a range; the ReLU turns a NaN into 0."""
    N, K = 272, 256
    xq, sx, wq, sw, bias, inv = _case(M, N, K, 5)
    xq[1, :] = 127
    wq[3, :] = 127
    sx[1] = 1e3  # row 1, channel 3: 127 * 127 * 256 * 1e3 * sw overflows fp16 -> Inf
    sw[3] = 1.0
    sw[5] = np.nan  # channel 5: NaN in every row
    for relu in (False, True):
        q, s = _run(sq, xq, sx, wq, sw, bias, relu, inv)
        q_ref, s_ref = oracle.w8a8_linear_quant_dynamic(xq, sx, wq, sw, bias, relu=relu, inv_s_next=inv)
        assert bits_equal(host(s), s_ref) and bits_equal(host(q), q_ref)
        assert np.isinf(host(s)[1]) and np.all(host(q)[1] == 0)


@pytest.mark.parametrize("rows", [3, 300])
def test_fixture_producer_dynamic(sq, rows):
    P = load("producer_dyn_3x3.txt")
    rep = rows // 3
    pad = lambda a: np.pad(np.asarray(a), ((0, 0), (0, 16 - np.asarray(a).shape[1])))
    xq = np.tile(pad(P["xq"].astype(np.int8)), (rep, 1))
    sx = np.tile(P["sx"].astype(np.float32), rep)
    wq = np.zeros((16, 16), np.int8)
    wq[:3] = pad(P["wq"].astype(np.int8))
    sw = np.zeros(16, np.float32)
    sw[:3] = P["sw"]
    bias = np.zeros(16, np.float16)
    bias[:3] = P["bias"]
    inv = np.zeros(16, np.float32)
    inv[:3] = P["inv_s"]
    q, s = _run(sq, xq, sx, wq, sw, bias, True, inv)
    assert np.array_equal(host(q)[:, :3], np.tile(P["q_relu"].astype(np.int8), (rep, 1)))
    assert np.all(host(q)[:, 3:] == 0)
    assert bits_equal(host(s), np.tile(P["sx_relu"].astype(np.float32), rep))
    q, s = _run(sq, xq, sx, wq, sw, bias, False, inv)
    assert np.array_equal(host(q)[:, :3], np.tile(P["q_plain"].astype(np.int8), (rep, 1)))
    sp = host(s).reshape(rep, 3)
    assert bits_equal(sp[:, :2], np.tile(P["sx_plain_rows01"].astype(np.float32), (rep, 1)))
    assert np.all(sp[:, 2] == np.float32(0.375) / np.float32(127))


@pytest.mark.parametrize("M", [24, 200])
def test_producer_dynamic_matches_unfused_gpu_chain(sq, M):
    """The fused codes equal the library's unfused path: sq_w8a8_linear to fp16, ReLU, then the
    per-token quantization sq_ln_quant_act with the next linear's 1/s."""
    N, K = 1024, 512
    xq, sx, wq, sw, bias, inv = _case(M, N, K, 44 + M)
    q, s = _run(sq, xq, sx, wq, sw, bias, True, inv)
    y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    sq.sq_w8a8_linear(dev(xq), dev(sx), dev(wq), dev(sw), y, dev(bias), workspace=sq.new_workspace(M, N, K))
    q2 = torch.empty_like(q)
    s2 = torch.empty_like(s)
    sq.sq_ln_quant_act(torch.relu(y), q2, s2, inv_s=dev(inv))
    assert torch.equal(q, q2) and torch.equal(s, s2)


def test_producer_dynamic_rejects_bad_arguments(sq):
    xq, sx, wq, sw, bias, inv = _case(8, 24, 16, 1)  # N = 24: not a multiple of 16
    q = torch.empty((8, 24), dtype=torch.int8, device="cuda")
    s = torch.empty(8, dtype=torch.float32, device="cuda")
    with pytest.raises(sq.SQError) as e:
        sq.sq_w8a8_linear_quant_dyn(dev(xq), dev(sx), dev(wq), dev(sw), q, s)
    assert e.value.status == 3
    xq, sx, wq, sw, bias, inv = _case(8, 32, 16, 1)
    q = torch.empty((8, 32), dtype=torch.int8, device="cuda")
    small = torch.zeros(64, dtype=torch.uint8, device="cuda")
    with pytest.raises(sq.SQError) as e:
        sq.sq_w8a8_linear_quant_dyn(dev(xq), dev(sx), dev(wq), dev(sw), q, s, workspace=small)
    assert e.value.status == 5
