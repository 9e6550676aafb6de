"""Producer-side quantization on the GPU against the oracle, bit for bit: the
linear whose epilogue emits the next linear's INT8 input at a static scale
(optional ReLU, the next linear's 1/s), through the stream-K kernel (M <= 32)
and the CTA-pair kernel (larger M), ragged shapes, saturation, and a two-layer
chain (FFN up -> ReLU -> FFN down) against the unfused composition."""
import numpy as np
import pytest
import torch

import oracle
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
    sw = rng.uniform(1e-4, 2e-3, N).astype(np.float32)
    bias = (rng.standard_normal(N) * 0.5).astype(np.float16)
    inv = rng.uniform(0.05, 3.0, N).astype(np.float32)
    return xq, sx, wq, sw, bias, inv


@pytest.mark.parametrize("M,N,K", [(1, 16, 16), (5, 272, 48), (32, 1040, 4112), (33, 256, 256),
                                   (300, 1008, 2064), (513, 4096, 1024)])
@pytest.mark.parametrize("relu", [False, True])
@pytest.mark.parametrize("with_inv_s", [False, True])
def test_producer_quant(sq, M, N, K, relu, with_inv_s):
    xq, sx, wq, sw, bias, inv = _case(M, N, K, M * 31 + N + K + relu)
    inv = inv if with_inv_s else None
    y = oracle.w8a8_linear(xq, sx, wq, sw, bias).astype(np.float32)
    a = np.maximum(y, 0) if relu else y
    x = a * (inv[None, :] if inv is not None else 1)
    r = np.float32(np.abs(x[np.isfinite(x)]).max() * 0.6)  # part of the outputs saturate
    q = torch.empty((M, N), dtype=torch.int8, device="cuda")
    s = torch.empty(M, dtype=torch.float32, device="cuda")
    ws = sq.new_workspace(M, N, K)
    sq.sq_w8a8_linear_quant(dev(xq), dev(sx), dev(wq), dev(sw), dev(np.array([r], np.float32)), q, s,
                            bias=dev(bias), relu=relu, inv_s_next=dev(inv), workspace=ws)
    q_ref, s_ref = oracle.w8a8_linear_quant_static(xq, sx, wq, sw, bias, relu=relu, inv_s_next=inv,
                                                   range_next=r)
    assert sq.sq_poll_status() == 0
    assert bits_equal(host(s), s_ref)
    assert bits_equal(host(q), q_ref)


def test_ffn_chain_matches_unfused(sq):
    """FFN up (producer) -> ReLU -> FFN down: the fused codes equal the codes
    of the unfused path (linear to fp16, ReLU, static quantization with 1/s)."""
    rng = np.random.default_rng(77)
    M, K, N = 40, 512, 1024
    xq, sx, wq, sw, bias, inv = _case(M, N, K, 78)
    r = np.float32(3.0)
    q = torch.empty((M, N), dtype=torch.int8, device="cuda")
    s = torch.empty(M, dtype=torch.float32, device="cuda")
    sq.sq_w8a8_linear_quant(dev(xq), dev(sx), dev(wq), dev(sw), dev(np.array([r], np.float32)), q, s,
                            bias=dev(bias), relu=True, inv_s_next=dev(inv))
    # unfused on the GPU: linear -> fp16 y, ReLU in torch, static quantization
    y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    sq.sq_w8a8_linear(dev(xq), dev(sx), dev(wq), dev(sw), y, dev(bias))
    a = torch.relu(y)
    q2 = torch.empty_like(q)
    s2 = torch.empty_like(s)
    sq.sq_ln_quant_act_static(a, q2, s2, dev(np.array([r], np.float32)), inv_s=dev(inv))
    assert torch.equal(q, q2) and torch.equal(s, s2)
    # and the down projection consumes them directly
    w2 = rng.integers(-127, 128, (256, N)).astype(np.int8)
    sw2 = rng.uniform(1e-4, 1e-3, 256).astype(np.float32)
    out = torch.empty((M, 256), dtype=torch.float16, device="cuda")
    sq.sq_w8a8_linear(q, s, dev(w2), dev(sw2), out)
    assert bits_equal(host(out), oracle.w8a8_linear(host(q), host(s), w2, sw2))
