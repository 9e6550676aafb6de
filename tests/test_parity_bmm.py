"""INT8 BMM on the GPU against the oracle, bit for bit: independent batch
items (attention heads) with per-row and per-column scales, ragged M / N / K
(rows past one item's end must never read the next item), an output row
stride that rules out TMA stores, per-head and per-token scales, and the
OPT-6.7B attention shapes (32 heads, 2048 tokens, head dim 128) with two heads
checked in full."""
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


def _case(B, M, N, K, seed, per_head=False):
    rng = np.random.default_rng(seed)
    a = rng.integers(-127, 128, (B, M, K)).astype(np.int8)
    b = rng.integers(-127, 128, (B, N, K)).astype(np.int8)
    if per_head:
        sa = np.repeat(rng.uniform(1e-3, 1e-2, (B, 1)), M, 1).astype(np.float32)
        sb = np.repeat(rng.uniform(1e-3, 1e-2, (B, 1)), N, 1).astype(np.float32)
    else:
        sa = rng.uniform(1e-3, 1e-2, (B, M)).astype(np.float32)
        sb = rng.uniform(1e-3, 1e-2, (B, N)).astype(np.float32)
    return a, sa, b, sb


@pytest.mark.parametrize("B,M,N,K", [(1, 1, 16, 16), (3, 37, 40, 48), (3, 37, 36, 48), (4, 300, 272, 144),
                                     (2, 256, 256, 256), (5, 129, 513, 1040), (32, 64, 64, 128),
                                     # 128-channel tiles (N <= 128) with two K boxes per stage:
                                     # ragged N and M, a last stage whose second box lies past K,
                                     # N % 8 != 0 (row stores), and N = 128 exactly
                                     (3, 300, 72, 1040), (2, 200, 100, 528), (2, 130, 128, 640)])
@pytest.mark.parametrize("per_head", [False, True])
def test_bmm(sq, B, M, N, K, per_head):
    a, sa, b, sb = _case(B, M, N, K, B * 7 + M + N + K + per_head, per_head)
    y = torch.empty((B, M, N), dtype=torch.float16, device="cuda")
    sq.sq_w8a8_bmm(dev(a), dev(sa), dev(b), dev(sb), y)
    assert sq.sq_poll_status() == 0
    assert bits_equal(host(y), oracle.w8a8_bmm(a, sa, b, sb))


@pytest.mark.parametrize("which", ["qk", "pv"])
def test_bmm_attention_shapes(sq, which):
    """OPT-6.7B attention, 2048 tokens: Q K^T is 32 x [2048 x 128] x [2048 x 128]^T,
    P V is 32 x [2048 x 2048] x [128 x 2048]^T (V stored transposed)."""
    B, M, N, K = (32, 2048, 2048, 128) if which == "qk" else (32, 2048, 128, 2048)
    a, sa, b, sb = _case(B, M, N, K, 1234 + (which == "pv"), per_head=True)
    y = torch.empty((B, M, N), dtype=torch.float16, device="cuda")
    sq.sq_w8a8_bmm(dev(a), dev(sa), dev(b), dev(sb), y)
    got = host(y)
    for i in (0, B - 1):
        assert bits_equal(got[i:i + 1], oracle.w8a8_bmm(a[i:i + 1], sa[i:i + 1], b[i:i + 1], sb[i:i + 1]))


@pytest.mark.parametrize("K", [256, 272])
def test_extreme_codes_short_k(sq, K):
    """All +-127 codes at short K (|acc| = K * 127^2, 4 129 024 at K = 256,
    4 386 688 at K = 272: either side of 2^22), through the BMM and the
    linear on the CTA-pair kernel."""
    B, M, N = 2, 300, 264
    a = np.full((B, M, K), 127, np.int8)
    a[:, 1::2] = -127
    b = np.full((B, N, K), 127, np.int8)
    b[:, 3::5] = -127
    rng = np.random.default_rng(K)
    sa = rng.uniform(1e-6, 1e-5, (B, M)).astype(np.float32)
    sb = rng.uniform(1e-6, 1e-5, (B, N)).astype(np.float32)
    y = torch.empty((B, M, N), dtype=torch.float16, device="cuda")
    sq.sq_w8a8_bmm(dev(a), dev(sa), dev(b), dev(sb), y)
    assert bits_equal(host(y), oracle.w8a8_bmm(a, sa, b, sb))
    # the same through the linear (CTA-pair kernel, M > 128)
    y2 = torch.empty((M, N), dtype=torch.float16, device="cuda")
    sq.sq_w8a8_linear(dev(a[0]), dev(sa[0]), dev(b[0]), dev(sb[0]), y2)
    assert bits_equal(host(y2), oracle.w8a8_linear(a[0], sa[0], b[0], sb[0]))
