"""The tensor-parallel building blocks on the GPU: per-row ranges, quantization
with given ranges and the standalone dequantization against the oracle, bit
for bit; and the column-/row-parallel layers on two ranks emulated as two
threads on one GPU (collectives are in-process reductions; no kernel waits
for another) against the unsharded layer, bit for bit."""
import threading

import numpy as np
import pytest
import torch

import oracle
import sq_inputs
from gpu_util import bits_equal, dev, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sq(cuda_device):
    import w8a8_int8_linear_channel_b200 as m
    return m


@pytest.mark.parametrize("rows,K,mode", [(1, 16, "act"), (37, 256, "act_inv"), (19, 4096, "fold"),
                                         (9, 20480, "act_inv"), (5, 49152, "fold"), (3, 1040, "fold")])
def test_row_ranges_and_ranged_quantization(sq, rows, K, mode):
    rng = np.random.default_rng(rows * 13 + K)
    x = (rng.standard_normal((rows, K)) * 2).astype(np.float16)
    vec = rng.uniform(0.05, 3.0, K).astype(np.float32)
    inv = vec if mode == "act_inv" else None
    s_fold = vec if mode == "fold" else None
    xr = oracle.fold_weight(x, s_fold).astype(np.float32) if s_fold is not None else oracle.act_rows(x, inv_s=inv)
    r = torch.empty(rows, dtype=torch.float32, device="cuda")
    sq.sq_row_ranges(dev(x), r, inv_s=dev(inv), s_fold=dev(s_fold))
    assert bits_equal(host(r), np.abs(xr).max(1).astype(np.float32))
    # quantize with wider ranges (as after a max over shards): some rows use another shard's max
    given = (np.abs(xr).max(1) * rng.choice([1.0, 1.5], rows)).astype(np.float32)
    q = torch.empty((rows, K), dtype=torch.int8, device="cuda")
    sc = torch.empty(rows, dtype=torch.float32, device="cuda")
    sq.sq_quantize_rows_ranged(dev(x), dev(given), q, sc, inv_s=dev(inv), s_fold=dev(s_fold))
    sc_ref = (given / np.float32(127)).astype(np.float32)
    q_ref = np.stack([oracle.quantize_with_scale(xr[i], sc_ref[i]) for i in range(rows)])
    assert bits_equal(host(sc), sc_ref) and bits_equal(host(q), q_ref)


@pytest.mark.parametrize("M,N", [(1, 4), (33, 260), (300, 4096)])
@pytest.mark.parametrize("with_bias", [False, True])
def test_dequant(sq, M, N, with_bias):
    rng = np.random.default_rng(M + N + with_bias)
    acc = rng.integers(-2 ** 28, 2 ** 28, (M, N)).astype(np.int32)
    sx = rng.uniform(1e-5, 1e-3, M).astype(np.float32)
    sw = rng.uniform(1e-5, 1e-3, N).astype(np.float32)
    bias = (rng.standard_normal(N)).astype(np.float16) if with_bias else None
    y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    sq.sq_dequant(dev(acc), dev(sx), dev(sw), y, dev(bias))
    assert bits_equal(host(y), oracle.dequant(acc, sx, sw, bias))


class ThreadComm:
    """Collectives among `world` threads of one process on one GPU: every
    thread deposits its tensor, one reduction in torch, results copied back."""

    def __init__(self, world, shared, rank):
        self.world, self.rank, self.sh = world, rank, shared

    def _exchange(self, t, reduce):
        sh = self.sh
        sh["slots"][self.rank] = t
        sh["bar"].wait()
        if self.rank == 0:
            sh["result"] = reduce(sh["slots"])
        sh["bar"].wait()
        res = sh["result"]
        sh["bar"].wait()
        return res

    def max_(self, t):
        t.copy_(self._exchange(t, lambda ts: torch.stack(ts).amax(0)))
        return t

    def sum_(self, t):
        t.copy_(self._exchange(t, lambda ts: torch.stack(ts).sum(0, dtype=t.dtype)))
        return t

    def gather_cols(self, t):
        return self._exchange(t.contiguous(), lambda ts: torch.cat(ts, dim=1)).clone()


def _run_ranks(world, fn):
    shared = {"slots": [None] * world, "bar": threading.Barrier(world), "result": None}
    out, errs = [None] * world, []

    def body(r):
        try:
            out[r] = fn(r, ThreadComm(world, shared, r))
        except BaseException as e:  # noqa: BLE001 -- reported below
            errs.append(e)
            shared["bar"].abort()

    th = [threading.Thread(target=body, args=(r,)) for r in range(world)]
    for t in th:
        t.start()
    for t in th:
        t.join(timeout=300)
    if errs:
        raise errs[0]
    return out


@pytest.mark.parametrize("world", [2, 4])
def test_tensor_parallel_layers_equal_unsharded(sq, world):
    from w8a8_int8_linear_channel_b200.tp import (ColumnParallelSmoothQuantLinear, LibsqOps,
                                                  RowParallelSmoothQuantLinear, shard_range)
    wl = sq_inputs.WORKLOADS["tiny_ln"]
    w, calib, h = sq_inputs.weight(wl), sq_inputs.calib_rows(wl), sq_inputs.run_rows(wl, 0, wl.M)
    g, b = sq_inputs.gamma(wl), sq_inputs.beta(wl)
    bias = (np.arange(wl.N) % 7 - 3).astype(np.float16) * np.float16(0.25)
    full = sq.SmoothQuantLinear.from_float(dev(w), dev(calib), wl.alpha, dev(g), dev(b), dev(bias))
    y_full = host(full(dev(h)))

    def col_rank(r, comm):
        lo, hi = shard_range(wl.N, r, world)
        layer = ColumnParallelSmoothQuantLinear.from_float(dev(w[lo:hi]), dev(calib), wl.alpha, dev(g), dev(b),
                                                           dev(bias[lo:hi]), ops=LibsqOps(), comm=comm)
        return host(layer.forward_gather(dev(h)))

    for y in _run_ranks(world, col_rank):
        assert bits_equal(y, y_full)

    wl2 = sq_inputs.WORKLOADS["tiny"]
    w2, calib2 = sq_inputs.weight(wl2), sq_inputs.calib_rows(wl2)
    h2 = sq_inputs.run_rows(wl2, 0, 48)  # 48 tokens: the stream-K path is not used for M > 32
    full2 = sq.SmoothQuantLinear.from_float(dev(w2), dev(calib2), wl2.alpha, bias=dev(bias))
    y_full2 = host(full2(dev(h2)))

    def row_rank(r, comm):
        lo, hi = shard_range(wl2.K, r, world)
        layer = RowParallelSmoothQuantLinear.from_float(dev(w2[:, lo:hi]), dev(calib2[:, lo:hi]), wl2.alpha,
                                                        dev(bias), ops=LibsqOps(), comm=comm)
        return host(layer.forward(dev(h2[:, lo:hi])))

    for y in _run_ranks(world, row_rank):
        assert bits_equal(y, y_full2)
    assert sq.sq_poll_status() == 0
