"""Tensor-parallel SmoothQuant W8A8 linear layers over torch.distributed.

The explainer runs the quantized models sharded over several GPUs (sections
"how far speed and memory improved": OPT-175B on 4 GPUs instead of 8, and
"does it hold for a 530B model": 8 INT8 GPUs instead of 16 FP16).  Two
shardings of one linear, both bit-identical to the unsharded layer:

* ``ColumnParallelSmoothQuantLinear`` -- every rank holds a slice of the output
  channels (rows of W).  The smoothing factor of input channel j needs
  b_j = max_n |W[n, j]| over ALL output channels, so the ranks max-reduce
  their column ranges once at calibration; per-output-channel weight scales
  and per-token activation quantization are then local.  The forward needs no
  collective (``forward_gather`` all-gathers the output when the consumer
  needs all channels).
* ``RowParallelSmoothQuantLinear`` -- every rank holds a slice of the input
  channels (columns of W and of the activation, e.g. the output of a
  column-parallel layer).  A weight row's scale and a token's scale span all
  input channels, so the ranks max-reduce per-row ranges (once per weight, and
  M floats per forward), quantize their slice with the global ranges, and
  sum-reduce the int32 partial accumulators (exact: integer addition is
  associative) before one dequantization.

Compute goes through an ``ops`` object (``LibsqOps``: libsq kernels on the
current stream) and collectives through a ``comm`` object (``DistComm``:
torch.distributed, NCCL on GPUs), so the host logic can also run on CPU.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import (MAX_K, sq_calibrate_absmax, sq_dequant, sq_ln_quant_act, sq_quantize_rows_ranged,
               sq_quantize_weight, sq_row_ranges, sq_smooth_fold, sq_w8a8_gemm_s32, sq_w8a8_linear,
               sq_w8a8_workspace_bytes)

__all__ = ["LibsqOps", "DistComm", "ColumnParallelSmoothQuantLinear", "RowParallelSmoothQuantLinear"]


class LibsqOps:
    """The layer's steps as libsq kernels on CUDA tensors (current stream)."""

    def col_absmax(self, x: torch.Tensor, gamma=None, beta=None, eps: float = 1e-5) -> torch.Tensor:
        amax = torch.zeros(x.shape[1], dtype=torch.float32, device=x.device)
        sq_calibrate_absmax(x, amax, gamma, beta, eps)
        return amax

    def smooth(self, amax_x, amax_w, alpha: float, gamma=None, beta=None):
        s = torch.empty_like(amax_x)
        inv_s = torch.empty_like(amax_x)
        gf = torch.empty_like(amax_x) if gamma is not None else None
        bf = torch.empty_like(amax_x) if beta is not None else None
        sq_smooth_fold(amax_x, amax_w, alpha, s, inv_s, gamma, beta, gf, bf)
        return s, inv_s, gf, bf

    def quantize_weight(self, w, s):
        wq = torch.empty(w.shape, dtype=torch.int8, device=w.device)
        sw = torch.empty(w.shape[0], dtype=torch.float32, device=w.device)
        sq_quantize_weight(w, wq, sw, s=s)
        return wq, sw

    def quant_act(self, h, gamma=None, beta=None, inv_s=None, eps: float = 1e-5):
        xq = torch.empty(h.shape, dtype=torch.int8, device=h.device)
        sx = torch.empty(h.shape[0], dtype=torch.float32, device=h.device)
        sq_ln_quant_act(h, xq, sx, gamma, beta, inv_s, eps)
        return xq, sx

    def row_ranges(self, x, inv_s=None, s_fold=None):
        r = torch.empty(x.shape[0], dtype=torch.float32, device=x.device)
        sq_row_ranges(x, r, inv_s=inv_s, s_fold=s_fold)
        return r

    def quantize_rows_ranged(self, x, ranges, inv_s=None, s_fold=None):
        q = torch.empty(x.shape, dtype=torch.int8, device=x.device)
        sc = torch.empty(x.shape[0], dtype=torch.float32, device=x.device)
        sq_quantize_rows_ranged(x, ranges, q, sc, inv_s=inv_s, s_fold=s_fold)
        return q, sc

    def linear(self, xq, sx, wq, sw, bias=None):
        M, N = xq.shape[0], wq.shape[0]
        y = torch.empty((M, N), dtype=torch.float16, device=xq.device)
        need = sq_w8a8_workspace_bytes(M, N, xq.shape[1])
        ws = torch.zeros(need, dtype=torch.uint8, device=xq.device) if need else None
        sq_w8a8_linear(xq, sx, wq, sw, y, bias, ws)
        return y

    def gemm_s32(self, xq, wq):
        M, N = xq.shape[0], wq.shape[0]
        acc = torch.empty((M, N), dtype=torch.int32, device=xq.device)
        need = sq_w8a8_workspace_bytes(M, N, xq.shape[1])
        ws = torch.zeros(need, dtype=torch.uint8, device=xq.device) if need else None
        sq_w8a8_gemm_s32(xq, wq, acc, ws)
        return acc

    def dequant(self, acc, sx, sw, bias=None):
        y = torch.empty(acc.shape, dtype=torch.float16, device=acc.device)
        sq_dequant(acc, sx, sw, y, bias)
        return y


class DistComm:
    """Collectives of one process group (torch.distributed)."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist, self.group = dist, group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)

    def max_(self, t: torch.Tensor) -> torch.Tensor:
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX, group=self.group)
        return t

    def sum_(self, t: torch.Tensor) -> torch.Tensor:
        self.dist.all_reduce(t, op=self.dist.ReduceOp.SUM, group=self.group)
        return t

    def gather_cols(self, t: torch.Tensor) -> torch.Tensor:
        parts = [torch.empty_like(t) for _ in range(self.world)]
        self.dist.all_gather(parts, t.contiguous(), group=self.group)
        return torch.cat(parts, dim=1)


def shard_range(n: int, rank: int, world: int):
    """[lo, hi) of rank's contiguous share of n (multiples of 16 except the last)."""
    per = ((n + world - 1) // world + 15) // 16 * 16
    lo = min(n, rank * per)
    return lo, min(n, lo + per)


class ColumnParallelSmoothQuantLinear:
    """This rank's output channels of a SmoothQuant W8A8 linear."""

    def __init__(self, wq, sw, bias, gamma_f, beta_f, inv_s, eps, ops, comm):
        self.wq, self.sw, self.bias = wq, sw, bias
        self.gamma_f, self.beta_f, self.inv_s, self.eps = gamma_f, beta_f, inv_s, eps
        self.ops, self.comm = ops, comm

    @classmethod
    def from_float(cls, w_shard, calib, alpha: float = 0.5, gamma=None, beta=None, bias_shard=None,
                   eps: float = 1e-5, ops=None, comm=None):
        """w_shard: fp16 [N_rank, K], this rank's output channels; calib: the
        layer's full calibration input [T, K] (the LayerNorm input with gamma)."""
        ops = ops or LibsqOps()
        comm = comm or DistComm()
        amax_x = comm.max_(ops.col_absmax(calib, gamma, beta, eps))  # the same on every rank
        amax_w = comm.max_(ops.col_absmax(w_shard))                  # b_j over ALL output channels
        s, inv_s, gf, bf = ops.smooth(amax_x, amax_w, alpha, gamma, beta)
        wq, sw = ops.quantize_weight(w_shard, s)
        return cls(wq, sw, bias_shard, gf, bf, None if gamma is not None else inv_s, eps, ops, comm)

    def forward(self, h):
        """h [M, K] (replicated) -> this rank's output columns [M, N_rank]."""
        xq, sx = self.ops.quant_act(h, self.gamma_f, self.beta_f, self.inv_s, self.eps)
        return self.ops.linear(xq, sx, self.wq, self.sw, self.bias)

    def forward_gather(self, h):
        """All output channels [M, N] on every rank."""
        return self.comm.gather_cols(self.forward(h))

    __call__ = forward


class RowParallelSmoothQuantLinear:
    """This rank's input channels of a SmoothQuant W8A8 linear (no LayerNorm
    in front: its input is a sharded activation, smoothed by multiplying by
    1/s at run time)."""

    def __init__(self, wq, sw, bias, inv_s, ops, comm):
        self.wq, self.sw, self.bias, self.inv_s = wq, sw, bias, inv_s
        self.ops, self.comm = ops, comm

    @classmethod
    def from_float(cls, w_shard, calib_shard, alpha: float = 0.5, bias=None, ops=None, comm=None):
        """w_shard: fp16 [N, K_rank] (all output channels, this rank's input
        channels); calib_shard: [T, K_rank], this rank's slice of the layer's
        calibration input; bias [N] is added once, after the reduction.  The
        layer's whole K (the sum of K_rank over ranks) must be at most MAX_K,
        the bound under which the all-reduced int32 sums of 127 x 127 products
        cannot overflow: one integer all-reduce of the slice widths checks it
        on every rank (ValueError) before anything is computed."""
        ops = ops or LibsqOps()
        comm = comm or DistComm()
        k_total = comm.sum_(torch.tensor([w_shard.shape[1]], dtype=torch.int64, device=w_shard.device))
        if int(k_total.item()) > MAX_K:
            raise ValueError(f"row-parallel K = {int(k_total.item())} over all ranks exceeds {MAX_K}: the "
                             "all-reduced int32 accumulators could overflow")
        amax_x = ops.col_absmax(calib_shard)  # channel j lives on one rank only
        amax_w = ops.col_absmax(w_shard)
        s, inv_s, _, _ = ops.smooth(amax_x, amax_w, alpha)
        w_ranges = comm.max_(ops.row_ranges(w_shard, s_fold=s))  # each output channel over all of K
        wq, sw = ops.quantize_rows_ranged(w_shard, w_ranges, s_fold=s)
        return cls(wq, sw, bias, inv_s, ops, comm)

    def forward(self, h_shard):
        """h_shard [M, K_rank] -> the full output [M, N] on every rank."""
        ranges = self.comm.max_(self.ops.row_ranges(h_shard, inv_s=self.inv_s))  # M floats
        xq, sx = self.ops.quantize_rows_ranged(h_shard, ranges, inv_s=self.inv_s)
        acc = self.comm.sum_(self.ops.gemm_s32(xq, self.wq))  # exact int32 partial sums
        return self.ops.dequant(acc, sx, self.sw, self.bias)

    __call__ = forward
