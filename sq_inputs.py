"""Seeded synthetic inputs for the SmoothQuant W8A8 linear workloads.

This module only draws random numbers; it holds none of the method's
arithmetic (no absmax, no smoothing, no quantization).  Both the CUDA path
(tests, bench) and the CPU oracle take their inputs from here.

The pages measure on OPT / BLOOM / GLM checkpoints and zero-shot suites, none
of which is available; these synthetic tensors with the same shapes and the
persistent per-channel activation outliers the SmoothQuant explainer
describes ("basic idea": outliers stay in the same channels across tokens)
stand in for them.

Every tensor comes from its own PCG64 stream keyed by (seed, tag[, block]),
so any block of rows can be regenerated without drawing the whole tensor.
Normal draws are float32 and rounded to fp16 once.
"""
from __future__ import annotations

import dataclasses
from typing import Optional, Sequence

import numpy as np

ROW_BLOCK = 256  # rows drawn per independent stream for activations/weights

_TAGS = {"h_cal": 1, "h_run": 2, "w": 3, "gamma": 4, "beta": 5, "bias": 6, "outliers": 7,
         "outlier_gain": 8}


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    K: int
    N: int
    M: int
    calib: int
    alpha: float
    n_outliers: int
    outlier_lo: float
    outlier_hi: float
    w_std: float
    ln: bool            # outliers enter through a LayerNorm gamma (True) or directly on X
    bias: bool
    fixed_outliers: Optional[Sequence[int]] = None
    beta_std: float = 0.01
    bias_std: float = 0.01
    seed: int = 0

    @property
    def gemm_ops(self) -> int:
        return 2 * self.M * self.N * self.K


# OPT-shaped workloads.  Outlier counts: 0.1% of 4096 -> 4, 0.1% of 12288 -> 12,
# 0.05% of 49152 -> 25 (round to nearest).
WORKLOADS = {
    "tiny": Workload("tiny", K=256, N=256, M=16, calib=128, alpha=0.5, n_outliers=2,
                     outlier_lo=60.0, outlier_hi=60.0, w_std=0.02, ln=False, bias=False,
                     fixed_outliers=(3, 77)),
    "tiny_ln": Workload("tiny_ln", K=256, N=256, M=16, calib=128, alpha=0.5, n_outliers=2,
                        outlier_lo=60.0, outlier_hi=60.0, w_std=0.02, ln=True, bias=False,
                        fixed_outliers=(3, 77), beta_std=0.0),
    "attn": Workload("attn", K=4096, N=4096, M=2048, calib=512, alpha=0.5, n_outliers=6,
                     outlier_lo=40.0, outlier_hi=100.0, w_std=0.02, ln=True, bias=False),
    "ffn_up": Workload("ffn_up", K=4096, N=16384, M=4096, calib=512, alpha=0.5, n_outliers=4,
                       outlier_lo=50.0, outlier_hi=50.0, w_std=0.02, ln=True, bias=True),
    "decode": Workload("decode", K=12288, N=49152, M=32, calib=512, alpha=0.5, n_outliers=12,
                       outlier_lo=80.0, outlier_hi=80.0, w_std=0.006, ln=True, bias=False),
    "ffn_down": Workload("ffn_down", K=49152, N=12288, M=8192, calib=1024, alpha=0.5,
                         n_outliers=25, outlier_lo=100.0, outlier_hi=100.0, w_std=0.006,
                         ln=False, bias=False),
}

DECODE_M = (1, 4, 8, 16, 32)
FFN_DOWN_ALPHAS = (0.0, 0.25, 0.5, 0.75, 0.85, 1.0)


def _rng(seed: int, tag: str, block: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64([seed, _TAGS[tag], block]))


def outlier_channels(wl: Workload) -> np.ndarray:
    if wl.fixed_outliers is not None:
        return np.asarray(wl.fixed_outliers, np.int64)
    rng = _rng(wl.seed, "outliers")
    return np.sort(rng.choice(wl.K, size=wl.n_outliers, replace=False)).astype(np.int64)


def outlier_gains(wl: Workload) -> np.ndarray:
    if wl.outlier_lo == wl.outlier_hi:
        return np.full(len(outlier_channels(wl)), wl.outlier_lo, np.float32)
    rng = _rng(wl.seed, "outlier_gain")
    return rng.uniform(wl.outlier_lo, wl.outlier_hi, size=len(outlier_channels(wl))).astype(np.float32)


def _normal_rows(seed: int, tag: str, K: int, row0: int, rows: int, std: float) -> np.ndarray:
    """Rows [row0, row0+rows) of an fp16 matrix whose ROW_BLOCK-row blocks are independent streams.
    Blocks are drawn on a thread pool when there are many of them (each block is its own stream,
    so the values do not depend on the number of threads)."""
    out = np.empty((rows, K), np.float16)
    spans = []
    r = row0
    while r < row0 + rows:
        blk = r // ROW_BLOCK
        b0 = blk * ROW_BLOCK
        take = min(b0 + ROW_BLOCK, row0 + rows) - r
        spans.append((blk, r - b0, r - row0, take))
        r += take

    def fill(span):
        blk, src, dst, take = span
        g = _rng(seed, tag, blk).standard_normal((ROW_BLOCK, K), dtype=np.float32)
        if std != 1.0:
            g *= np.float32(std)
        out[dst:dst + take] = g[src:src + take].astype(np.float16)

    if len(spans) < 2 or rows * K < (1 << 22):
        for sp in spans:
            fill(sp)
    else:
        import os
        from concurrent.futures import ThreadPoolExecutor
        with ThreadPoolExecutor(max(1, min(len(spans), os.cpu_count() or 1, 32))) as ex:
            list(ex.map(fill, spans))
    return out


def gamma(wl: Workload) -> Optional[np.ndarray]:
    """LayerNorm gamma: 1 except the outlier channels (LN workloads only)."""
    if not wl.ln:
        return None
    g = np.ones(wl.K, np.float32)
    g[outlier_channels(wl)] = outlier_gains(wl)
    return g


def beta(wl: Workload) -> Optional[np.ndarray]:
    if not wl.ln:
        return None
    if wl.beta_std == 0.0:
        return np.zeros(wl.K, np.float32)
    return (_rng(wl.seed, "beta").standard_normal(wl.K, dtype=np.float32) * np.float32(wl.beta_std))


def bias(wl: Workload) -> Optional[np.ndarray]:
    if not wl.bias:
        return None
    b = _rng(wl.seed, "bias").standard_normal(wl.N, dtype=np.float32) * np.float32(wl.bias_std)
    return b.astype(np.float16)


def _activation_rows(wl: Workload, tag: str, row0: int, rows: int) -> np.ndarray:
    h = _normal_rows(wl.seed, tag, wl.K, row0, rows, 1.0)
    if not wl.ln:
        # Outliers directly on X (the input of a linear that follows an activation).
        ch = outlier_channels(wl)
        gains = outlier_gains(wl).astype(np.float32)
        h[:, ch] = (h[:, ch].astype(np.float32) * gains[None, :]).astype(np.float16)
    return h


def calib_rows(wl: Workload, row0: int = 0, rows: Optional[int] = None) -> np.ndarray:
    """Calibration tokens (the LayerNorm input h for LN workloads, X otherwise), fp16 [rows, K]."""
    rows = wl.calib - row0 if rows is None else rows
    return _activation_rows(wl, "h_cal", row0, rows)


def run_rows(wl: Workload, row0: int = 0, rows: Optional[int] = None) -> np.ndarray:
    """Runtime tokens, same distribution as the calibration tokens, fp16 [rows, K]."""
    rows = wl.M - row0 if rows is None else rows
    return _activation_rows(wl, "h_run", row0, rows)


def weight(wl: Workload, row0: int = 0, rows: Optional[int] = None) -> np.ndarray:
    """nn.Linear weight W [N, K] fp16 ~ N(0, w_std^2)."""
    rows = wl.N - row0 if rows is None else rows
    return _normal_rows(wl.seed, "w", wl.K, row0, rows, wl.w_std)


def with_(wl: Workload, **kw) -> Workload:
    return dataclasses.replace(wl, **kw)
