"""The tensor-parallel layers' compute steps on the CPU through the oracle, so
the layers' host logic (sharding, the collectives, reassembly) runs on gloo
ranks without a GPU.  Same interface as the product's LibsqOps; tensors are
CPU torch tensors.  Test infrastructure only."""
import numpy as np
import torch

import oracle


def _np(t):
    return None if t is None else t.detach().cpu().numpy()


def _t(a):
    return torch.from_numpy(np.ascontiguousarray(a))


class OracleOps:
    def col_absmax(self, x, gamma=None, beta=None, eps: float = 1e-5):
        return _t(oracle.calibrate_absmax(_np(x), gamma=_np(gamma), beta=_np(beta), eps=eps))

    def smooth(self, amax_x, amax_w, alpha, gamma=None, beta=None):
        s, inv_s = oracle.smooth(_np(amax_x), _np(amax_w), alpha)
        gf, bf = oracle.fold_ln(_np(gamma), _np(beta), inv_s) if gamma is not None else (None, None)
        return _t(s), _t(inv_s), None if gf is None else _t(gf), None if bf is None else _t(bf)

    def quantize_weight(self, w, s):
        wq, sw = oracle.quantize_weight(oracle.fold_weight(_np(w), _np(s)))
        return _t(wq), _t(sw)

    def quant_act(self, h, gamma=None, beta=None, inv_s=None, eps: float = 1e-5):
        xq, sx = oracle.ln_quant_act(_np(h), _np(gamma), _np(beta), _np(inv_s), eps)
        return _t(xq), _t(sx)

    @staticmethod
    def _rows(x, inv_s, s_fold):
        if s_fold is not None:
            return oracle.fold_weight(_np(x), _np(s_fold)).astype(np.float32)
        return oracle.act_rows(_np(x), inv_s=_np(inv_s))

    def row_ranges(self, x, inv_s=None, s_fold=None):
        return _t(np.abs(self._rows(x, inv_s, s_fold)).max(axis=1).astype(np.float32))

    def quantize_rows_ranged(self, x, ranges, inv_s=None, s_fold=None):
        rows = self._rows(x, inv_s, s_fold)
        r = _np(ranges)
        sc = (r / np.float32(127)).astype(np.float32)
        q = np.stack([oracle.quantize_with_scale(rows[i], sc[i]) for i in range(rows.shape[0])])
        return _t(q), _t(sc)

    def linear(self, xq, sx, wq, sw, bias=None):
        return _t(oracle.w8a8_linear(_np(xq), _np(sx), _np(wq), _np(sw), _np(bias)))

    def gemm_s32(self, xq, wq):
        return _t(oracle.int_gemm(_np(xq), _np(wq)))

    def dequant(self, acc, sx, sw, bias=None):
        return _t(oracle.dequant(_np(acc), _np(sx), _np(sw), _np(bias)))
