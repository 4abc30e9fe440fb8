"""The context-parallel exchange's arithmetic on CPU float64 tensors, from the
fp64 oracle (the operator's passes) and plain torch (decays, folds and row
copies written out from their definitions).  Test infrastructure only: it
lets the exchange logic of the split operator run on CPU ranks (gloo)."""
import numpy as np
import torch

import oracle


def _np(t):
    return None if t is None else t.detach().to(torch.float64).numpy()


def _t(a):
    return None if a is None else torch.from_numpy(np.ascontiguousarray(a))


class OracleOps:
    def segment_decay(self, g):
        return torch.exp(g.sum(dim=2))

    def fold(self, E_all, X_all, r, direction, init):
        h = torch.zeros_like(X_all[0]) if init is None else init.clone()
        qs = range(0, r) if direction == 0 else range(X_all.shape[0] - 1, r, -1)
        for q in qs:
            h = E_all[q][..., None] * h + X_all[q]
        return h

    def rows(self, dst, dst_off, n, A=None, a_off=0, a_scale=1.0, B=None, b_off=0):
        val = torch.zeros_like(dst[:, :, dst_off:dst_off + n])
        if A is not None:
            val = val + a_scale * A[:, :, a_off:a_off + n]
        if B is not None:
            val = val + B[:, :, b_off:b_off + n]
        dst[:, :, dst_off:dst_off + n] = val
        return dst

    def gla_fwd(self, q, k, v, g, h0):
        o, hT = oracle.gla_fwd(_np(q), _np(k), _np(v), _np(g), _np(h0))
        return _t(o), _t(hT)

    def gla_bwd(self, q, k, v, g, dO, h0, dhT):
        r = oracle.gla_bwd(_np(q), _np(k), _np(v), _np(g), _np(dO), _np(h0), _np(dhT))
        return {k_: _t(x) for k_, x in r.items()}

    def swa_fwd(self, q, k, v, meta_k, meta_v, w, scale):
        o, lse = oracle.swa_meta_fwd(_np(q), _np(k), _np(v), _np(meta_k), _np(meta_v), w, scale)
        return _t(o), _t(lse)

    def swa_bwd(self, q, k, v, meta_k, meta_v, lse, dO, w, scale, o):
        r = oracle.swa_meta_bwd(_np(q), _np(k), _np(v), _np(meta_k), _np(meta_v), _np(dO), w,
                                scale)
        return {k_: _t(x) for k_, x in r.items()}
