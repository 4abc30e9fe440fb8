"""fp64 CPU oracle for the Lizard hybrid attention operator.

TEST INFRASTRUCTURE ONLY.  The tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` are the only callers.  The CUDA library never
imports, links or calls anything in this directory, and this module imports
nothing from the CUDA library's package.

The arithmetic lives in ``lizard_oracle.cpp`` (plain loops in fp64, threaded
over (batch, head) pairs).  This module only builds it with g++, converts
numpy arrays to contiguous float64 and calls it through ctypes.

Definitions follow "Lizard: An Efficient Linearization Framework for Large
Language Models" (gist.science technical summary, section 2a): gated linear
attention S_t = diag(exp(g_t)) S_{t-1} + k_t v_t^T, o_t = q_t^T S_t; sliding
window softmax with meta-memory sinks; output o = o_gla + alpha * o_swa.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lizard_oracle.cpp")
_LIB = os.path.join(_HERE, "liblizard_oracle.so")
_lock = threading.Lock()
_lib = None

_D = ctypes.POINTER(ctypes.c_double)
_I64 = ctypes.POINTER(ctypes.c_int64)
_i = ctypes.c_int
_f = ctypes.c_double


def build(src: str = _SRC, out: str = _LIB, extra: tuple = ()) -> str:
    """Compile the oracle with g++ (no CUDA involved)."""
    cmd = ["g++", "-O2", "-std=c++17", "-shared", "-fPIC", "-pthread", *extra,
           "-o", out, src]
    subprocess.run(cmd, check=True)
    return out


def _needs_build() -> bool:
    return (not os.path.exists(_LIB)) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC)


def load(path: str | None = None):
    """Return the ctypes handle (building the default library if stale)."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    with _lock:
        if _lib is None:
            if _needs_build():
                build()
            _lib = _bind(ctypes.CDLL(_LIB))
    return _lib


def _bind(lib):
    lib.oracle_gla_fwd.argtypes = [_i] * 5 + [_D] * 7 + [_i]
    lib.oracle_gla_chunked_fwd.argtypes = [_i] * 6 + [_D] * 7 + [_i]
    lib.oracle_swa_meta_fwd.argtypes = [_i] * 7 + [_f] + [_D] * 7 + [_i]
    lib.oracle_hybrid_fwd.argtypes = [_i] * 7 + [_f, _f] + [_D] * 11 + [_i]
    lib.oracle_gla_bwd.argtypes = [_i] * 5 + [_D] * 12 + [_i]
    lib.oracle_swa_meta_bwd.argtypes = [_i] * 7 + [_f] + [_D] * 11 + [_i]
    lib.oracle_hybrid_bwd.argtypes = [_i] * 7 + [_f, _f] + [_D] * 17 + [_i]
    lib.oracle_decode_step.argtypes = ([_i] * 6 + [_f, _f] + [_D] * 3 + [_I64] +
                                       [_D] * 7 + [_i])
    lib.oracle_mse_loss.argtypes = [ctypes.c_int64] + [_D] * 4
    lib.oracle_gate_from_logits.argtypes = [ctypes.c_int64, _D, ctypes.c_double, _D]
    lib.oracle_dlogits.argtypes = [ctypes.c_int64, _D, ctypes.c_double, _D, _D]
    lib.oracle_qkg_projection.argtypes = [_i] * 5 + [_D] * 4 + [ctypes.c_double] + [_D] * 3
    for name in ("oracle_qkg_projection", "oracle_gate_from_logits", "oracle_dlogits", "oracle_mse_loss", "oracle_gla_fwd", "oracle_gla_chunked_fwd", "oracle_swa_meta_fwd",
                 "oracle_hybrid_fwd", "oracle_gla_bwd", "oracle_swa_meta_bwd",
                 "oracle_hybrid_bwd", "oracle_decode_step"):
        getattr(lib, name).restype = ctypes.c_int
    return lib


def _in(x):
    if x is None:
        return None, None
    a = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    return a, a.ctypes.data_as(_D)


def _out(shape):
    a = np.zeros(shape, dtype=np.float64)
    return a, a.ctypes.data_as(_D)


def _check(rc, name):
    if rc != 0:
        raise ValueError(f"{name}: invalid arguments (rc={rc})")


def _shape_qkv(q, v):
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    return B, H, T, dk, dv


def gla_fwd(q, k, v, g, h0=None, *, nthreads=0, lib=None):
    """Token-by-token gated recurrence.  Returns (o [B,H,T,dv], hT [B,H,dk,dv])."""
    lib = lib or load()
    (q, pq), (k, pk), (v, pv), (g, pg), (h0, ph) = map(_in, (q, k, v, g, h0))
    B, H, T, dk, dv = _shape_qkv(q, v)
    o, po = _out((B, H, T, dv))
    hT, phT = _out((B, H, dk, dv))
    _check(lib.oracle_gla_fwd(B, H, T, dk, dv, pq, pk, pv, pg, ph, po, phT, nthreads),
           "gla_fwd")
    return o, hT


def gla_chunked_fwd(q, k, v, g, chunk, h0=None, *, nthreads=0, lib=None):
    """Chunked rearrangement of the recurrence (identity test only)."""
    lib = lib or load()
    (q, pq), (k, pk), (v, pv), (g, pg), (h0, ph) = map(_in, (q, k, v, g, h0))
    B, H, T, dk, dv = _shape_qkv(q, v)
    o, po = _out((B, H, T, dv))
    hT, phT = _out((B, H, dk, dv))
    _check(lib.oracle_gla_chunked_fwd(B, H, T, dk, dv, int(chunk), pq, pk, pv, pg, ph,
                                      po, phT, nthreads), "gla_chunked_fwd")
    return o, hT


def swa_meta_fwd(q, k, v, meta_k, meta_v, w, scale, *, nthreads=0, lib=None):
    """Window + meta softmax.  meta_v=None is the sink-only mode.

    Returns (o_swa [B,H,T,dv], lse [B,H,T])."""
    lib = lib or load()
    (q, pq), (k, pk), (v, pv) = map(_in, (q, k, v))
    M = 0 if meta_k is None else int(np.asarray(meta_k).shape[1])
    (mk, pmk), (mv, pmv) = _in(meta_k), _in(meta_v)
    B, H, T, dk, dv = _shape_qkv(q, v)
    o, po = _out((B, H, T, dv))
    lse, pl = _out((B, H, T))
    _check(lib.oracle_swa_meta_fwd(B, H, T, dk, dv, int(w), M, float(scale), pq, pk, pv,
                                   pmk, pmv, po, pl, nthreads), "swa_meta_fwd")
    return o, lse


def hybrid_fwd(q, k, v, g, meta_k, meta_v, w, scale, alpha, h0=None, *, nthreads=0,
               lib=None):
    """o = o_gla + alpha * o_swa.  Returns dict(o, hT, lse, o_swa)."""
    lib = lib or load()
    (q, pq), (k, pk), (v, pv), (g, pg), (h0, ph) = map(_in, (q, k, v, g, h0))
    M = 0 if meta_k is None else int(np.asarray(meta_k).shape[1])
    (mk, pmk), (mv, pmv) = _in(meta_k), _in(meta_v)
    B, H, T, dk, dv = _shape_qkv(q, v)
    o, po = _out((B, H, T, dv))
    hT, phT = _out((B, H, dk, dv))
    lse, pl = _out((B, H, T))
    osw, pos_ = _out((B, H, T, dv))
    _check(lib.oracle_hybrid_fwd(B, H, T, dk, dv, int(w), M, float(scale), float(alpha),
                                 pq, pk, pv, pg, pmk, pmv, ph, po, phT, pl, pos_,
                                 nthreads), "hybrid_fwd")
    return {"o": o, "hT": hT, "lse": lse, "o_swa": osw}


def gla_bwd(q, k, v, g, dO, h0=None, dhT=None, *, nthreads=0, lib=None):
    """Hand-written gradient of the gated recurrence.

    Returns dict(dq, dk, dv, dg, dh0)."""
    lib = lib or load()
    (q, pq), (k, pk), (v, pv), (g, pg), (h0, ph), (dO, pdo), (dhT, pdh) = map(
        _in, (q, k, v, g, h0, dO, dhT))
    B, H, T, dk, dv = _shape_qkv(q, v)
    dq, pdq = _out((B, H, T, dk))
    dk_, pdk = _out((B, H, T, dk))
    dv_, pdv = _out((B, H, T, dv))
    dg, pdg = _out((B, H, T, dk))
    dh0, pdh0 = _out((B, H, dk, dv))
    _check(lib.oracle_gla_bwd(B, H, T, dk, dv, pq, pk, pv, pg, ph, pdo, pdh, pdq, pdk,
                              pdv, pdg, pdh0, nthreads), "gla_bwd")
    return {"dq": dq, "dk": dk_, "dv": dv_, "dg": dg, "dh0": dh0}


def swa_meta_bwd(q, k, v, meta_k, meta_v, dO, w, scale, *, nthreads=0, lib=None):
    """Gradient of the window + meta softmax; dO = dL/d(o_swa).

    Returns dict(dq, dk, dv, dmeta_k, dmeta_v) (dmeta_v None in sink-only mode)."""
    lib = lib or load()
    (q, pq), (k, pk), (v, pv), (dO, pdo) = map(_in, (q, k, v, dO))
    M = 0 if meta_k is None else int(np.asarray(meta_k).shape[1])
    (mk, pmk), (mv, pmv) = _in(meta_k), _in(meta_v)
    B, H, T, dk, dv = _shape_qkv(q, v)
    dq, pdq = _out((B, H, T, dk))
    dk_, pdk = _out((B, H, T, dk))
    dv_, pdv = _out((B, H, T, dv))
    dmk, pdmk = _out((H, M, dk))
    dmv, pdmv = _out((H, M, dv))
    _check(lib.oracle_swa_meta_bwd(B, H, T, dk, dv, int(w), M, float(scale), pq, pk, pv,
                                   pmk, pmv, pdo, pdq, pdk, pdv, pdmk, pdmv, nthreads),
           "swa_meta_bwd")
    return {"dq": dq, "dk": dk_, "dv": dv_, "dmeta_k": dmk,
            "dmeta_v": dmv if meta_v is not None else None}


def hybrid_bwd(q, k, v, g, meta_k, meta_v, dO, w, scale, alpha, h0=None, dhT=None, *,
               nthreads=0, lib=None):
    """Gradient of o = o_gla + alpha * o_swa.

    Returns dict(dq, dk, dv, dg, dh0, dmeta_k, dmeta_v, dalpha)."""
    lib = lib or load()
    (q, pq), (k, pk), (v, pv), (g, pg), (h0, ph), (dO, pdo), (dhT, pdh) = map(
        _in, (q, k, v, g, h0, dO, dhT))
    M = 0 if meta_k is None else int(np.asarray(meta_k).shape[1])
    (mk, pmk), (mv, pmv) = _in(meta_k), _in(meta_v)
    B, H, T, dk, dv = _shape_qkv(q, v)
    dq, pdq = _out((B, H, T, dk))
    dk_, pdk = _out((B, H, T, dk))
    dv_, pdv = _out((B, H, T, dv))
    dg, pdg = _out((B, H, T, dk))
    dh0, pdh0 = _out((B, H, dk, dv))
    dmk, pdmk = _out((H, M, dk))
    dmv, pdmv = _out((H, M, dv))
    da, pda = _out((1,))
    _check(lib.oracle_hybrid_bwd(B, H, T, dk, dv, int(w), M, float(scale), float(alpha),
                                 pq, pk, pv, pg, pmk, pmv, ph, pdo, pdh, pdq, pdk, pdv,
                                 pdg, pdh0, pdmk, pdmv, pda, nthreads), "hybrid_bwd")
    return {"dq": dq, "dk": dk_, "dv": dv_, "dg": dg, "dh0": dh0, "dmeta_k": dmk,
            "dmeta_v": dmv if meta_v is not None else None, "dalpha": float(da[0])}


def decode_step(state, kring, vring, pos, q, k, v, g, meta_k, meta_v, scale, alpha, *,
                nthreads=0, lib=None):
    """One generation step.  Returns dict(o, state, kring, vring, pos) (new arrays;
    the inputs are not modified)."""
    lib = lib or load()
    state = np.array(state, dtype=np.float64, order="C", copy=True)
    kring = np.array(kring, dtype=np.float64, order="C", copy=True)
    vring = np.array(vring, dtype=np.float64, order="C", copy=True)
    pos = np.array(pos, dtype=np.int64, order="C", copy=True)
    (q, pq), (k, pk), (v, pv), (g, pg) = map(_in, (q, k, v, g))
    M = 0 if meta_k is None else int(np.asarray(meta_k).shape[1])
    (mk, pmk), (mv, pmv) = _in(meta_k), _in(meta_v)
    Bd, H, dk = q.shape
    dv = v.shape[-1]
    w = kring.shape[2]
    o, po = _out((Bd, H, dv))
    _check(lib.oracle_decode_step(Bd, H, dk, dv, w, M, float(scale), float(alpha),
                                  state.ctypes.data_as(_D), kring.ctypes.data_as(_D),
                                  vring.ctypes.data_as(_D), pos.ctypes.data_as(_I64),
                                  pq, pk, pv, pg, pmk, pmv, po, nthreads), "decode_step")
    return {"o": o, "state": state, "kring": kring, "vring": vring, "pos": pos}


def mse_loss(o, target, *, lib=None):
    """Stage-1 distillation loss: mean over every element of (o - target)^2.

    Returns (loss, dO) with dO = dloss/do = 2 (o - target) / o.size."""
    lib = lib or load()
    (o, po), (t, pt) = _in(o), _in(target)
    if o.shape != t.shape:
        raise ValueError("mse_loss: o and target differ in shape")
    loss, pl = _out((1,))
    dO, pd = _out(o.shape)
    _check(lib.oracle_mse_loss(int(o.size), po, pt, pl, pd), "mse_loss")
    return float(loss[0]), dO


def gate_from_logits(z, scale=1.0, *, lib=None):
    """Log-gate g = scale * log sigma(z) from the gate logit z (same shape)."""
    lib = lib or load()
    z, pz = _in(z)
    g, pg = _out(z.shape)
    _check(lib.oracle_gate_from_logits(int(z.size), pz, float(scale), pg), "gate_from_logits")
    return g


def dlogits(z, dg, scale=1.0, *, lib=None):
    """dL/dz from dL/dg through g = scale * log sigma(z)."""
    lib = lib or load()
    (z, pz), (dg, pdg) = _in(z), _in(dg)
    if z.shape != dg.shape:
        raise ValueError("dlogits: z and dg differ in shape")
    dz, pdz = _out(z.shape)
    _check(lib.oracle_dlogits(int(z.size), pz, float(scale), pdg, pdz), "dlogits")
    return dz


def qkg_projection(x, Wq, Wk, Wg, H, dk, scale=1.0, *, lib=None):
    """q = x Wq^T, k = x Wk^T (phi = identity), g = scale * log sigma(x Wg^T),
    each [B, H, T, dk] (None where its weight is None).  x [B, T, Dm], W
    [H*dk, Dm]."""
    lib = lib or load()
    (x, px) = _in(x)
    B, T, Dm = x.shape
    ws = [_in(w) for w in (Wq, Wk, Wg)]
    outs = [(_out((B, H, T, dk)) if w is not None else (None, None)) for w in (Wq, Wk, Wg)]
    _check(lib.oracle_qkg_projection(B, T, Dm, H, dk, px, ws[0][1], ws[1][1], ws[2][1],
                                     float(scale), outs[0][1], outs[1][1], outs[2][1]),
           "qkg_projection")
    return outs[0][0], outs[1][0], outs[2][0]

