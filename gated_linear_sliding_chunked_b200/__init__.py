"""Python binding of the B200 hybrid attention library (liblizard.so).

The operator is the hybrid attention of "Lizard: An Efficient Linearization
Framework for Large Language Models" (gist.science technical summary,
section 2a): gated linear attention S_t = diag(exp(g_t)) S_{t-1} + k_t v_t^T,
o_gla_t = q_t^T S_t, plus sliding-window softmax attention with meta-memory
sink tokens, summed as o = o_gla + alpha * o_swa.

Everything here is argument marshalling: the ``lz_*`` functions have the C
ABI's names and arguments (include/lizard.h) and take torch tensors for the
pointers; the helpers without the prefix only allocate outputs and scratch
with torch and call them.  Every step of the computation runs in the CUDA
library.  There is no CPU fallback: if liblizard.so is missing, loading it
raises.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "liblizard.so")

LZ_OK, LZ_ERR_INVALID_ARG, LZ_ERR_UNSUPPORTED, LZ_ERR_CUDA, LZ_ERR_TIMEOUT = range(5)
LZ_F32, LZ_BF16 = 0, 1
(LZ_WS_GLA_FWD, LZ_WS_HYBRID_FWD, LZ_WS_GLA_BWD, LZ_WS_SWA_BWD, LZ_WS_HYBRID_BWD,
 LZ_WS_CHUNK_STATES, LZ_WS_HYBRID_FWD_MSE) = range(7)

EXPORTS = ("lz_gla_fwd", "lz_gla_bwd", "lz_swa_meta_fwd", "lz_hybrid_fwd", "lz_swa_meta_bwd",
           "lz_hybrid_bwd", "lz_gla_decode_step", "lz_workspace_bytes", "lz_last_error",
           "lz_version", "lz_timing_enable", "lz_timing_only", "lz_timing_read",
           "lz_swa_meta_bwd_noalloc", "lz_device_check", "lz_prefer_tcgen05", "lz_decode_prefill",
           "lz_hybrid_fwd_mse", "lz_selftest_bounded_wait", "lz_cp_segment_decay", "lz_cp_fold",
           "lz_cp_rows", "lz_tcgen05_all", "lz_qkg_projection", "lz_fused_gate_logits")

# size of the static scratch array behind lz_swa_meta_bwd_noalloc
LZ_NOALLOC_SCRATCH_BYTES = 16 << 20


class LzError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"lizard status {status}: {message}")
        self.status = status


class LzDims(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("T", ctypes.c_int),
                ("dk", ctypes.c_int), ("dv", ctypes.c_int), ("chunk", ctypes.c_int),
                ("w", ctypes.c_int), ("M", ctypes.c_int), ("io", ctypes.c_int),
                ("scale", ctypes.c_float), ("alpha", ctypes.c_float),
                ("gate_logits", ctypes.c_int), ("gate_scale", ctypes.c_float)]


_lib = None
_P = ctypes.c_void_p


def load(path: str = LIB_PATH):
    """Load liblizard.so (raises if it is absent: there is no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"CUDA library not built: {path} is missing "
                           "(run python -m gated_linear_sliding_chunked_b200.build)")
    lib = ctypes.CDLL(path)
    D = ctypes.POINTER(LzDims)
    sz = ctypes.c_size_t
    lib.lz_workspace_bytes.argtypes = [D, ctypes.c_int]
    lib.lz_workspace_bytes.restype = sz
    lib.lz_gla_fwd.argtypes = [D] + [_P] * 8 + [_P, sz, _P]
    lib.lz_swa_meta_fwd.argtypes = [D] + [_P] * 7 + [_P]
    lib.lz_hybrid_fwd.argtypes = [D] + [_P] * 12 + [_P, sz, _P]
    lib.lz_hybrid_fwd_mse.argtypes = [D] + [_P] * 15 + [_P, sz, _P]
    lib.lz_gla_bwd.argtypes = [D] + [_P] * 14 + [_P, sz, _P]
    lib.lz_swa_meta_bwd.argtypes = [D] + [_P] * 13 + [_P, sz, _P]
    lib.lz_hybrid_bwd.argtypes = [D] + [_P] * 21 + [_P, sz, _P]
    lib.lz_swa_meta_bwd_noalloc.argtypes = [D] + [_P] * 13 + [_P]
    lib.lz_gla_decode_step.argtypes = ([ctypes.c_int] * 7 + [ctypes.c_float] * 2 +
                                       [_P] * 11 + [_P])
    lib.lz_device_check.argtypes = [_P]
    lib.lz_selftest_bounded_wait.argtypes = [_P]
    lib.lz_decode_prefill.argtypes = [ctypes.c_int] * 7 + [_P] * 8 + [_P]
    lib.lz_prefer_tcgen05.argtypes = [ctypes.c_int]
    ci = ctypes.c_int
    lib.lz_tcgen05_all.argtypes = [ci]
    lib.lz_fused_gate_logits.argtypes = [ci]
    lib.lz_qkg_projection.argtypes = [ci] * 5 + [_P] * 4 + [ctypes.c_float] + [_P] * 3 + [_P]
    lib.lz_cp_segment_decay.argtypes = [ci, ci, ci, _P, _P, _P]
    lib.lz_cp_fold.argtypes = [ci] * 6 + [_P] * 4 + [_P]
    lib.lz_cp_rows.argtypes = ([ci] * 4 + [_P, ci, ci, ctypes.c_float, _P, ci, ci, _P, ci, ci] +
                               [_P])
    lib.lz_timing_enable.argtypes = [ctypes.c_int]
    lib.lz_timing_only.argtypes = [ctypes.c_char_p]
    lib.lz_timing_read.argtypes = [ctypes.c_char_p, sz, ctypes.POINTER(ctypes.c_float),
                                   ctypes.c_int]
    for name in EXPORTS:
        if name in ("lz_last_error", "lz_version"):
            getattr(lib, name).restype = ctypes.c_char_p
            getattr(lib, name).argtypes = []
        elif name != "lz_workspace_bytes":
            getattr(lib, name).restype = ctypes.c_int
    _lib = lib
    return lib


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int):
    if status != LZ_OK:
        raise LzError(status, load().lz_last_error().decode())


def io_of(dtype) -> int:
    if dtype == torch.float32:
        return LZ_F32
    if dtype == torch.bfloat16:
        return LZ_BF16
    raise TypeError(f"unsupported I/O dtype {dtype}")


def make_dims(B, H, T, dk, dv, *, chunk=64, w=1, M=0, io=LZ_BF16, scale=None,
              alpha=0.5, gate_logits=False, gate_scale=1.0) -> LzDims:
    """gate_logits: the `g` tensors of the calls are bf16 gate logits z (the
    log-gate is gate_scale * log sigma(z)) instead of fp32 log-gates."""
    if scale is None:
        scale = 1.0 / math.sqrt(dk)
    return LzDims(B, H, T, dk, dv, chunk, w, M, io, float(scale), float(alpha),
                  int(bool(gate_logits)), float(gate_scale))


# --------------------------------------------------------------------------
# C ABI mirrors (pointers from tensors, nothing else)
# --------------------------------------------------------------------------
def lz_workspace_bytes(dims: LzDims, which: int) -> int:
    return int(load().lz_workspace_bytes(ctypes.byref(dims), which))


def lz_device_check(stream=None):
    """Raises LzError(LZ_ERR_TIMEOUT) if a bounded device wait of a library
    kernel gave up since the last check (synchronizes the stream)."""
    _check(load().lz_device_check(_stream(stream)))


def lz_selftest_bounded_wait(stream=None):
    """Launches the library's failure-path self-test: a bounded device wait
    that nothing completes gives up after 0.2 s; the next lz_device_check
    raises LzError(LZ_ERR_TIMEOUT)."""
    _check(load().lz_selftest_bounded_wait(_stream(stream)))


def lz_prefer_tcgen05(on: bool) -> bool:
    """Window kernels on tcgen05 where they apply (the default) or, with
    False, on the warp-level ones, for the calling thread; returns the
    previous setting."""
    return bool(load().lz_prefer_tcgen05(1 if on else 0))


def lz_tcgen05_all(on: bool) -> bool:
    """Also the tcgen05 kernels that measured slower than their warp-level
    counterparts (the gated backward's per-chunk gradients, the window
    backward's query side), for the calling thread (default False); returns
    the previous setting."""
    return bool(load().lz_tcgen05_all(1 if on else 0))


def lz_fused_gate_logits(on: bool) -> bool:
    """Gates given as logits mapped inside every gated kernel (True) instead
    of by one pass into the workspace (False, the default), for the calling
    thread; returns the previous setting."""
    return bool(load().lz_fused_gate_logits(1 if on else 0))


def lz_timing_enable(on: bool):
    load().lz_timing_enable(1 if on else 0)


def lz_timing_only(name: str | None):
    """Time only the launches of kernel `name` (None: every launch)."""
    load().lz_timing_only(name.encode() if name else None)


def lz_timing_read(max_records: int = 1 << 16):
    """[(kernel name, milliseconds)] of the launches recorded since the last
    read (waits for them to finish)."""
    stride = 48
    names = ctypes.create_string_buffer(stride * max_records)
    ms = (ctypes.c_float * max_records)()
    n = load().lz_timing_read(names, stride, ms, max_records)
    out = []
    for i in range(min(n, max_records)):
        nm = names.raw[i * stride:(i + 1) * stride].split(b"\0", 1)[0].decode()
        out.append((nm, float(ms[i])))
    return out


def lz_gla_fwd(dims, q, k, v, g, h0, o, hT, chunk_states, ws, ws_bytes, stream=None):
    _check(load().lz_gla_fwd(ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(h0),
                             _ptr(o), _ptr(hT), _ptr(chunk_states), _ptr(ws), ws_bytes,
                             _stream(stream)))


def lz_swa_meta_fwd(dims, q, k, v, meta_k, meta_v, o, lse, stream=None):
    _check(load().lz_swa_meta_fwd(ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v), _ptr(meta_k),
                                  _ptr(meta_v), _ptr(o), _ptr(lse), _stream(stream)))


def lz_hybrid_fwd_mse(dims, q, k, v, g, meta_k, meta_v, h0, target, o, hT, lse, o_swa,
                      chunk_states, loss, dO, ws, ws_bytes, stream=None):
    _check(load().lz_hybrid_fwd_mse(ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v), _ptr(g),
                                    _ptr(meta_k), _ptr(meta_v), _ptr(h0), _ptr(target), _ptr(o),
                                    _ptr(hT), _ptr(lse), _ptr(o_swa), _ptr(chunk_states),
                                    _ptr(loss), _ptr(dO), _ptr(ws), ws_bytes, _stream(stream)))


def lz_hybrid_fwd(dims, q, k, v, g, meta_k, meta_v, h0, o, hT, lse, o_swa, chunk_states, ws,
                  ws_bytes, stream=None):
    _check(load().lz_hybrid_fwd(ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v), _ptr(g),
                                _ptr(meta_k), _ptr(meta_v), _ptr(h0), _ptr(o), _ptr(hT),
                                _ptr(lse), _ptr(o_swa), _ptr(chunk_states), _ptr(ws), ws_bytes,
                                _stream(stream)))


def lz_gla_bwd(dims, q, k, v, g, h0, dO, dhT, chunk_states, hT, dq, dk, dv, dg, dh0, ws,
               ws_bytes, stream=None):
    _check(load().lz_gla_bwd(ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(h0),
                             _ptr(dO), _ptr(dhT), _ptr(chunk_states), _ptr(hT), _ptr(dq),
                             _ptr(dk), _ptr(dv), _ptr(dg), _ptr(dh0), _ptr(ws), ws_bytes,
                             _stream(stream)))


def lz_swa_meta_bwd(dims, q, k, v, meta_k, meta_v, lse, o, dO, dq, dk, dv, dmeta_k, dmeta_v,
                    ws, ws_bytes, stream=None):
    _check(load().lz_swa_meta_bwd(ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v), _ptr(meta_k),
                                  _ptr(meta_v), _ptr(lse), _ptr(o), _ptr(dO), _ptr(dq), _ptr(dk),
                                  _ptr(dv), _ptr(dmeta_k), _ptr(dmeta_v), _ptr(ws), ws_bytes,
                                  _stream(stream)))


def lz_swa_meta_bwd_noalloc(dims, q, k, v, meta_k, meta_v, lse, o, dO, dq, dk, dv, dmeta_k,
                            dmeta_v, stream=None):
    """lz_swa_meta_bwd without caller scratch: for callers that cannot
    allocate device memory; uses the library's static scratch array (see
    include/lizard.h for the size limit and the rule against overlapping
    calls)."""
    _check(load().lz_swa_meta_bwd_noalloc(ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v),
                                          _ptr(meta_k), _ptr(meta_v), _ptr(lse), _ptr(o),
                                          _ptr(dO),
                                          _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dmeta_k),
                                          _ptr(dmeta_v), _stream(stream)))


def lz_hybrid_bwd(dims, q, k, v, g, meta_k, meta_v, h0, lse, o_swa, chunk_states, hT, dO, dhT,
                  dq, dk, dv, dg, dh0, dmeta_k, dmeta_v, dalpha, ws, ws_bytes, stream=None):
    _check(load().lz_hybrid_bwd(ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v), _ptr(g),
                                _ptr(meta_k), _ptr(meta_v), _ptr(h0), _ptr(lse), _ptr(o_swa),
                                _ptr(chunk_states), _ptr(hT), _ptr(dO),
                                _ptr(dhT), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dg), _ptr(dh0),
                                _ptr(dmeta_k), _ptr(dmeta_v), _ptr(dalpha), _ptr(ws), ws_bytes,
                                _stream(stream)))


def lz_gla_decode_step(Bd, H, dk, dv, w, M, io, scale, alpha, state, kring, vring, pos, q, k,
                       v, g, meta_k, meta_v, o, stream=None):
    _check(load().lz_gla_decode_step(Bd, H, dk, dv, w, M, io, float(scale), float(alpha),
                                     _ptr(state), _ptr(kring), _ptr(vring), _ptr(pos), _ptr(q),
                                     _ptr(k), _ptr(v), _ptr(g), _ptr(meta_k), _ptr(meta_v),
                                     _ptr(o), _stream(stream)))


# --------------------------------------------------------------------------
# Allocating helpers (torch owns memory; the library computes)
# --------------------------------------------------------------------------
def _dims_from(q, v, *, chunk, w, M, scale, alpha, g=None, gate_scale=1.0):
    """A bf16 `g` is read as gate logits (log-gate = gate_scale * log sigma(g));
    an fp32 `g` as log-gates."""
    B, H, T, dk = q.shape
    logits = g is not None and g.dtype != torch.float32
    return make_dims(B, H, T, dk, v.shape[-1], chunk=chunk, w=w, M=M, io=io_of(q.dtype),
                     scale=scale, alpha=alpha, gate_logits=logits, gate_scale=gate_scale)


def _ws(dims, which, device):
    n = lz_workspace_bytes(dims, which)
    return (torch.empty(max(n, 1), dtype=torch.uint8, device=device), n)


def _M(meta_k):
    return 0 if meta_k is None else int(meta_k.shape[1])


def _chunk_states(dims, device):
    """Buffer for the forward's chunk states, or None where the kernels keep
    none (LZ_WS_CHUNK_STATES)."""
    n = lz_workspace_bytes(dims, LZ_WS_CHUNK_STATES)
    return torch.empty(n, dtype=torch.uint8, device=device) if n else None


def gla_fwd(q, k, v, g, h0=None, *, chunk=64, gate_scale=1.0, want_hT=False, want_chunk_states=False,
            stream=None):
    """Returns (o, hT), or (o, hT, chunk_states) with want_chunk_states.  A bf16
    g holds gate logits (log-gate = gate_scale * log sigma(g))."""
    d = _dims_from(q, v, chunk=chunk, w=1, M=0, scale=None, alpha=0.0, g=g, gate_scale=gate_scale)
    o = torch.empty(q.shape[:-1] + (v.shape[-1],), dtype=q.dtype, device=q.device)
    hT = torch.empty(q.shape[0], q.shape[1], q.shape[-1], v.shape[-1], dtype=torch.float32,
                     device=q.device) if want_hT else None
    cs = _chunk_states(d, q.device) if want_chunk_states else None
    ws, n = _ws(d, LZ_WS_GLA_FWD, q.device)
    lz_gla_fwd(d, q, k, v, g, h0, o, hT, cs, ws, n, stream)
    return (o, hT, cs) if want_chunk_states else (o, hT)


def swa_meta_fwd(q, k, v, meta_k, meta_v, *, w, scale=None, want_lse=True, stream=None):
    d = _dims_from(q, v, chunk=64, w=w, M=_M(meta_k), scale=scale, alpha=1.0)
    o = torch.empty(q.shape[:-1] + (v.shape[-1],), dtype=q.dtype, device=q.device)
    lse = torch.empty(q.shape[:-1], dtype=torch.float32, device=q.device) if want_lse else None
    lz_swa_meta_fwd(d, q, k, v, meta_k, meta_v, o, lse, stream)
    return o, lse


def hybrid_fwd(q, k, v, g, meta_k, meta_v, *, w, alpha, scale=None, chunk=64, h0=None,
               gate_scale=1.0, want_hT=False, want_lse=False, want_o_swa=False,
               want_chunk_states=False, stream=None):
    """A bf16 g holds gate logits (log-gate = gate_scale * log sigma(g))."""
    d = _dims_from(q, v, chunk=chunk, w=w, M=_M(meta_k), scale=scale, alpha=alpha, g=g,
                   gate_scale=gate_scale)
    dev = q.device
    o = torch.empty(q.shape[:-1] + (v.shape[-1],), dtype=q.dtype, device=dev)
    hT = torch.empty(q.shape[0], q.shape[1], q.shape[-1], v.shape[-1], dtype=torch.float32,
                     device=dev) if want_hT else None
    lse = torch.empty(q.shape[:-1], dtype=torch.float32, device=dev) if want_lse else None
    osw = torch.empty_like(o) if want_o_swa else None
    cs = _chunk_states(d, dev) if want_chunk_states else None
    ws, n = _ws(d, LZ_WS_HYBRID_FWD, dev)
    lz_hybrid_fwd(d, q, k, v, g, meta_k, meta_v, h0, o, hT, lse, osw, cs, ws, n, stream)
    return {"o": o, "hT": hT, "lse": lse, "o_swa": osw, "chunk_states": cs}


def hybrid_fwd_mse(q, k, v, g, meta_k, meta_v, target, *, w, alpha, scale=None, chunk=64,
                   h0=None, gate_scale=1.0, want_dO=True, want_hT=False, want_lse=False, want_o_swa=False,
                   want_chunk_states=False, stream=None):
    """hybrid_fwd plus the stage-1 loss mean((o - target)^2); the result adds
    "loss" (0-dim fp32 tensor on the device) and "dO" (its gradient, or None)."""
    d = _dims_from(q, v, chunk=chunk, w=w, M=_M(meta_k), scale=scale, alpha=alpha, g=g,
                   gate_scale=gate_scale)
    dev = q.device
    o = torch.empty(q.shape[:-1] + (v.shape[-1],), dtype=q.dtype, device=dev)
    hT = torch.empty(q.shape[0], q.shape[1], q.shape[-1], v.shape[-1], dtype=torch.float32,
                     device=dev) if want_hT else None
    lse = torch.empty(q.shape[:-1], dtype=torch.float32, device=dev) if want_lse else None
    osw = torch.empty_like(o) if want_o_swa else None
    cs = _chunk_states(d, dev) if want_chunk_states else None
    loss = torch.empty((), dtype=torch.float32, device=dev)
    dO = torch.empty_like(o) if want_dO else None
    ws, n = _ws(d, LZ_WS_HYBRID_FWD_MSE, dev)
    lz_hybrid_fwd_mse(d, q, k, v, g, meta_k, meta_v, h0, target, o, hT, lse, osw, cs, loss, dO,
                      ws, n, stream)
    return {"o": o, "hT": hT, "lse": lse, "o_swa": osw, "chunk_states": cs, "loss": loss,
            "dO": dO}


def gla_bwd(q, k, v, g, dO, h0=None, dhT=None, *, chunk=64, chunk_states=None, hT=None,
            gate_scale=1.0, want_dh0=False, stream=None):
    """chunk_states, hT: the forward's (optional; see lz_gla_bwd)."""
    d = _dims_from(q, v, chunk=chunk, w=1, M=0, scale=None, alpha=0.0, g=g, gate_scale=gate_scale)
    dev = q.device
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dg = torch.empty(g.shape, dtype=torch.float32, device=dev)  # dL/dz for gate logits
    dh0 = torch.empty(q.shape[0], q.shape[1], q.shape[-1], v.shape[-1], dtype=torch.float32,
                      device=dev) if want_dh0 else None
    ws, n = _ws(d, LZ_WS_GLA_BWD, dev)
    lz_gla_bwd(d, q, k, v, g, h0, dO, dhT, chunk_states, hT, dq, dk, dv, dg, dh0, ws, n, stream)
    return {"dq": dq, "dk": dk, "dv": dv, "dg": dg, "dh0": dh0}


def swa_meta_bwd(q, k, v, meta_k, meta_v, lse, dO, *, w, scale=None, o=None, stream=None):
    """o: the forward output (optional; see lz_swa_meta_bwd)."""
    M = _M(meta_k)
    d = _dims_from(q, v, chunk=64, w=w, M=M, scale=scale, alpha=1.0)
    dev = q.device
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dmk = torch.empty(q.shape[1], M, q.shape[-1], dtype=torch.float32, device=dev) if M else None
    dmv = torch.empty(q.shape[1], M, v.shape[-1], dtype=torch.float32, device=dev) \
        if (M and meta_v is not None) else None
    ws, n = _ws(d, LZ_WS_SWA_BWD, dev)
    lz_swa_meta_bwd(d, q, k, v, meta_k, meta_v, lse, o, dO, dq, dk, dv, dmk, dmv, ws, n, stream)
    return {"dq": dq, "dk": dk, "dv": dv, "dmeta_k": dmk, "dmeta_v": dmv}


def hybrid_bwd(q, k, v, g, meta_k, meta_v, lse, dO, *, w, alpha, scale=None, chunk=64,
               h0=None, dhT=None, o_swa=None, chunk_states=None, hT=None, gate_scale=1.0,
               want_dh0=False, stream=None):
    """o_swa, chunk_states, hT: the forward's (optional; see lz_hybrid_bwd).  A bf16
    g holds gate logits; dg then receives dL/dg_logits (fp32)."""
    M = _M(meta_k)
    d = _dims_from(q, v, chunk=chunk, w=w, M=M, scale=scale, alpha=alpha, g=g,
                   gate_scale=gate_scale)
    dev = q.device
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dg = torch.empty(g.shape, dtype=torch.float32, device=dev)  # dL/dz for gate logits
    dh0 = torch.empty(q.shape[0], q.shape[1], q.shape[-1], v.shape[-1], dtype=torch.float32,
                      device=dev) if want_dh0 else None
    dmk = torch.empty(q.shape[1], M, q.shape[-1], dtype=torch.float32, device=dev) if M else None
    dmv = torch.empty(q.shape[1], M, v.shape[-1], dtype=torch.float32, device=dev) \
        if (M and meta_v is not None) else None
    dalpha = torch.empty(4, dtype=torch.float32, device=dev)
    ws, n = _ws(d, LZ_WS_HYBRID_BWD, dev)
    lz_hybrid_bwd(d, q, k, v, g, meta_k, meta_v, h0, lse, o_swa, chunk_states, hT, dO, dhT, dq,
                  dk, dv, dg, dh0, dmk, dmv, dalpha, ws, n, stream)
    return {"dq": dq, "dk": dk, "dv": dv, "dg": dg, "dh0": dh0, "dmeta_k": dmk,
            "dmeta_v": dmv, "dalpha": dalpha[:1]}


def lz_decode_prefill(Bd, H, T, dk, dv, w, io, k, v, lens, hT, state, kring, vring, pos,
                      stream=None):
    _check(load().lz_decode_prefill(Bd, H, T, dk, dv, w, io, _ptr(k), _ptr(v), _ptr(lens),
                                    _ptr(hT), _ptr(state), _ptr(kring), _ptr(vring), _ptr(pos),
                                    _stream(stream)))


def decode_prefill(k, v, hT, *, w, lens=None, stream=None):
    """Decode buffers after a prefill of k, v [Bd, H, T, 128] with final state
    hT: returns (state, kring, vring, pos) ready for decode_step.  lens: an
    int64 tensor [Bd] of per-sequence prompt lengths (right-padded prompts,
    padding with k = 0 and g = 0), or None for T each."""
    Bd, H, T, dk = k.shape
    dv = v.shape[-1]
    dev = k.device
    if lens is not None:
        lens = lens.to(device=dev, dtype=torch.int64).contiguous()
        if lens.shape != (Bd,):
            raise ValueError(f"lens must have shape ({Bd},), got {tuple(lens.shape)}")
    state = torch.empty(Bd, H, dk, dv, dtype=torch.float32, device=dev)
    kring = torch.zeros(Bd, H, w, dk, dtype=k.dtype, device=dev)
    vring = torch.zeros(Bd, H, w, dv, dtype=v.dtype, device=dev)
    pos = torch.empty(Bd, dtype=torch.int64, device=dev)
    lz_decode_prefill(Bd, H, T, dk, dv, w, io_of(k.dtype), k, v, lens, hT, state, kring, vring,
                      pos, stream)
    return state, kring, vring, pos


def decode_step(state, kring, vring, pos, q, k, v, g, meta_k, meta_v, *, alpha, scale=None,
                o=None, stream=None):
    """One in-place generation step; returns o [Bd, H, dv]."""
    Bd, H, dk = q.shape
    dv = v.shape[-1]
    w = kring.shape[2]
    M = _M(meta_k)
    if scale is None:
        scale = 1.0 / math.sqrt(dk)
    if o is None:
        o = torch.empty(Bd, H, dv, dtype=q.dtype, device=q.device)
    lz_gla_decode_step(Bd, H, dk, dv, w, M, io_of(q.dtype), scale, alpha, state, kring, vring,
                       pos, q, k, v, g, meta_k, meta_v, o, stream)
    return o


# ---- context parallelism (one sequence over several ranks) -----------------
def lz_cp_segment_decay(BH, T, dk, g, E, stream=None):
    _check(load().lz_cp_segment_decay(BH, T, dk, _ptr(g), _ptr(E), _stream(stream)))


def lz_cp_fold(R, r, direction, BH, dk, dv, E, X, init, out, stream=None):
    _check(load().lz_cp_fold(R, r, direction, BH, dk, dv, _ptr(E), _ptr(X), _ptr(init),
                             _ptr(out), _stream(stream)))


def lz_cp_rows(BH, d, io, n, A, a_T, a_off, a_scale, B, b_T, b_off, dst, dst_T, dst_off,
               stream=None):
    _check(load().lz_cp_rows(BH, d, io, n, _ptr(A), a_T, a_off, float(a_scale), _ptr(B), b_T,
                             b_off, _ptr(dst), dst_T, dst_off, _stream(stream)))


def segment_decay(g):
    """Per (batch, head, key dim) product of a segment's gates: g [B, H, T, dk]
    fp32 log-gates -> [B, H, dk] fp32."""
    B, H, T, dk = g.shape
    E = torch.empty(B, H, dk, dtype=torch.float32, device=g.device)
    lz_cp_segment_decay(B * H, T, dk, g, E)
    return E


def cp_fold(E_all, X_all, r, direction, init=None):
    """Fold over segments (see lz_cp_fold): E_all [R, B, H, dk], X_all
    [R, B, H, dk, dv] fp32 -> [B, H, dk, dv]."""
    R, B, H, dk, dv = X_all.shape
    out = torch.empty(B, H, dk, dv, dtype=torch.float32, device=X_all.device)
    lz_cp_fold(R, r, direction, B * H, dk, dv, E_all.contiguous(), X_all.contiguous(),
               None if init is None else init.contiguous(), out)
    return out


def cp_rows(dst, dst_off, n, A=None, a_off=0, a_scale=1.0, B=None, b_off=0):
    """dst[:, :, dst_off + t] = a_scale * A[:, :, a_off + t] + B[:, :, b_off + t]
    for t < n, in place on dst ([batch, head, rows, d] tensors of one dtype;
    None = zeros).  Returns dst."""
    Bb, H, dT, d = dst.shape
    for x in (A, B):
        if x is not None and (x.dtype != dst.dtype or x.shape[:2] != dst.shape[:2]
                              or x.shape[3] != d):
            raise ValueError("cp_rows: tensors must share dtype, batch, heads and d")
    lz_cp_rows(Bb * H, d, io_of(dst.dtype), n, A, 0 if A is None else A.shape[2], a_off, a_scale,
               B, 0 if B is None else B.shape[2], b_off, dst, dT, dst_off)
    return dst


# ---- the projections in front of the operator ------------------------------
def lz_qkg_projection(B, T, Dm, H, dk, x, Wq, Wk, Wg, gate_scale, q, k, g, stream=None):
    _check(load().lz_qkg_projection(B, T, Dm, H, dk, _ptr(x), _ptr(Wq), _ptr(Wk), _ptr(Wg),
                                    float(gate_scale), _ptr(q), _ptr(k), _ptr(g),
                                    _stream(stream)))


def qkg_projection(x, Wq=None, Wk=None, Wg=None, *, heads, gate_scale=1.0, stream=None):
    """x [B, T, Dm] bf16, W [heads * dk, Dm] bf16 -> (q, k, g): q, k [B, heads,
    T, dk] bf16 and g = gate_scale * logsigmoid(x Wg^T) [B, heads, T, dk] fp32
    (None where the weight is None)."""
    B, T, Dm = x.shape
    Wany = next(w for w in (Wq, Wk, Wg) if w is not None)
    dk = Wany.shape[0] // heads
    dev = x.device
    q = torch.empty(B, heads, T, dk, dtype=torch.bfloat16, device=dev) if Wq is not None else None
    k = torch.empty(B, heads, T, dk, dtype=torch.bfloat16, device=dev) if Wk is not None else None
    g = torch.empty(B, heads, T, dk, dtype=torch.float32, device=dev) if Wg is not None else None
    lz_qkg_projection(B, T, Dm, heads, dk, x, Wq, Wk, Wg, gate_scale, q, k, g, stream)
    return q, k, g

