"""The C-ABI library loads, exports every entry point include/lizard.h
declares, and rejects bad arguments on the host before any launch.  No
compute call is made (CPU only)."""
import ctypes
import os
import re

import pytest

import gated_linear_sliding_chunked_b200 as L
from gated_linear_sliding_chunked_b200 import build as lbuild

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                      "lizard.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(lz_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    lbuild.build()
    return L.load()


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("lz_gla_fwd", "lz_gla_bwd", "lz_swa_meta_fwd", "lz_hybrid_fwd",
              "lz_gla_decode_step", "lz_swa_meta_bwd", "lz_hybrid_bwd", "lz_workspace_bytes",
              "lz_last_error"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_version(lib):
    assert b"sm_100a" in lib.lz_version()


FAKE = 0x7F0000000000  # never dereferenced: validation fails first


def _dims(**kw):
    base = dict(B=1, H=2, T=64, dk=64, dv=64, chunk=64, w=8, M=2, io=L.LZ_BF16, scale=0.125,
                alpha=0.5, gate_logits=0, gate_scale=1.0)
    base.update(kw)
    return L.LzDims(*[base[f] for f, _ in L.LzDims._fields_])


def _call_hybrid(lib, d, **ptrs):
    p = dict(q=FAKE, k=FAKE, v=FAKE, g=FAKE, mk=FAKE, mv=FAKE, h0=None, o=FAKE, hT=None,
             lse=None, osw=None, ws=FAKE)
    p.update(ptrs)
    return lib.lz_hybrid_fwd(ctypes.byref(d), p["q"], p["k"], p["v"], p["g"], p["mk"], p["mv"],
                             p["h0"], p["o"], p["hT"], p["lse"], p["osw"], None, p["ws"],
                             ptrs.get("ws_bytes", 1 << 40), 0)


@pytest.mark.parametrize("kw,status", [
    (dict(dk=96), L.LZ_ERR_UNSUPPORTED),
    (dict(dv=32), L.LZ_ERR_UNSUPPORTED),
    (dict(chunk=48), L.LZ_ERR_UNSUPPORTED),
    (dict(w=0), L.LZ_ERR_UNSUPPORTED),
    (dict(w=1025), L.LZ_ERR_UNSUPPORTED),
    (dict(M=17), L.LZ_ERR_UNSUPPORTED),
    (dict(M=-1), L.LZ_ERR_UNSUPPORTED),
    (dict(io=7), L.LZ_ERR_UNSUPPORTED),
    (dict(T=-1), L.LZ_ERR_INVALID_ARG),
    (dict(B=-2), L.LZ_ERR_INVALID_ARG),
])
def test_bad_shapes_rejected(lib, kw, status):
    assert _call_hybrid(lib, _dims(**kw)) == status
    assert lib.lz_last_error()


@pytest.mark.parametrize("which", ["q", "k", "v", "g", "o", "mk"])
def test_null_required_pointer_rejected(lib, which):
    assert _call_hybrid(lib, _dims(), **{which: None}) == L.LZ_ERR_INVALID_ARG
    assert b"NULL" in lib.lz_last_error()


def test_meta_k_may_be_null_without_meta(lib):
    # M == 0: meta_k NULL passes validation; the workspace check then fails
    # because no workspace is given, still before any launch.
    st = _call_hybrid(lib, _dims(M=0), mk=None, mv=None, ws=None)
    assert st == L.LZ_ERR_INVALID_ARG and b"workspace" in lib.lz_last_error()


@pytest.mark.parametrize("which", ["q", "v", "g", "o", "h0", "lse"])
def test_misaligned_pointer_rejected(lib, which):
    assert _call_hybrid(lib, _dims(), **{which: FAKE + 4}) == L.LZ_ERR_INVALID_ARG
    assert b"aligned" in lib.lz_last_error()


def test_short_workspace_rejected(lib):
    d = _dims()
    need = L.lz_workspace_bytes(d, L.LZ_WS_HYBRID_FWD)
    assert need > 0
    assert _call_hybrid(lib, d, ws_bytes=need - 1) == L.LZ_ERR_INVALID_ARG
    assert b"too small" in lib.lz_last_error()


def test_workspace_sizes_grow_with_problem(lib):
    small = L.lz_workspace_bytes(_dims(T=64), L.LZ_WS_HYBRID_BWD)
    big = L.lz_workspace_bytes(_dims(T=4096), L.LZ_WS_HYBRID_BWD)
    assert 0 < small < big
    assert L.lz_workspace_bytes(_dims(dk=96), L.LZ_WS_HYBRID_BWD) == 0


def test_decode_validation(lib):
    f = lib.lz_gla_decode_step
    args = [FAKE] * 11
    assert f(4, 2, 64, 128, 16, 2, L.LZ_BF16, 0.1, 0.5, *args, 0) == L.LZ_ERR_UNSUPPORTED
    assert f(4, 2, 128, 128, 0, 2, L.LZ_BF16, 0.1, 0.5, *args, 0) == L.LZ_ERR_UNSUPPORTED
    assert f(4, 2, 128, 128, 16, 17, L.LZ_BF16, 0.1, 0.5, *args, 0) == L.LZ_ERR_UNSUPPORTED
    # the position word holds a 15-bit arrival count of the heads during a step
    assert f(4, 32768, 128, 128, 16, 2, L.LZ_BF16, 0.1, 0.5, *args, 0) == L.LZ_ERR_UNSUPPORTED
    assert f(-1, 2, 128, 128, 16, 2, L.LZ_BF16, 0.1, 0.5, *args, 0) == L.LZ_ERR_INVALID_ARG
    bad = list(args)
    bad[0] = None  # state
    assert f(4, 2, 128, 128, 16, 2, L.LZ_BF16, 0.1, 0.5, *bad, 0) == L.LZ_ERR_INVALID_ARG
    bad = list(args)
    bad[3] = FAKE + 8  # pos misaligned
    assert f(4, 2, 128, 128, 16, 2, L.LZ_BF16, 0.1, 0.5, *bad, 0) == L.LZ_ERR_INVALID_ARG


def test_backward_validation(lib):
    d = _dims()
    P = [FAKE] * 21
    # lse is required by the hybrid backward
    P2 = list(P)
    P2[7] = None
    assert lib.lz_hybrid_bwd(ctypes.byref(d), *P2, FAKE, 1 << 40, 0) == L.LZ_ERR_INVALID_ARG
    # dalpha only needs 4-byte alignment, but not 2
    P3 = list(P)
    P3[20] = FAKE + 2
    assert lib.lz_hybrid_bwd(ctypes.byref(d), *P3, FAKE, 1 << 40, 0) == L.LZ_ERR_INVALID_ARG
    assert lib.lz_gla_bwd(ctypes.byref(_dims(dk=32)), *([FAKE] * 14), FAKE, 1 << 40, 0) == \
        L.LZ_ERR_UNSUPPORTED


def test_chunk_states_size_and_validation(lib):
    """The forward's chunk states exist for bf16 with d = 128 only; handing
    them to a backward that gets dL/dhT also needs the final state."""
    d = _dims(T=200, dk=128, dv=128)
    assert L.lz_workspace_bytes(d, L.LZ_WS_CHUNK_STATES) == 1 * 2 * 4 * 128 * 128 * 2
    assert L.lz_workspace_bytes(_dims(T=200, dk=128, dv=128, io=L.LZ_F32),
                                L.LZ_WS_CHUNK_STATES) == 0
    assert L.lz_workspace_bytes(_dims(T=200), L.LZ_WS_CHUNK_STATES) == 0
    P = [FAKE] * 21
    P[12] = FAKE  # dhT given
    P[10] = None  # hT missing
    assert lib.lz_hybrid_bwd(ctypes.byref(d), *P, FAKE, 1 << 40, 0) == L.LZ_ERR_INVALID_ARG
    assert b"hT" in lib.lz_last_error()
    # the same for the gated-only backward (chunk_states at 8, hT at 9)
    G = [FAKE] * 14
    G[9] = None
    assert lib.lz_gla_bwd(ctypes.byref(d), *G, FAKE, 1 << 40, 0) == L.LZ_ERR_INVALID_ARG


def test_decode_prefill_validation(lib):
    f = lib.lz_decode_prefill
    # k, v, lens, hT, state, kring, vring, pos
    args = [FAKE, FAKE, None, None, FAKE, FAKE, FAKE, FAKE]
    assert f(2, 2, 10, 64, 128, 16, L.LZ_BF16, *args, 0) == L.LZ_ERR_UNSUPPORTED
    assert f(2, 2, 10, 128, 128, 0, L.LZ_BF16, *args, 0) == L.LZ_ERR_UNSUPPORTED
    assert f(2, 2, -1, 128, 128, 16, L.LZ_BF16, *args, 0) == L.LZ_ERR_INVALID_ARG
    bad = list(args)
    bad[0] = None  # k missing with T > 0
    assert f(2, 2, 10, 128, 128, 16, L.LZ_BF16, *bad, 0) == L.LZ_ERR_INVALID_ARG
    bad = list(args)
    bad[7] = FAKE + 8  # pos misaligned
    assert f(2, 2, 10, 128, 128, 16, L.LZ_BF16, *bad, 0) == L.LZ_ERR_INVALID_ARG
    bad = list(args)
    bad[2] = FAKE + 8  # lens misaligned
    assert f(2, 2, 10, 128, 128, 16, L.LZ_BF16, *bad, 0) == L.LZ_ERR_INVALID_ARG


def _call_hybrid_mse(lib, d, **ptrs):
    p = dict(q=FAKE, k=FAKE, v=FAKE, g=FAKE, mk=FAKE, mv=FAKE, h0=None, target=FAKE,
             o=FAKE, hT=None, lse=None, osw=None, loss=FAKE, dO=None, ws=FAKE)
    p.update(ptrs)
    return lib.lz_hybrid_fwd_mse(ctypes.byref(d), p["q"], p["k"], p["v"], p["g"], p["mk"],
                                 p["mv"], p["h0"], p["target"], p["o"], p["hT"], p["lse"],
                                 p["osw"], None, p["loss"], p["dO"], p["ws"],
                                 ptrs.get("ws_bytes", 1 << 40), 0)


@pytest.mark.parametrize("which", ["target", "loss", "o", "q"])
def test_stage1_loss_null_pointer_rejected(lib, which):
    assert _call_hybrid_mse(lib, _dims(), **{which: None}) == L.LZ_ERR_INVALID_ARG
    assert b"NULL" in lib.lz_last_error()


def test_stage1_loss_validation(lib):
    d = _dims(dk=128, dv=128)
    # the loss gradient may not overlap the output
    nbytes = d.B * d.H * d.T * d.dv * 2
    assert _call_hybrid_mse(lib, d, dO=FAKE + nbytes // 2) == L.LZ_ERR_INVALID_ARG
    assert b"overlap" in lib.lz_last_error()
    assert _call_hybrid_mse(lib, d, target=FAKE + 2) == L.LZ_ERR_INVALID_ARG
    # its scratch adds the partial sums to the forward's
    need = L.lz_workspace_bytes(d, L.LZ_WS_HYBRID_FWD_MSE)
    assert need > L.lz_workspace_bytes(d, L.LZ_WS_HYBRID_FWD)
    assert _call_hybrid_mse(lib, d, dO=FAKE + nbytes, ws_bytes=need - 1) == L.LZ_ERR_INVALID_ARG
    assert b"too small" in lib.lz_last_error()
    # empty problem: scratch of the partial sums only, no data pointers needed
    e = _dims(T=0)
    assert L.lz_workspace_bytes(e, L.LZ_WS_HYBRID_FWD_MSE) == 0


@pytest.mark.parametrize("kw,status", [
    (dict(gate_logits=1, io=L.LZ_F32, dk=128, dv=128), L.LZ_ERR_UNSUPPORTED),
    (dict(gate_logits=1, dk=64, dv=64), L.LZ_ERR_UNSUPPORTED),
    (dict(gate_logits=2, dk=128, dv=128), L.LZ_ERR_INVALID_ARG),
    (dict(gate_logits=1, dk=128, dv=128, gate_scale=0.0), L.LZ_ERR_INVALID_ARG),
    (dict(gate_logits=1, dk=128, dv=128, gate_scale=float("nan")), L.LZ_ERR_INVALID_ARG),
])
def test_gate_logits_validation(lib, kw, status):
    assert _call_hybrid(lib, _dims(**kw)) == status
    assert lib.lz_last_error()


def test_gate_logits_workspace(lib):
    """Gate logits take the two-level state pass for any length, so its
    scratch is there even for one chunk; every gated and hybrid workspace
    also holds the mapped fp32 log-gates (B*H*T*dk floats, 256-byte
    rounded), the window-only one does not."""
    d0 = _dims(dk=128, dv=128, T=64)
    d1 = _dims(dk=128, dv=128, T=64, gate_logits=1, gate_scale=0.0625)
    assert L.lz_workspace_bytes(d1, L.LZ_WS_HYBRID_FWD) > L.lz_workspace_bytes(d0, L.LZ_WS_HYBRID_FWD)
    e0 = _dims(dk=128, dv=128, T=300)
    e1 = _dims(dk=128, dv=128, T=300, gate_logits=1, gate_scale=0.0625)
    gates = (e1.B * e1.H * e1.T * e1.dk * 4 + 255) // 256 * 256
    for kind in (L.LZ_WS_GLA_FWD, L.LZ_WS_HYBRID_FWD, L.LZ_WS_HYBRID_FWD_MSE, L.LZ_WS_GLA_BWD,
                 L.LZ_WS_HYBRID_BWD):
        assert L.lz_workspace_bytes(e1, kind) - L.lz_workspace_bytes(e0, kind) == gates, kind
    for kind in (L.LZ_WS_SWA_BWD, L.LZ_WS_CHUNK_STATES):
        assert L.lz_workspace_bytes(e1, kind) == L.lz_workspace_bytes(e0, kind), kind


def test_binding_reads_bf16_gates_as_logits():
    """The helpers pass fp32 gates as log-gates and bf16 gates as logits."""
    import torch
    q = torch.zeros(1, 2, 8, 128, dtype=torch.bfloat16)
    v = torch.zeros(1, 2, 8, 128, dtype=torch.bfloat16)
    d = L._dims_from(q, v, chunk=64, w=4, M=0, scale=None, alpha=0.5,
                     g=torch.zeros(1, 2, 8, 128, dtype=torch.float32))
    assert d.gate_logits == 0
    d = L._dims_from(q, v, chunk=64, w=4, M=0, scale=None, alpha=0.5,
                     g=torch.zeros(1, 2, 8, 128, dtype=torch.bfloat16), gate_scale=0.25)
    assert d.gate_logits == 1 and abs(d.gate_scale - 0.25) < 1e-7
    assert L.lz_workspace_bytes(d, L.LZ_WS_HYBRID_BWD) > 0


def test_context_parallel_validation(lib):
    """The context-parallel calls refuse bad arguments before any launch."""
    assert lib.lz_cp_segment_decay(4, 16, 96, FAKE, FAKE, 0) == L.LZ_ERR_UNSUPPORTED
    assert lib.lz_cp_segment_decay(4, -1, 128, FAKE, FAKE, 0) == L.LZ_ERR_INVALID_ARG
    assert lib.lz_cp_segment_decay(4, 16, 128, FAKE + 4, FAKE, 0) == L.LZ_ERR_INVALID_ARG
    f = lib.lz_cp_fold
    assert f(2, 2, 0, 4, 128, 128, FAKE, FAKE, None, FAKE, 0) == L.LZ_ERR_INVALID_ARG  # r >= R
    assert f(2, 0, 2, 4, 128, 128, FAKE, FAKE, None, FAKE, 0) == L.LZ_ERR_INVALID_ARG  # dir
    assert f(2, 0, 0, 4, 128, 126, FAKE, FAKE, None, FAKE, 0) == L.LZ_ERR_UNSUPPORTED
    assert f(2, 1, 0, 4, 128, 128, FAKE, None, None, FAKE, 0) == L.LZ_ERR_INVALID_ARG
    assert b"NULL" in lib.lz_last_error()
    r = lib.lz_cp_rows
    # rows [10, 20) of a 15-row source
    assert r(4, 128, L.LZ_BF16, 10, FAKE, 15, 10, 1.0, None, 0, 0, FAKE, 64, 0, 0) == \
        L.LZ_ERR_INVALID_ARG
    assert b"outside" in lib.lz_last_error()
    assert r(4, 128, 7, 10, FAKE, 64, 0, 1.0, None, 0, 0, FAKE, 64, 0, 0) == L.LZ_ERR_UNSUPPORTED
    assert r(4, 128, L.LZ_BF16, 0, None, 0, 0, 1.0, None, 0, 0, FAKE, 64, 0, 0) == L.LZ_OK


def test_projection_validation(lib):
    """The projection refuses bad arguments before any launch."""
    f = lib.lz_qkg_projection
    ok = dict(B=2, T=8, Dm=256, H=2, dk=128)
    args = lambda **kw: [kw.get(n, ok[n]) for n in ("B", "T", "Dm", "H", "dk")]
    P = [FAKE, FAKE, FAKE, FAKE]  # x, Wq, Wk, Wg
    O = [FAKE, FAKE, FAKE]        # q, k, g
    assert f(*args(Dm=100), *P, ctypes.c_float(1.0), *O, 0) == L.LZ_ERR_UNSUPPORTED
    assert f(*args(dk=96), *P, ctypes.c_float(1.0), *O, 0) == L.LZ_ERR_UNSUPPORTED
    assert f(*args(H=1), *P, ctypes.c_float(1.0), *O, 0) == L.LZ_ERR_UNSUPPORTED  # H*dk = 128
    assert f(*args(), *P, ctypes.c_float(0.0), *O, 0) == L.LZ_ERR_INVALID_ARG
    assert f(*args(), FAKE, FAKE, None, FAKE, ctypes.c_float(1.0), *O, 0) == L.LZ_ERR_INVALID_ARG
    assert b"both" in lib.lz_last_error()
    assert f(*args(), FAKE + 8, FAKE, FAKE, FAKE, ctypes.c_float(1.0), *O, 0) == \
        L.LZ_ERR_INVALID_ARG
    assert f(*args(T=0), *P, ctypes.c_float(1.0), *O, 0) == L.LZ_OK



def test_kernel_choice_switches_are_per_thread(lib):
    """The per-thread switches (tcgen05 kernels, the gate-logit map) return
    the previous setting and leave other host threads' settings alone.  No
    device is touched."""
    import threading
    switches = (L.lz_prefer_tcgen05, L.lz_tcgen05_all, L.lz_fused_gate_logits)
    defaults = (True, False, False)
    for sw, dflt in zip(switches, defaults):
        assert sw(not dflt) == dflt
        assert sw(dflt) == (not dflt)
        assert sw(dflt) == dflt
    seen = {}

    def other():
        seen["other"] = [sw(d) for sw, d in zip(switches, defaults)]

    for sw, dflt in zip(switches, defaults):
        sw(not dflt)
    try:
        t = threading.Thread(target=other)
        t.start()
        t.join()
    finally:
        for sw, dflt in zip(switches, defaults):
            sw(dflt)
    assert seen["other"] == list(defaults)
