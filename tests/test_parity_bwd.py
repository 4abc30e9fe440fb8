"""Backward parity: every gradient of the CUDA library vs the fp64 oracle's
hand-written backward (itself pinned to finite differences)."""
import math

import numpy as np
import pytest
import torch

import gated_linear_sliding_chunked_b200 as L
from gated_linear_sliding_chunked_b200 import inputs as I
import oracle
from parity_util import assert_close, np64, oracle_inputs, small_problem

pytestmark = pytest.mark.gpu

DTYPES = [torch.float32, torch.bfloat16]


@pytest.mark.parametrize("dtype", DTYPES, ids=["f32", "bf16"])
@pytest.mark.parametrize("T,dk,dv", [(1, 64, 64), (37, 64, 64), (130, 128, 128),
                                     (200, 64, 128), (257, 128, 64)])
@pytest.mark.parametrize("with_state", [False, True])
@pytest.mark.parametrize("saved", [False, True], ids=["state-pass", "saved-states"])
def test_gla_bwd(dtype, T, dk, dv, with_state, saved):
    """saved: the backward gets the forward's chunk states and final state
    (used by the bf16 d = 128 kernels, ignored elsewhere)."""
    cpu, dev = small_problem(20 + T, 2, 2, T, dk, dv, 0, dtype, train=True, h0=with_state)
    dhT = dev["dhT"] if with_state else None
    cs = hT = None
    if saved:
        _, hT, cs = L.gla_fwd(dev["q"], dev["k"], dev["v"], dev["g"], dev.get("h0"),
                              want_hT=True, want_chunk_states=True)
    res = L.gla_bwd(dev["q"], dev["k"], dev["v"], dev["g"], dev["dO"], dev.get("h0"), dhT,
                    chunk_states=cs, hT=hT, want_dh0=True)
    x = oracle_inputs(cpu, ("q", "k", "v", "g", "dO", "h0", "dhT"))
    ref = oracle.gla_bwd(x["q"], x["k"], x["v"], x["g"], x["dO"], x["h0"],
                         x["dhT"] if with_state else None)
    for name in ("dq", "dk", "dv", "dg", "dh0"):
        assert_close(name, res[name], ref[name], dtype)


@pytest.mark.parametrize("dtype", DTYPES, ids=["f32", "bf16"])
@pytest.mark.parametrize("T,w,M,sink", [(1, 1, 2, False), (50, 1, 0, False),
                                        (130, 33, 4, False), (130, 33, 4, True),
                                        (150, 200, 0, False), (290, 128, 16, False),
                                        (1100, 128, 8, False)])
@pytest.mark.parametrize("with_o", [False, True], ids=["rebuild-D", "saved-o"])
def test_swa_meta_bwd(dtype, T, w, M, sink, with_o):
    """with_o: the forward output is passed, so D = dO . o comes off it."""
    cpu, dev = small_problem(40 + T + w, 2, 2, T, 128, 128, M, dtype, train=True)
    mk = dev["meta_k"] if M else None
    mv = dev["meta_v"] if (M and not sink) else None
    o, lse = L.swa_meta_fwd(dev["q"], dev["k"], dev["v"], mk, mv, w=w)
    res = L.swa_meta_bwd(dev["q"], dev["k"], dev["v"], mk, mv, lse, dev["dO"], w=w,
                         o=o if with_o else None)
    x = oracle_inputs(cpu, ("q", "k", "v", "meta_k", "meta_v", "dO"))
    ref = oracle.swa_meta_bwd(x["q"], x["k"], x["v"], x["meta_k"] if M else None,
                              x["meta_v"] if (M and not sink) else None, x["dO"], w,
                              1 / math.sqrt(128))
    for name in ("dq", "dk", "dv"):
        assert_close(name, res[name], ref[name], dtype)
    if M:
        assert_close("dmeta_k", res["dmeta_k"], ref["dmeta_k"], dtype)
        if not sink:
            assert_close("dmeta_v", res["dmeta_v"], ref["dmeta_v"], dtype)


@pytest.mark.parametrize("T,w,M", [(1, 1, 2), (300, 64, 4), (1100, 128, 8), (260, 700, 0),
                                   (513, 129, 16), (700, 33, 0)])
@pytest.mark.parametrize("mode", ["tcgen05", "warp-mma", "tcgen05-all"])
def test_swa_meta_bwd_kernels(T, w, M, mode):
    """The bf16 window-backward kernels against the oracle: the key side on
    tcgen05 (default) or warp-level, and with lz_tcgen05_all also the query
    side on tcgen05 (w <= 129); a clean device status word afterwards."""
    cpu, dev = small_problem(90 + T + w, 2, 2, T, 128, 128, M, torch.bfloat16, train=True)
    mk = dev["meta_k"] if M else None
    mv = dev["meta_v"] if M else None
    prev = L.lz_prefer_tcgen05(mode != "warp-mma")
    prev_all = L.lz_tcgen05_all(mode == "tcgen05-all")
    try:
        o, lse = L.swa_meta_fwd(dev["q"], dev["k"], dev["v"], mk, mv, w=w)
        L.lz_timing_enable(True)
        res = L.swa_meta_bwd(dev["q"], dev["k"], dev["v"], mk, mv, lse, dev["dO"], w=w, o=o)
        torch.cuda.synchronize()
    finally:
        L.lz_timing_enable(False)
        L.lz_prefer_tcgen05(prev)
        L.lz_tcgen05_all(prev_all)
    ran = {name for name, _ in L.lz_timing_read()}
    if T > 0:
        assert ("swa_bwd_q_tc" in ran) == (mode == "tcgen05-all" and w <= 129), ran
    L.lz_device_check()
    x = oracle_inputs(cpu, ("q", "k", "v", "meta_k", "meta_v", "dO"))
    ref = oracle.swa_meta_bwd(x["q"], x["k"], x["v"], x["meta_k"] if M else None,
                              x["meta_v"] if M else None, x["dO"], w, 1 / math.sqrt(128))
    for name in ("dq", "dk", "dv") + (("dmeta_k", "dmeta_v") if M else ()):
        assert_close(name, res[name], ref[name], torch.bfloat16)


@pytest.mark.parametrize("dtype", DTYPES, ids=["f32", "bf16"])
@pytest.mark.parametrize("alpha", [0.0, 0.5, 2.0])
@pytest.mark.parametrize("saved", ["none", "o_swa", "all"])
def test_hybrid_bwd(dtype, alpha, saved):
    """saved: which forward results the backward gets (window output; also
    the gated chunk states and final state)."""
    T, w, M = 210, 40, 6
    cpu, dev = small_problem(77, 2, 2, T, 128, 128, M, dtype, train=True, h0=True)
    fwd = L.hybrid_fwd(dev["q"], dev["k"], dev["v"], dev["g"], dev["meta_k"], dev["meta_v"],
                       w=w, alpha=alpha, h0=dev["h0"], want_lse=True, want_o_swa=saved != "none",
                       want_hT=saved == "all", want_chunk_states=saved == "all")
    res = L.hybrid_bwd(dev["q"], dev["k"], dev["v"], dev["g"], dev["meta_k"], dev["meta_v"],
                       fwd["lse"], dev["dO"], w=w, alpha=alpha, h0=dev["h0"], dhT=dev["dhT"],
                       o_swa=fwd["o_swa"], chunk_states=fwd["chunk_states"], hT=fwd["hT"],
                       want_dh0=True)
    x = oracle_inputs(cpu, ("q", "k", "v", "g", "meta_k", "meta_v", "dO", "h0", "dhT"))
    ref = oracle.hybrid_bwd(x["q"], x["k"], x["v"], x["g"], x["meta_k"], x["meta_v"], x["dO"], w,
                            1 / math.sqrt(128), alpha, x["h0"], x["dhT"])
    for name in ("dq", "dk", "dv", "dg", "dh0", "dmeta_k", "dmeta_v"):
        assert_close(name, res[name], ref[name], dtype)
    assert_close("dalpha", res["dalpha"].cpu().double().numpy(), np.array([ref["dalpha"]]), dtype)


def test_launch_timing_filter():
    """lz_timing_only narrows the launch timing to one kernel name; None
    restores timing of every launch."""
    cpu, dev = small_problem(41, 2, 2, 200, 128, 128, 0, torch.bfloat16, train=True)
    L.lz_timing_read()
    runs = {}
    for only in ("gla_bwd_chunks", None):
        L.lz_timing_only(only)
        L.lz_timing_enable(True)
        try:
            L.gla_bwd(dev["q"], dev["k"], dev["v"], dev["g"], dev["dO"])
            torch.cuda.synchronize()
        finally:
            L.lz_timing_enable(False)
            L.lz_timing_only(None)
        runs[only] = [name for name, _ in L.lz_timing_read()]
    assert runs["gla_bwd_chunks"] == ["gla_bwd_chunks"], runs
    assert "gla_bwd_chunks" in runs[None] and len(set(runs[None])) > 1, runs
    L.lz_device_check()


@pytest.mark.parametrize("T", [1, 64, 128, 129, 300, 700])
@pytest.mark.parametrize("tc", [True, False], ids=["tcgen05", "warp-mma"])
def test_gla_bwd_kernels(T, tc):
    """Both bf16 per-chunk backward kernels (tcgen05 over 128-token chunks and
    warp-level over 64-token chunks) against the oracle, with the kernel that
    ran named by the library's launch timing and a clean status word."""
    cpu, dev = small_problem(300 + T, 2, 2, T, 128, 128, 0, torch.bfloat16, train=True, h0=True)
    prev = L.lz_tcgen05_all(tc)
    L.lz_timing_enable(True)
    try:
        res = L.gla_bwd(dev["q"], dev["k"], dev["v"], dev["g"], dev["dO"], dev["h0"], dev["dhT"],
                        want_dh0=True)
        torch.cuda.synchronize()
    finally:
        L.lz_timing_enable(False)
        L.lz_tcgen05_all(prev)
    ran = {name for name, _ in L.lz_timing_read()}
    assert ("gla_bwd_chunks_tc" in ran) == tc, ran
    L.lz_device_check()
    x = oracle_inputs(cpu, ("q", "k", "v", "g", "dO", "h0", "dhT"))
    ref = oracle.gla_bwd(x["q"], x["k"], x["v"], x["g"], x["dO"], x["h0"], x["dhT"])
    for name in ("dq", "dk", "dv", "dg", "dh0"):
        assert_close(name, res[name], ref[name], torch.bfloat16)


def test_gla_bwd_full_forgetting():
    """g = -30 everywhere: the elementwise-exponent path of the backward."""
    cpu, dev = small_problem(3, 1, 2, 45, 64, 64, 0, torch.float32, train=True)
    g = torch.full((1, 2, 45, 64), -30.0)
    g[..., ::2, :] = -0.05
    res = L.gla_bwd(dev["q"], dev["k"], dev["v"], g.cuda(), dev["dO"])
    x = oracle_inputs(cpu, ("q", "k", "v", "dO"))
    ref = oracle.gla_bwd(x["q"], x["k"], x["v"], g.double().numpy(), x["dO"])
    for name in ("dq", "dk", "dv", "dg"):
        assert_close(name, res[name], ref[name], torch.float32)


@pytest.mark.parametrize("tc", [False, True], ids=["warp-mma", "tcgen05"])
@pytest.mark.parametrize("fill", [0.0, -30.0, "mixed", "one-dim", "strong"])
def test_gla_bwd_gate_edge_cases_bf16(fill, tc):
    """The tensor-core backward's gate paths (bf16, d = 128): g = 0 (no
    decay), g = -30 (full forgetting: elementwise diagonal blocks), a mixture
    inside each chunk, one fast-decaying key dim among slow ones (per-pair
    sub-block factors), and the long-context distribution logsigmoid(N(-1,
    1.5)) with no /16.  Every gradient, dg included, meets the plain
    relative-L2 bar in every regime (dg's in-chunk running sum cancels
    exactly in the kernel, so fast forgetting does not amplify rounding)."""
    T = 200
    cpu, dev = small_problem(31, 1, 2, T, 128, 128, 0, torch.bfloat16, train=True, h0=True)
    gen = torch.Generator().manual_seed(5)
    if fill == "mixed":
        g = torch.full((1, 2, T, 128), -0.01)
        g[..., ::3, :] = -30.0
    elif fill == "one-dim":
        g = torch.full((1, 2, T, 128), -0.02)
        g[..., 70:90, 5] = -9.0
    elif fill == "strong":
        g = torch.nn.functional.logsigmoid(torch.randn(1, 2, T, 128, generator=gen) * 1.5 - 1.0)
    else:
        g = torch.full((1, 2, T, 128), float(fill))
    prev = L.lz_tcgen05_all(tc)  # tcgen05: the fast-decaying chunks fall back
    try:
        res = L.gla_bwd(dev["q"], dev["k"], dev["v"], g.cuda(), dev["dO"], dev["h0"], dev["dhT"],
                        want_dh0=True)
    finally:
        L.lz_tcgen05_all(prev)
    x = oracle_inputs(cpu, ("q", "k", "v", "dO", "h0", "dhT"))
    ref = oracle.gla_bwd(x["q"], x["k"], x["v"], g.double().numpy(), x["dO"], x["h0"], x["dhT"])
    for name in ("dq", "dk", "dv", "dh0", "dg"):
        assert_close(f"{name}[g={fill}]", res[name], ref[name], torch.bfloat16)


def test_gla_bwd_long_context_gates_full_length():
    """One head over the long-context workload's whole length (T = 65536)
    with its fast-forgetting gates logsigmoid(N(-1, 1.5)) and a synthetic
    dO ~ N(0, 1): every gradient of the bf16 tensor-core backward, dg with
    the plain relative-L2 bar."""
    wl = I.LONG_BF16.with_(H=1, M=0, train=True)
    x = I.make_inputs(wl, seed=3, device="cpu")
    dev = {k: v.cuda() for k, v in x.items()}
    res = L.gla_bwd(dev["q"], dev["k"], dev["v"], dev["g"], dev["dO"])
    xs = {k: np64(v) for k, v in x.items()}
    ref = oracle.gla_bwd(xs["q"], xs["k"], xs["v"], xs["g"], xs["dO"])
    for name in ("dq", "dk", "dv", "dg"):
        assert_close(f"{name}[T=65536]", res[name], ref[name], torch.bfloat16)


@pytest.mark.parametrize("T,w,M,sink", [(1, 1, 2, False), (64, 64, 0, False), (127, 129, 8, False),
                                         (129, 33, 3, True), (300, 128, 16, False),
                                         (700, 100, 4, True), (300, 130, 4, False),
                                         (260, 300, 2, False)])
@pytest.mark.parametrize("states", [False, True], ids=["no-states", "chunk-states"])
def test_hybrid_bwd_split_query_side(T, w, M, sink, states):
    """bf16 hybrid backward given the window output: the query side keeps D
    and the meta terms, the tcgen05 key side stores its dS tiles and dq is
    formed from them (swa_bwd_dq), for ragged lengths, windows up to 129
    keys, sink-only meta tokens and none; wider windows take the unsplit
    query side.  With and without the forward's chunk states (the gated
    first level then skips its own state pass).  Run twice, bit-identical."""
    alpha = 0.7
    cpu, dev = small_problem(500 + T + w, 2, 2, T, 128, 128, M, torch.bfloat16, train=True)
    mk = dev["meta_k"] if M else None
    mv = dev["meta_v"] if (M and not sink) else None
    fwd = L.hybrid_fwd(dev["q"], dev["k"], dev["v"], dev["g"], mk, mv, w=w, alpha=alpha,
                       want_lse=True, want_o_swa=True, want_chunk_states=states)
    L.lz_timing_read()
    L.lz_timing_enable(True)
    try:
        runs = [L.hybrid_bwd(dev["q"], dev["k"], dev["v"], dev["g"], mk, mv, fwd["lse"],
                             dev["dO"], w=w, alpha=alpha, o_swa=fwd["o_swa"],
                             chunk_states=fwd["chunk_states"]) for _ in range(2)]
        torch.cuda.synchronize()
    finally:
        L.lz_timing_enable(False)
    ran = {name for name, _ in L.lz_timing_read()}
    if w <= 129:
        assert {"swa_bwd_meta", "swa_bwd_kv_tc", "swa_bwd_dq"} <= ran, ran
        assert "swa_bwd_q_mma" not in ran, ran
    else:
        assert "swa_bwd_q_mma" in ran and not {"swa_bwd_meta", "swa_bwd_dq"} & ran, ran
    L.lz_device_check()
    x = oracle_inputs(cpu, ("q", "k", "v", "g", "meta_k", "meta_v", "dO"))
    ref = oracle.hybrid_bwd(x["q"], x["k"], x["v"], x["g"], x["meta_k"] if M else None,
                            x["meta_v"] if (M and not sink) else None, x["dO"], w,
                            1 / math.sqrt(128), alpha)
    res = runs[0]
    for name in ("dq", "dk", "dv", "dg"):
        assert_close(name, res[name], ref[name], torch.bfloat16)
    if M > 0:
        assert_close("dmeta_k", res["dmeta_k"], ref["dmeta_k"], torch.bfloat16)
        if not sink:
            assert_close("dmeta_v", res["dmeta_v"], ref["dmeta_v"], torch.bfloat16)
    assert_close("dalpha", res["dalpha"].cpu().double().numpy(), np.array([ref["dalpha"]]),
                 torch.bfloat16)
    for name in ("dq", "dk", "dv", "dg", "dmeta_k", "dmeta_v", "dalpha"):
        if runs[0].get(name) is not None:
            assert torch.equal(runs[0][name], runs[1][name]), name


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 64)], ids=["bf16", "f32"])
@pytest.mark.parametrize("B,T", [(2, 0), (0, 70)], ids=["no-tokens", "no-sequences"])
def test_hybrid_empty_inputs(dtype, d, B, T):
    """Degenerate shapes through the forward and the backward.  With no
    tokens the state passes through unchanged both ways (hT = h0, dh0 =
    dhT), and with either no tokens or no sequences the meta-token gradients
    and dalpha are exactly zero (the outputs start as uninitialised memory,
    so the library must write them)."""
    H, M = 2, 4
    cpu, dev = small_problem(61 + T, B, H, T, d, d, M, dtype, train=True, h0=True)
    bf = dtype == torch.bfloat16
    f = L.hybrid_fwd(dev["q"], dev["k"], dev["v"], dev["g"], dev["meta_k"], dev["meta_v"], w=16,
                     alpha=0.5, h0=dev["h0"], want_hT=True, want_lse=True, want_o_swa=bf,
                     want_chunk_states=bf)
    b = None
    for _ in range(2):
        if b is not None:  # NaN-filled and freed: the next call's outputs reuse these blocks
            for t in (b["dmeta_k"], b["dmeta_v"], b["dalpha"]):
                t.fill_(float("nan"))
            torch.cuda.synchronize()
            del b
        b = L.hybrid_bwd(dev["q"], dev["k"], dev["v"], dev["g"], dev["meta_k"], dev["meta_v"],
                         f["lse"], dev["dO"], w=16, alpha=0.5, h0=dev["h0"], dhT=dev["dhT"],
                         o_swa=f["o_swa"], chunk_states=f["chunk_states"], want_dh0=True)
        L.lz_device_check()
        assert f["o"].numel() == 0 and f["hT"].shape == (B, H, d, d)
        for name in ("dq", "dk", "dv", "dg"):
            assert b[name].numel() == 0, name
        if B:
            assert torch.equal(f["hT"].cpu(), cpu["h0"])
            assert torch.equal(b["dh0"].cpu(), cpu["dhT"])
        assert torch.equal(b["dmeta_k"].cpu(), torch.zeros(H, M, d))
        assert torch.equal(b["dmeta_v"].cpu(), torch.zeros(H, M, d))
        assert float(b["dalpha"].item()) == 0.0


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 64)], ids=["bf16", "f32"])
def test_hybrid_max_window_and_meta(dtype, d):
    """The largest window the library takes (w = 1024) and the most meta
    tokens (M = 16), at a ragged length past the window: forward and every
    gradient against the oracle."""
    T, w, M, alpha = 1100, 1024, 16, 0.8
    cpu, dev = small_problem(1100 + d, 1, 2, T, d, d, M, dtype, train=True, h0=True)
    f = L.hybrid_fwd(dev["q"], dev["k"], dev["v"], dev["g"], dev["meta_k"], dev["meta_v"], w=w,
                     alpha=alpha, h0=dev["h0"], want_hT=True, want_lse=True)
    b = L.hybrid_bwd(dev["q"], dev["k"], dev["v"], dev["g"], dev["meta_k"], dev["meta_v"],
                     f["lse"], dev["dO"], w=w, alpha=alpha, h0=dev["h0"], dhT=dev["dhT"],
                     want_dh0=True)
    L.lz_device_check()
    x = oracle_inputs(cpu, ("q", "k", "v", "g", "meta_k", "meta_v", "dO", "h0", "dhT"))
    sc = 1 / math.sqrt(d)
    rf = oracle.hybrid_fwd(x["q"], x["k"], x["v"], x["g"], x["meta_k"], x["meta_v"], w, sc,
                           alpha, x["h0"])
    rb = oracle.hybrid_bwd(x["q"], x["k"], x["v"], x["g"], x["meta_k"], x["meta_v"], x["dO"], w,
                           sc, alpha, x["h0"], x["dhT"])
    assert_close("o", f["o"], rf["o"], dtype)
    assert_close("hT", f["hT"], rf["hT"], dtype)
    for name in ("dq", "dk", "dv", "dg", "dh0", "dmeta_k", "dmeta_v"):
        assert_close(name, b[name], rb[name], dtype)
    assert_close("dalpha", b["dalpha"].cpu().double().numpy(), np.array([rb["dalpha"]]), dtype)


def test_bwd_determinism():
    cpu, dev = small_problem(8, 2, 2, 300, 128, 128, 4, torch.bfloat16, train=True)
    fwd = L.hybrid_fwd(dev["q"], dev["k"], dev["v"], dev["g"], dev["meta_k"], dev["meta_v"],
                       w=64, alpha=0.5, want_lse=True)
    runs = [L.hybrid_bwd(dev["q"], dev["k"], dev["v"], dev["g"], dev["meta_k"], dev["meta_v"],
                         fwd["lse"], dev["dO"], w=64, alpha=0.5) for _ in range(2)]
    for name in ("dq", "dk", "dv", "dg", "dmeta_k", "dmeta_v", "dalpha"):
        assert torch.equal(runs[0][name], runs[1][name]), name


@pytest.mark.parametrize("tc", [False, True], ids=["warp-mma", "tcgen05"])
def test_workload_train_sampled(tc):
    """Llama-3-8B-shaped training layer (B=2, H=32, T=8192): fwd + bwd at full
    size on the GPU; every per-token gradient checked on sampled heads, meta
    gradients for one head exactly (both batch rows), dalpha over all heads.
    tc: the gated backward's per-chunk gradients on the tcgen05 kernel."""
    wl = I.TRAIN_BF16
    x = I.make_inputs(wl, seed=0, device="cpu")
    dev = {k: v.cuda() for k, v in x.items()}
    fwd = L.hybrid_fwd(dev["q"], dev["k"], dev["v"], dev["g"], dev["meta_k"], dev["meta_v"],
                       w=wl.w, alpha=wl.alpha, chunk=wl.chunk, want_lse=True, want_o_swa=True,
                       want_chunk_states=True)
    prev = L.lz_tcgen05_all(tc)
    try:
        res = L.hybrid_bwd(dev["q"], dev["k"], dev["v"], dev["g"], dev["meta_k"], dev["meta_v"],
                           fwd["lse"], dev["dO"], w=wl.w, alpha=wl.alpha, chunk=wl.chunk,
                           o_swa=fwd["o_swa"], chunk_states=fwd["chunk_states"])
    finally:
        L.lz_tcgen05_all(prev)
    torch.cuda.synchronize()
    L.lz_device_check()
    h = 5
    for b in range(wl.B):
        sl = lambda t: np64(t[b:b + 1, h:h + 1])
        ref = oracle.hybrid_bwd(sl(x["q"]), sl(x["k"]), sl(x["v"]), sl(x["g"]),
                                np64(x["meta_k"][h:h + 1]), np64(x["meta_v"][h:h + 1]),
                                sl(x["dO"]), wl.w, wl.scale, wl.alpha)
        for name in ("dq", "dk", "dv", "dg"):
            assert_close(f"{name}[{b},{h}]", res[name][b:b + 1, h:h + 1], ref[name],
                         torch.bfloat16)
        if b == 0:
            mk_acc, mv_acc = ref["dmeta_k"].copy(), ref["dmeta_v"].copy()
        else:
            mk_acc += ref["dmeta_k"]
            mv_acc += ref["dmeta_v"]
    assert_close("dmeta_k[h]", res["dmeta_k"][h:h + 1], mk_acc, torch.bfloat16)
    assert_close("dmeta_v[h]", res["dmeta_v"][h:h + 1], mv_acc, torch.bfloat16)
    # dalpha = sum over every (b, h, t) of dO . o_swa, with o_swa from the oracle
    xs = {k: np64(v) for k, v in x.items() if k in ("q", "k", "v", "meta_k", "meta_v", "dO")}
    o_swa, _ = oracle.swa_meta_fwd(xs["q"], xs["k"], xs["v"], xs["meta_k"], xs["meta_v"], wl.w,
                                   wl.scale)
    dal = float(np.sum(xs["dO"] * o_swa))
    assert_close("dalpha", res["dalpha"].cpu().double().numpy(), np.array([dal]),
                 torch.bfloat16)


def test_training_step_under_cuda_graph():
    """The forward + backward step (whose gated passes fork onto the library's
    side stream and join back) captured into a CUDA graph and replayed gives
    the eager results bit for bit."""
    cpu, dev = small_problem(55, 2, 2, 333, 128, 128, 4, torch.bfloat16, train=True, h0=True)

    def step():
        f = L.hybrid_fwd(dev["q"], dev["k"], dev["v"], dev["g"], dev["meta_k"], dev["meta_v"],
                         w=64, alpha=0.5, h0=dev["h0"], want_hT=True, want_lse=True,
                         want_o_swa=True, want_chunk_states=True)
        b = L.hybrid_bwd(dev["q"], dev["k"], dev["v"], dev["g"], dev["meta_k"], dev["meta_v"],
                         f["lse"], dev["dO"], w=64, alpha=0.5, h0=dev["h0"], dhT=dev["dhT"],
                         o_swa=f["o_swa"], chunk_states=f["chunk_states"], hT=f["hT"],
                         want_dh0=True)
        return f, b

    f0, b0 = step()
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        f1, b1 = step()
    graph.replay()
    torch.cuda.synchronize()
    for name in ("o", "hT", "lse", "o_swa"):
        assert torch.equal(f1[name], f0[name]), name
    for name in ("dq", "dk", "dv", "dg", "dh0", "dmeta_k", "dmeta_v", "dalpha"):
        assert torch.equal(b1[name], b0[name]), name
    L.lz_device_check()
