"""Forward parity: CUDA library (through the C ABI) vs the fp64 oracle.

Small problems span several chunks and key tiles with ragged tails; the
named workloads run at full size (or on sampled (batch, head) pairs, which
are independent problems, when the oracle would take too long)."""
import math

import numpy as np
import pytest
import torch

import gated_linear_sliding_chunked_b200 as L
from gated_linear_sliding_chunked_b200 import inputs as I
import oracle
from parity_util import TOL, assert_close, np64, oracle_inputs, small_problem

pytestmark = pytest.mark.gpu

DTYPES = [torch.float32, torch.bfloat16]


@pytest.mark.parametrize("dtype", DTYPES, ids=["f32", "bf16"])
@pytest.mark.parametrize("T,dk,dv", [(1, 64, 64), (15, 64, 64), (100, 128, 128),
                                     (257, 128, 64), (300, 64, 128)])
@pytest.mark.parametrize("with_h0", [False, True])
def test_gla_fwd(dtype, T, dk, dv, with_h0):
    cpu, dev = small_problem(1 + T, 2, 2, T, dk, dv, 0, dtype, h0=with_h0)
    o, hT = L.gla_fwd(dev["q"], dev["k"], dev["v"], dev["g"], dev.get("h0"), want_hT=True)
    x = oracle_inputs(cpu, ("q", "k", "v", "g", "h0"))
    ro, rhT = oracle.gla_fwd(x["q"], x["k"], x["v"], x["g"], x["h0"])
    assert_close("o", o, ro, dtype)
    assert_close("hT", hT, rhT, dtype)


@pytest.mark.parametrize("dtype", DTYPES, ids=["f32", "bf16"])
@pytest.mark.parametrize("T,w,M,sink", [(1, 1, 0, False), (40, 1, 3, False), (77, 7, 0, False),
                                        (130, 64, 4, False), (130, 64, 4, True),
                                        (200, 300, 0, False), (333, 128, 16, False)])
def test_swa_meta_fwd(dtype, T, w, M, sink):
    cpu, dev = small_problem(7 + T + w, 1, 3, T, 128, 128, M, dtype)
    mk = dev["meta_k"] if M else None
    mv = dev["meta_v"] if (M and not sink) else None
    o, lse = L.swa_meta_fwd(dev["q"], dev["k"], dev["v"], mk, mv, w=w)
    x = oracle_inputs(cpu, ("q", "k", "v", "meta_k", "meta_v"))
    ro, rl = oracle.swa_meta_fwd(x["q"], x["k"], x["v"], x["meta_k"] if M else None,
                                 x["meta_v"] if (M and not sink) else None, w,
                                 1.0 / math.sqrt(128))
    assert_close("o_swa", o, ro, dtype)
    assert_close("lse", lse, rl, torch.float32)


@pytest.mark.parametrize("dtype", DTYPES, ids=["f32", "bf16"])
@pytest.mark.parametrize("alpha", [0.0, 0.5, 2.0])
def test_hybrid_fwd(dtype, alpha):
    T, w, M = 190, 33, 5
    cpu, dev = small_problem(11, 2, 2, T, 128, 128, M, dtype, h0=True)
    res = L.hybrid_fwd(dev["q"], dev["k"], dev["v"], dev["g"], dev["meta_k"], dev["meta_v"],
                       w=w, alpha=alpha, h0=dev["h0"], want_hT=True, want_lse=True,
                       want_o_swa=True)
    x = oracle_inputs(cpu, ("q", "k", "v", "g", "meta_k", "meta_v", "h0"))
    ref = oracle.hybrid_fwd(x["q"], x["k"], x["v"], x["g"], x["meta_k"], x["meta_v"], w,
                            1 / math.sqrt(128), alpha, x["h0"])
    for name in ("o", "hT", "lse", "o_swa"):
        assert_close(name, res[name], ref[name], dtype if name in ("o", "o_swa") else
                     (dtype if name == "hT" else torch.float32))


@pytest.mark.parametrize("dtype,d", [(torch.float32, 64), (torch.bfloat16, 128)],
                         ids=["f32-d64", "bf16-d128"])
def test_gate_edge_cases(dtype, d):
    """g = 0 (no decay), g = -30 (full forgetting: the elementwise path), a
    mixture inside one chunk, and one decaying key dim among slow ones."""
    T = 150
    cpu, dev = small_problem(3, 1, 2, T, d, d, 0, dtype)
    for fill in (0.0, -30.0, "mixed", "one-dim"):
        g = torch.zeros(1, 2, T, d)
        if fill == "mixed":
            g[..., ::3, :] = -30.0
            g[..., 1::3, :] = -0.01
        elif fill == "one-dim":
            g[..., :] = -0.02
            g[..., 70:90, 5] = -9.0
        else:
            g.fill_(fill)
        o, hT = L.gla_fwd(dev["q"], dev["k"], dev["v"], g.cuda(), want_hT=True)
        ro, rhT = oracle.gla_fwd(np64(cpu["q"]), np64(cpu["k"]), np64(cpu["v"]), g.double().numpy())
        assert_close(f"o[g={fill}]", o, ro, dtype)
        assert_close(f"hT[g={fill}]", hT, rhT, dtype)


def test_empty_sequence_keeps_state():
    cpu, dev = small_problem(5, 1, 2, 0, 64, 64, 2, torch.float32, h0=True)
    res = L.hybrid_fwd(dev["q"], dev["k"], dev["v"], dev["g"], dev["meta_k"], dev["meta_v"],
                       w=4, alpha=0.5, h0=dev["h0"], want_hT=True)
    torch.cuda.synchronize()
    assert torch.equal(res["hT"].cpu(), cpu["h0"])


def test_determinism():
    cpu, dev = small_problem(9, 2, 2, 300, 128, 128, 4, torch.bfloat16)
    a = L.hybrid_fwd(dev["q"], dev["k"], dev["v"], dev["g"], dev["meta_k"], dev["meta_v"],
                     w=64, alpha=0.5)["o"]
    b = L.hybrid_fwd(dev["q"], dev["k"], dev["v"], dev["g"], dev["meta_k"], dev["meta_v"],
                     w=64, alpha=0.5)["o"]
    assert torch.equal(a, b)


# --------------------------------------------------------------------------
# named workloads
# --------------------------------------------------------------------------
def _run_workload(wl, pairs=None):
    x = I.make_inputs(wl, seed=0, device="cpu")
    dev = {k: v.cuda() for k, v in x.items()}
    res = L.hybrid_fwd(dev["q"], dev["k"], dev["v"], dev["g"], dev["meta_k"], dev["meta_v"],
                       w=wl.w, alpha=wl.alpha, chunk=wl.chunk, want_hT=True, want_lse=True)
    torch.cuda.synchronize()
    B, H = wl.B, wl.H
    if pairs is None:
        pairs = [(b, h) for b in range(B) for h in range(H)]
    for (b, h) in pairs:
        sl = lambda t: np64(t[b:b + 1, h:h + 1])
        ref = oracle.hybrid_fwd(sl(x["q"]), sl(x["k"]), sl(x["v"]), sl(x["g"]),
                                np64(x["meta_k"][h:h + 1]), np64(x["meta_v"][h:h + 1]), wl.w,
                                wl.scale, wl.alpha)
        dt = wl.torch_dtype
        assert_close(f"o[{b},{h}]", res["o"][b:b + 1, h:h + 1], ref["o"], dt)
        assert_close(f"hT[{b},{h}]", res["hT"][b:b + 1, h:h + 1], ref["hT"], dt)
        assert_close(f"lse[{b},{h}]", res["lse"][b:b + 1, h:h + 1], ref["lse"], torch.float32)


def test_workload_tiny_fp32_full():
    _run_workload(I.TINY_F32)


def test_workload_fwd_bf16_full():
    wl = I.FWD_BF16
    x = I.make_inputs(wl, seed=0, device="cpu")
    dev = {k: v.cuda() for k, v in x.items()}
    res = L.hybrid_fwd(dev["q"], dev["k"], dev["v"], dev["g"], dev["meta_k"], dev["meta_v"],
                       w=wl.w, alpha=wl.alpha, chunk=wl.chunk, want_hT=True, want_lse=True)
    xs = {k: np64(v) for k, v in x.items()}
    ref = oracle.hybrid_fwd(xs["q"], xs["k"], xs["v"], xs["g"], xs["meta_k"], xs["meta_v"],
                            wl.w, wl.scale, wl.alpha)
    assert_close("o", res["o"], ref["o"], torch.bfloat16)
    assert_close("hT", res["hT"], ref["hT"], torch.bfloat16)
    assert_close("lse", res["lse"], ref["lse"], torch.float32)


def test_workload_long_context_sampled():
    """T = 65536, strong forgetting: two sampled heads against the oracle."""
    _run_workload(I.LONG_BF16, pairs=[(0, 0), (0, 31)])


def test_window_forward_dispatch_and_device_status():
    """bf16, d = 128: the tcgen05 kernel by default for w <= 129, the
    warp-level one for wider windows or when asked for; no bounded device
    wait gives up."""
    cpu, dev = small_problem(21, 2, 2, 700, 128, 128, 8, torch.bfloat16)
    L.lz_timing_read()
    L.lz_timing_enable(True)
    prev = L.lz_prefer_tcgen05(True)
    try:
        for tc in (True, False):
            L.lz_prefer_tcgen05(tc)
            for w in (129, 300):
                L.swa_meta_fwd(dev["q"], dev["k"], dev["v"], dev["meta_k"], dev["meta_v"], w=w)
        names = [n for n, _ in L.lz_timing_read()]
    finally:
        L.lz_timing_enable(False)
        L.lz_prefer_tcgen05(prev)
    assert names == ["swa_fwd_tc", "swa_fwd_mma", "swa_fwd_mma", "swa_fwd_mma"], names
    L.lz_device_check()


def test_bounded_wait_failure_path_is_reported_and_device_stays_usable():
    """A bounded device wait that nothing completes (the library's self-test
    kernel) gives up, the status word reports it once, and the next kernels
    run and match the oracle."""
    L.lz_device_check()  # start from a clean word
    L.lz_selftest_bounded_wait()
    with pytest.raises(L.LzError) as err:
        L.lz_device_check()
    assert err.value.status == L.LZ_ERR_TIMEOUT
    L.lz_device_check()  # cleared by the read
    cpu, dev = small_problem(23, 1, 2, 150, 128, 128, 4, torch.bfloat16)
    res = L.hybrid_fwd(dev["q"], dev["k"], dev["v"], dev["g"], dev["meta_k"], dev["meta_v"],
                       w=64, alpha=0.5)
    x = oracle_inputs(cpu, ("q", "k", "v", "g", "meta_k", "meta_v"))
    ref = oracle.hybrid_fwd(x["q"], x["k"], x["v"], x["g"], x["meta_k"], x["meta_v"], 64,
                            1 / math.sqrt(128), 0.5)
    assert_close("o", res["o"], ref["o"], torch.bfloat16)
    L.lz_device_check()


@pytest.mark.parametrize("T,w,M,sink", [(1, 1, 0, False), (77, 7, 0, False), (130, 64, 4, True),
                                        (333, 128, 16, False), (700, 129, 8, False)])
@pytest.mark.parametrize("tc", [True, False], ids=["tcgen05", "warp-mma"])
def test_swa_meta_fwd_kernels(T, w, M, sink, tc):
    """Both bf16 window forwards against the oracle."""
    cpu, dev = small_problem(7 + T + w, 1, 3, T, 128, 128, M, torch.bfloat16)
    mk = dev["meta_k"] if M else None
    mv = dev["meta_v"] if (M and not sink) else None
    prev = L.lz_prefer_tcgen05(tc)
    try:
        o, lse = L.swa_meta_fwd(dev["q"], dev["k"], dev["v"], mk, mv, w=w)
    finally:
        L.lz_prefer_tcgen05(prev)
    L.lz_device_check()
    x = oracle_inputs(cpu, ("q", "k", "v", "meta_k", "meta_v"))
    ro, rl = oracle.swa_meta_fwd(x["q"], x["k"], x["v"], x["meta_k"] if M else None,
                                 x["meta_v"] if (M and not sink) else None, w,
                                 1.0 / math.sqrt(128))
    assert_close("o_swa", o, ro, torch.bfloat16)
    assert_close("lse", lse, rl, torch.float32)
