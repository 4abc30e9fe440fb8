"""Gate logits (the gate as sigma(z), z from the projection upstream): the
log-gate is scale * log sigma(z) and the backward returns dL/dz.  Both ways
the library takes them: one pass maps them to fp32 log-gates in the
workspace and one more maps dL/dg to dL/dz (the default), or every gated
kernel maps them as it loads them (lz_fused_gate_logits).  CUDA library
through the C ABI vs the fp64 oracle (the oracle's gate map, then its
operator and its chain rule)."""
import math

import numpy as np
import pytest
import torch

import gated_linear_sliding_chunked_b200 as L
import oracle
from parity_util import assert_close, np64, oracle_inputs, small_problem

pytestmark = pytest.mark.gpu

D = 128


@pytest.fixture(params=[False, True], ids=["mapped-once", "fused"], autouse=True)
def logits_mode(request):
    prev = L.lz_fused_gate_logits(request.param)
    yield request.param
    L.lz_fused_gate_logits(prev)


def _logits(seed, shape, mu, sigma):
    gen = torch.Generator().manual_seed(seed)
    return (torch.randn(*shape, generator=gen) * sigma + mu).to(torch.bfloat16)


def _case(seed, T, mu=2.0, sigma=1.0, s=1.0 / 16, h0=True):
    cpu, dev = small_problem(seed, 2, 2, T, D, D, 4, torch.bfloat16, train=True, h0=h0)
    z = _logits(seed + 7, (2, 2, T, D), mu, sigma)
    x = oracle_inputs(cpu, ("q", "k", "v", "meta_k", "meta_v", "dO", "h0", "dhT"))
    x["g"] = oracle.gate_from_logits(np64(z), s)
    return cpu, dev, z, x


@pytest.mark.parametrize("T", [1, 77, 333])
def test_hybrid_fwd_bwd_with_gate_logits(T):
    s, w, alpha = 1.0 / 16, 48, 0.6
    cpu, dev, z, x = _case(60 + T, T, s=s)
    zd = z.cuda()
    f = L.hybrid_fwd(dev["q"], dev["k"], dev["v"], zd, dev["meta_k"], dev["meta_v"], w=w,
                     alpha=alpha, h0=dev["h0"], gate_scale=s, want_hT=True, want_lse=True,
                     want_o_swa=True, want_chunk_states=True)
    b = L.hybrid_bwd(dev["q"], dev["k"], dev["v"], zd, dev["meta_k"], dev["meta_v"], f["lse"],
                     dev["dO"], w=w, alpha=alpha, h0=dev["h0"], dhT=dev["dhT"],
                     o_swa=f["o_swa"], chunk_states=f["chunk_states"], hT=f["hT"], gate_scale=s,
                     want_dh0=True)
    sc = 1 / math.sqrt(D)
    rf = oracle.hybrid_fwd(x["q"], x["k"], x["v"], x["g"], x["meta_k"], x["meta_v"], w, sc, alpha,
                           x["h0"])
    rb = oracle.hybrid_bwd(x["q"], x["k"], x["v"], x["g"], x["meta_k"], x["meta_v"], x["dO"], w, sc,
                           alpha, x["h0"], x["dhT"])
    assert_close("o", f["o"], rf["o"], torch.bfloat16)
    assert_close("hT", f["hT"], rf["hT"], torch.bfloat16)
    for name in ("dq", "dk", "dv", "dh0", "dmeta_k", "dmeta_v"):
        assert_close(name, b[name], rb[name], torch.bfloat16)
    assert_close("dz", b["dg"], oracle.dlogits(np64(z), rb["dg"], s), torch.bfloat16)
    L.lz_device_check()


def test_gate_logits_equal_the_log_gates_they_stand_for():
    """The same problem given as logits and as the fp32 log-gates they map
    to, through the same kernels (the warp-level ones: gates given as logits
    always take them): outputs and gradients agree to far below the bf16 bar,
    and dz is the chain rule applied to the log-gate run's dg."""
    s, w, alpha, T = 0.25, 64, 0.5, 300
    cpu, dev, z, x = _case(71, T, mu=1.0, sigma=1.5, s=s)
    zd = z.cuda()
    g32 = torch.from_numpy(x["g"]).float().cuda()
    out = {}
    prev = L.lz_prefer_tcgen05(False)
    try:
        for key, gate in (("z", zd), ("g", g32)):
            f = L.hybrid_fwd(dev["q"], dev["k"], dev["v"], gate, dev["meta_k"], dev["meta_v"],
                             w=w, alpha=alpha, h0=dev["h0"], gate_scale=s, want_hT=True,
                             want_lse=True)
            b = L.hybrid_bwd(dev["q"], dev["k"], dev["v"], gate, dev["meta_k"], dev["meta_v"],
                             f["lse"], dev["dO"], w=w, alpha=alpha, h0=dev["h0"],
                             dhT=dev["dhT"], gate_scale=s, want_dh0=True)
            out[key] = (f, b)
    finally:
        L.lz_prefer_tcgen05(prev)
    (fz, bz), (fg, bg) = out["z"], out["g"]
    for name in ("o", "hT"):
        assert_close(name, fz[name], np64(fg[name]), torch.bfloat16, factor=0.1)
    for name in ("dq", "dk", "dv", "dh0"):
        assert_close(name, bz[name], np64(bg[name]), torch.bfloat16, factor=0.1)
    assert_close("dz", bz["dg"], oracle.dlogits(np64(z), np64(bg["dg"]), s), torch.bfloat16,
                 factor=0.1)


def test_gla_fwd_bwd_with_gate_logits_strong_decay():
    """Fast forgetting from the logits (scale 1, z ~ N(-4, 2)): the gated
    kernels' elementwise-exponent paths read the gates through the same map."""
    s, T = 1.0, 130
    cpu, dev, z, x = _case(81, T, mu=-4.0, sigma=2.0, s=s)
    zd = z.cuda()
    o, hT, cs = L.gla_fwd(dev["q"], dev["k"], dev["v"], zd, dev["h0"], gate_scale=s, want_hT=True,
                          want_chunk_states=True)
    ro, rhT = oracle.gla_fwd(x["q"], x["k"], x["v"], x["g"], x["h0"])
    assert_close("o", o, ro, torch.bfloat16)
    assert_close("hT", hT, rhT, torch.bfloat16)
    for saved in (False, True):
        b = L.gla_bwd(dev["q"], dev["k"], dev["v"], zd, dev["dO"], dev["h0"], dev["dhT"],
                      chunk_states=cs if saved else None, hT=hT if saved else None, gate_scale=s,
                      want_dh0=True)
        rb = oracle.gla_bwd(x["q"], x["k"], x["v"], x["g"], x["dO"], x["h0"], x["dhT"])
        for name in ("dq", "dk", "dv", "dh0"):
            assert_close(f"{name} (saved={saved})", b[name], rb[name], torch.bfloat16)
    L.lz_device_check()


def test_gate_logits_empty_sequence_keeps_state():
    """T = 0 with gate logits: no chunk, hT = h0, dh0 = dhT."""
    cpu, dev, z, x = _case(91, 0)
    o, hT = L.gla_fwd(dev["q"], dev["k"], dev["v"], z.cuda(), dev["h0"], gate_scale=0.5,
                      want_hT=True)
    assert o.numel() == 0
    assert torch.equal(hT, dev["h0"])
    b = L.gla_bwd(dev["q"], dev["k"], dev["v"], z.cuda(), dev["dO"], dev["h0"], dev["dhT"],
                  gate_scale=0.5, want_dh0=True)
    assert torch.equal(b["dh0"], dev["dhT"])
