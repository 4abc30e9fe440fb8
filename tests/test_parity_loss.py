"""Stage-1 distillation loss (mean squared error between the hybrid output and
a teacher's attention output) and its gradient: CUDA library through the C
ABI vs the fp64 oracle, then the whole stage-1 step (forward, loss, backward
fed with the loss gradient)."""
import math

import numpy as np
import pytest
import torch

import gated_linear_sliding_chunked_b200 as L
import oracle
from parity_util import TOL, assert_close, np64, oracle_inputs, small_problem

pytestmark = pytest.mark.gpu


def _teacher(seed, shape, dtype):
    """Synthetic stand-in for the teacher's attention output."""
    gen = torch.Generator().manual_seed(seed)
    return (torch.randn(*shape, generator=gen) * 0.5).to(dtype)


def _run(dtype, B, H, T, d, w, M, alpha, seed):
    cpu, dev = small_problem(seed, B, H, T, d, d, M, dtype, h0=True)
    tgt = _teacher(seed + 1, (B, H, T, d), dtype)
    res = L.hybrid_fwd_mse(dev["q"], dev["k"], dev["v"], dev["g"], dev["meta_k"],
                           dev["meta_v"], tgt.cuda(), w=w, alpha=alpha, h0=dev["h0"],
                           want_lse=True)
    x = oracle_inputs(cpu, ("q", "k", "v", "g", "meta_k", "meta_v", "h0"))
    ref = oracle.hybrid_fwd(x["q"], x["k"], x["v"], x["g"], x["meta_k"], x["meta_v"], w,
                            1 / math.sqrt(d), alpha, x["h0"])
    rloss, rdO = oracle.mse_loss(ref["o"], np64(tgt))
    return cpu, dev, tgt, res, ref, rloss, rdO


@pytest.mark.parametrize("dtype,d", [(torch.float32, 64), (torch.bfloat16, 64),
                                     (torch.bfloat16, 128), (torch.float32, 128)],
                         ids=["f32-d64", "bf16-d64", "bf16-d128-fused", "f32-d128"])
@pytest.mark.parametrize("T", [1, 77, 333])
def test_stage1_loss(dtype, d, T):
    _, _, _, res, ref, rloss, rdO = _run(dtype, 2, 2, T, d, 40, 4, 0.7, 300 + T + d)
    assert_close("o", res["o"], ref["o"], dtype)
    got = float(res["loss"].cpu())
    assert abs(got - rloss) <= TOL[dtype] * abs(rloss), (got, rloss)
    assert_close("dO", res["dO"], rdO, dtype)


def test_stage1_loss_reproducible_and_optional_gradient():
    args = (torch.bfloat16, 2, 4, 700, 128, 64, 8, 0.5, 5)
    _, dev, tgt, a, _, _, _ = _run(*args)
    _, _, _, b, _, _, _ = _run(*args)
    assert torch.equal(a["loss"], b["loss"]) and torch.equal(a["dO"], b["dO"])
    c = L.hybrid_fwd_mse(dev["q"], dev["k"], dev["v"], dev["g"], dev["meta_k"], dev["meta_v"],
                         tgt.cuda(), w=64, alpha=0.5, h0=dev["h0"], want_dO=False)
    assert c["dO"] is None and torch.equal(c["loss"], a["loss"])
    assert torch.equal(c["o"], a["o"])
    # the plain forward gives the same output
    p = L.hybrid_fwd(dev["q"], dev["k"], dev["v"], dev["g"], dev["meta_k"], dev["meta_v"],
                     w=64, alpha=0.5, h0=dev["h0"])
    assert torch.equal(p["o"], a["o"])


def test_stage1_loss_target_equals_output():
    """A teacher output equal to the stored output: the loss is the rounding
    of the output alone (bf16: at most (2^-8)^2 of its mean square) and the
    fp32 path gives exactly 0."""
    for dtype, d in ((torch.float32, 64), (torch.bfloat16, 128)):
        cpu, dev = small_problem(9, 1, 2, 150, d, d, 4, dtype)
        o = L.hybrid_fwd(dev["q"], dev["k"], dev["v"], dev["g"], dev["meta_k"], dev["meta_v"],
                         w=32, alpha=1.0)["o"]
        res = L.hybrid_fwd_mse(dev["q"], dev["k"], dev["v"], dev["g"], dev["meta_k"],
                               dev["meta_v"], o.clone(), w=32, alpha=1.0)
        ms = float((o.double() ** 2).mean())
        got = float(res["loss"].cpu())
        if dtype == torch.float32:
            assert got == 0.0 and not torch.any(res["dO"])
        else:
            assert 0.0 <= got <= ms * 2.0 ** -16 * 1.01


def test_stage1_loss_empty():
    cpu, dev = small_problem(1, 1, 2, 0, 128, 128, 4, torch.bfloat16)
    res = L.hybrid_fwd_mse(dev["q"], dev["k"], dev["v"], dev["g"], dev["meta_k"],
                           dev["meta_v"], torch.empty_like(dev["v"]), w=16, alpha=1.0)
    assert float(res["loss"].cpu()) == 0.0


@pytest.mark.parametrize("dtype,d", [(torch.float32, 64), (torch.bfloat16, 128)],
                         ids=["f32-d64", "bf16-d128"])
def test_stage1_step(dtype, d):
    """Forward, loss, and the backward fed with the loss gradient: every
    operator gradient vs the oracle's composed step."""
    T, w, M, alpha = 210, 48, 6, 0.8
    cpu, dev = small_problem(41, 2, 2, T, d, d, M, dtype, h0=True)
    tgt = _teacher(42, (2, 2, T, d), dtype)
    fwd = L.hybrid_fwd_mse(dev["q"], dev["k"], dev["v"], dev["g"], dev["meta_k"],
                           dev["meta_v"], tgt.cuda(), w=w, alpha=alpha, h0=dev["h0"],
                           want_lse=True, want_o_swa=True, want_hT=True, want_chunk_states=True)
    res = L.hybrid_bwd(dev["q"], dev["k"], dev["v"], dev["g"], dev["meta_k"], dev["meta_v"],
                       fwd["lse"], fwd["dO"], w=w, alpha=alpha, h0=dev["h0"],
                       o_swa=fwd["o_swa"], chunk_states=fwd["chunk_states"], hT=fwd["hT"],
                       want_dh0=True)
    x = oracle_inputs(cpu, ("q", "k", "v", "g", "meta_k", "meta_v", "h0"))
    ref = oracle.hybrid_fwd(x["q"], x["k"], x["v"], x["g"], x["meta_k"], x["meta_v"], w,
                            1 / math.sqrt(d), alpha, x["h0"])
    _, rdO = oracle.mse_loss(ref["o"], np64(tgt))
    rg = oracle.hybrid_bwd(x["q"], x["k"], x["v"], x["g"], x["meta_k"], x["meta_v"], rdO, w,
                           1 / math.sqrt(d), alpha, x["h0"], None)
    for name in ("dq", "dk", "dv", "dg", "dh0", "dmeta_k", "dmeta_v"):
        assert_close(name, res[name], rg[name], dtype)
    assert_close("dalpha", res["dalpha"].cpu().double().numpy(), np.array([rg["dalpha"]]), dtype)
