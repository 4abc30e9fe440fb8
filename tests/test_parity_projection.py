"""The projections in front of the operator (q, k with the identity feature
map; the fp32 log-gates scale * log sigma(x Wg^T)) on the tcgen05 kernel vs
the fp64 oracle, on the same bf16 inputs."""
import numpy as np
import pytest
import torch

import gated_linear_sliding_chunked_b200 as L
import oracle
from parity_util import assert_close, np64

pytestmark = pytest.mark.gpu


def _case(seed, B, T, Dm, H, dk, wstd=None):
    gen = torch.Generator().manual_seed(seed)
    wstd = wstd if wstd is not None else 1.0 / np.sqrt(Dm)
    x = torch.randn(B, T, Dm, generator=gen).to(torch.bfloat16)
    W = [(torch.randn(H * dk, Dm, generator=gen) * wstd).to(torch.bfloat16) for _ in range(3)]
    return x, W


@pytest.mark.parametrize("B,T,Dm,H,dk", [(1, 1, 64, 2, 128), (2, 150, 136, 4, 64),
                                         (1, 300, 512, 2, 128), (3, 77, 1000, 8, 64)])
def test_projection_matches_oracle(B, T, Dm, H, dk):
    """Ragged token tiles (T not a multiple of 128), ragged hidden size (Dm not
    a multiple of 64), both head dims; every output against the oracle."""
    x, W = _case(500 + T + Dm, B, T, Dm, H, dk)
    s = 1.0 / 16
    q, k, g = L.qkg_projection(x.cuda(), *(w.cuda() for w in W), heads=H, gate_scale=s)
    rq, rk, rg = oracle.qkg_projection(np64(x), *(np64(w) for w in W), H, dk, s)
    assert_close("q", q, rq, torch.bfloat16)
    assert_close("k", k, rk, torch.bfloat16)
    assert_close("g", g, rg, torch.float32, factor=10.0)  # fp32 output of bf16 products
    L.lz_device_check()


def test_projection_subset_and_gate_only():
    """A NULL weight skips its output; the gate alone as well."""
    x, W = _case(520, 2, 64, 256, 2, 128)
    xd = x.cuda()
    q, k, g = L.qkg_projection(xd, None, None, W[2].cuda(), heads=2, gate_scale=0.5)
    assert q is None and k is None
    _, _, rg = oracle.qkg_projection(np64(x), None, None, np64(W[2]), 2, 128, 0.5)
    assert_close("g", g, rg, torch.float32, factor=10.0)
    q, k, g = L.qkg_projection(xd, W[0].cuda(), W[1].cuda(), None, heads=2)
    rq, rk, _ = oracle.qkg_projection(np64(x), np64(W[0]), np64(W[1]), None, 2, 128)
    assert g is None
    assert_close("q", q, rq, torch.bfloat16)
    assert_close("k", k, rk, torch.bfloat16)


def test_projection_llama_layer_sampled_tokens():
    """The training layer's shape (B=2, T=8192, Dm=4096, 32 heads of 128): the
    whole projection on the GPU, eight sampled tokens of both batch rows
    checked against the oracle over every head and feature."""
    B, T, Dm, H, dk = 2, 8192, 4096, 32, 128
    x, W = _case(530, B, T, Dm, H, dk)
    q, k, g = L.qkg_projection(x.cuda(), *(w.cuda() for w in W), heads=H, gate_scale=1.0 / 16)
    torch.cuda.synchronize()
    idx = [0, 1, 127, 128, 4095, 4100, 8190, 8191]
    rq, rk, rg = oracle.qkg_projection(np64(x[:, idx]), *(np64(w) for w in W), H, dk, 1.0 / 16)
    assert_close("q", q[:, :, idx], rq, torch.bfloat16)
    assert_close("k", k[:, :, idx], rk, torch.bfloat16)
    assert_close("g", g[:, :, idx], rg, torch.float32, factor=10.0)
    L.lz_device_check()
