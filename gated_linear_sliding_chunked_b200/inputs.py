"""Seeded synthetic inputs for the hybrid attention operator.

This module only draws random numbers; it holds none of the operator's
arithmetic.  Both the CUDA path (tests, bench) and the fp64 oracle (tests)
receive the tensors made here, so they see identical, already-rounded values.

Workload shapes stand in for the Llama-3-8B / Mistral-7B attention layers the
Lizard pages evaluate at up to 32K-64K context (H = 32 heads of d = 128); the
pages publish no dataset or trained weights that reach the operator, so every
tensor is drawn from the distributions listed per workload below.

Recipe (per workload, seed s):
  * a ``torch.Generator`` seeded with s draws, in this order, q, k, v, the
    gate logits, meta_k, meta_v (and dO for training workloads), all fp32;
  * q, k, v are then rounded once to the I/O dtype (bf16 or fp32);
  * log-gates g = logsigmoid(N(mu, sigma)) / div stay fp32;
  * decode workloads draw state, K ring and V ring as N(0, 0.1^2).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch
import torch.nn.functional as F


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    T: int
    dk: int
    dv: int
    chunk: int
    w: int
    M: int
    io: str            # "f32" or "bf16"
    qk: str            # "scaled": N(0,1)/sqrt(dk);  "l2norm": that, then unit rows
    v_scale: float     # v ~ N(0,1) * v_scale
    g_mu: float
    g_sigma: float
    g_div: float
    alpha: float = 0.5
    train: bool = False

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.dk)

    @property
    def torch_dtype(self):
        return torch.float32 if self.io == "f32" else torch.bfloat16

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


@dataclass(frozen=True)
class DecodeWorkload:
    name: str
    Bd: int
    H: int
    dk: int
    dv: int
    w: int
    M: int
    steps: int
    pos0: int
    state_std: float = 0.1
    alpha: float = 0.5
    # per-step q, k, v, g follow the bf16 forward workload's recipe
    g_mu: float = 2.0
    g_sigma: float = 1.0
    g_div: float = 16.0

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.dk)

    def with_(self, **kw) -> "DecodeWorkload":
        return replace(self, **kw)


TINY_F32 = Workload("tiny fp32 hybrid fwd B1 H2 T256 d64", 1, 2, 256, 64, 64, 64, 64, 4,
                    "f32", "scaled", 1.0 / 8.0, 0.0, 1.0, 16.0)
FWD_BF16 = Workload("bf16 hybrid fwd B4 H16 T2048 d128 w64 M4", 4, 16, 2048, 128, 128, 64,
                    64, 4, "bf16", "l2norm", 1.0, 2.0, 1.0, 16.0)
TRAIN_BF16 = Workload("Llama-3-8B-shaped layer bf16 fwd+bwd B2 H32 T8192 d128 w128 M8", 2,
                      32, 8192, 128, 128, 64, 128, 8, "bf16", "scaled",
                      1.0 / math.sqrt(128.0), 0.0, 1.0, 16.0, train=True)
LONG_BF16 = Workload("long-context bf16 fwd B1 H32 T65536 d128 C128 w128 M8", 1, 32, 65536,
                     128, 128, 128, 128, 8, "bf16", "scaled", 1.0 / math.sqrt(128.0),
                     -1.0, 1.5, 1.0)
DECODE = DecodeWorkload("decode bf16 I/O fp32 state Bd128 H32 d128 w128 M8", 128, 32, 128,
                        128, 128, 8, 1000, 128)

WORKLOADS = {"tiny": TINY_F32, "fwd": FWD_BF16, "train": TRAIN_BF16, "long": LONG_BF16}


def _randn(gen, shape, device):
    return torch.randn(*shape, generator=gen, device=device, dtype=torch.float32)


def make_inputs(wl: Workload, seed: int = 0, device="cpu") -> dict:
    """Draw one batch for a prefill / training workload.

    Returns q, k, v (I/O dtype), g (fp32), meta_k, meta_v (I/O dtype) and, for
    training workloads, dO (I/O dtype)."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    B, H, T, dk, dv, M = wl.B, wl.H, wl.T, wl.dk, wl.dv, wl.M
    q = _randn(gen, (B, H, T, dk), device) / math.sqrt(dk)
    k = _randn(gen, (B, H, T, dk), device) / math.sqrt(dk)
    if wl.qk == "l2norm":
        q = F.normalize(q, dim=-1)
        k = F.normalize(k, dim=-1)
    v = _randn(gen, (B, H, T, dv), device) * wl.v_scale
    g = F.logsigmoid(_randn(gen, (B, H, T, dk), device) * wl.g_sigma + wl.g_mu) / wl.g_div
    mk = _randn(gen, (H, max(M, 0), dk), device)
    mv = _randn(gen, (H, max(M, 0), dv), device)
    dt = wl.torch_dtype
    out = {"q": q.to(dt), "k": k.to(dt), "v": v.to(dt), "g": g.contiguous(),
           "meta_k": mk.to(dt), "meta_v": mv.to(dt)}
    if wl.train:
        out["dO"] = _randn(gen, (B, H, T, dv), device).to(dt)
    return out


def make_teacher_output(wl: Workload, seed: int = 0, device="cpu", std: float = 0.5):
    """Synthetic stand-in for a teacher's attention output [B, H, T, dv] (the
    target of the first training stage; no teacher weights are available)."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    return (_randn(gen, (wl.B, wl.H, wl.T, wl.dv), device) * std).to(wl.torch_dtype)


def make_decode_state(wl: DecodeWorkload, seed: int = 0, device="cpu") -> dict:
    """Initial decode state: fp32 state, bf16 K/V rings, positions, meta."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    Bd, H, dk, dv, w, M = wl.Bd, wl.H, wl.dk, wl.dv, wl.w, wl.M
    state = _randn(gen, (Bd, H, dk, dv), device) * wl.state_std
    kring = (_randn(gen, (Bd, H, w, dk), device) * wl.state_std).to(torch.bfloat16)
    vring = (_randn(gen, (Bd, H, w, dv), device) * wl.state_std).to(torch.bfloat16)
    pos = torch.full((Bd,), wl.pos0, dtype=torch.int64, device=device)
    mk = _randn(gen, (H, M, dk), device).to(torch.bfloat16)
    mv = _randn(gen, (H, M, dv), device).to(torch.bfloat16)
    return {"state": state, "kring": kring, "vring": vring, "pos": pos,
            "meta_k": mk, "meta_v": mv}


def make_decode_tokens(wl: DecodeWorkload, steps: int, seed: int = 1, device="cpu") -> dict:
    """Per-step q, k, v (bf16, unit rows for q and k) and g (fp32), stacked
    over ``steps``: shapes [steps, Bd, H, d]."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    Bd, H, dk, dv = wl.Bd, wl.H, wl.dk, wl.dv
    q = F.normalize(_randn(gen, (steps, Bd, H, dk), device) / math.sqrt(dk), dim=-1)
    k = F.normalize(_randn(gen, (steps, Bd, H, dk), device) / math.sqrt(dk), dim=-1)
    v = _randn(gen, (steps, Bd, H, dv), device)
    g = F.logsigmoid(_randn(gen, (steps, Bd, H, dk), device) * wl.g_sigma + wl.g_mu) / wl.g_div
    return {"q": q.to(torch.bfloat16), "k": k.to(torch.bfloat16),
            "v": v.to(torch.bfloat16), "g": g.contiguous()}
