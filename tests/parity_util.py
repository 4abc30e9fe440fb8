"""Helpers shared by the GPU parity tests: relative L2 error, oracle calls on
the exact (already rounded) inputs the CUDA path sees, and seeded small
problems.  The oracle is imported only here, in the tests."""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle

# relative-L2 bars per output tensor: fp32 I/O and bf16 I/O (fp32 accumulate)
TOL = {torch.float32: 1e-5, torch.bfloat16: 2e-2}


def rel_l2(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref.ravel())
    num = np.linalg.norm((got - ref).ravel())
    if den == 0.0:
        return num
    return num / den


def np64(t):
    if t is None:
        return None
    return t.detach().to("cpu", torch.float64).numpy()


def assert_close(name, got, ref, dtype, factor=1.0):
    err = rel_l2(np64(got) if torch.is_tensor(got) else got, ref)
    tol = TOL[dtype] * factor
    assert np.isfinite(err) and err <= tol, f"{name}: rel-L2 {err:.3e} > {tol:.1e}"
    return err


def small_problem(seed, B, H, T, dk, dv, M, dtype, *, g_mu=0.0, g_sigma=1.0, g_div=16.0,
                  qk_scale=None, device="cuda", train=False, h0=False):
    """Seeded inputs drawn on the CPU, rounded to the I/O dtype, then copied."""
    gen = torch.Generator().manual_seed(seed)
    qk_scale = 1.0 / math.sqrt(dk) if qk_scale is None else qk_scale
    r = lambda *s: torch.randn(*s, generator=gen)
    x = {
        "q": (r(B, H, T, dk) * qk_scale).to(dtype),
        "k": (r(B, H, T, dk) * qk_scale).to(dtype),
        "v": r(B, H, T, dv).to(dtype),
        "g": torch.nn.functional.logsigmoid(r(B, H, T, dk) * g_sigma + g_mu) / g_div,
        "meta_k": r(H, M, dk).to(dtype),
        "meta_v": r(H, M, dv).to(dtype),
    }
    if train:
        x["dO"] = r(B, H, T, dv).to(dtype)
        x["dhT"] = r(B, H, dk, dv) * 0.1
    if h0:
        x["h0"] = r(B, H, dk, dv) * 0.1
    cpu = {k: v.contiguous() for k, v in x.items()}
    dev = {k: v.to(device) for k, v in cpu.items()}
    return cpu, dev


def oracle_inputs(cpu: dict, keys):
    return {k: (np64(cpu[k]) if cpu.get(k) is not None else None) for k in keys}
