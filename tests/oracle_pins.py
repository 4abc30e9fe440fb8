"""Pins that tie the fp64 oracle to facts fixed outside the oracle itself.

Each ``pin_*`` function raises AssertionError when the oracle handle ``lib``
disagrees with the fact it checks.  ``test_oracle_pins.py`` runs them on the
real oracle; ``test_oracle_mutants.py`` runs them on deliberately broken
builds and requires every mutant to fail at least one pin.

Sources of the facts (Lizard technical summary on gist.science, section 2a,
plus mathematics):
  * the gated state update S_t = diag(exp(g_t)) S_{t-1} + k_t v_t^T has the
    closed-form solution S_t = sum_{s<=t} diag(exp(G_t - G_s)) k_s v_s^T +
    diag(exp(G_t)) h0 with G the running sum of g (unrolled recurrence);
  * all gates equal to one (g = 0) leave plain causal linear attention,
    o = tril(Q K^T) V;
  * full forgetting (g -> -inf) leaves o_t = (q_t . k_t) v_t;
  * the section 2c chunked rearrangement equals the recurrence exactly;
  * a window covering the whole prefix without meta tokens is causal
    softmax attention (torch's scaled_dot_product_attention, fp64);
  * meta tokens are extra always-visible keys (sinks) in the softmax;
    sink-only mode rescales the no-meta output by exp(lse0 - lse);
  * o = o_gla + alpha o_swa is affine in alpha;
  * gradients equal central finite differences;
  * decoding token by token reproduces the prefill.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle

RNG = np.random.default_rng


def _rel(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    den = np.linalg.norm(b.ravel())
    return np.linalg.norm((a - b).ravel()) / (den if den > 0 else 1.0)


def _gla_inputs(seed, B=2, H=2, T=37, dk=8, dv=6, g_mu=0.0, g_sigma=1.0, g_div=1.0):
    r = RNG(seed)
    q = r.standard_normal((B, H, T, dk)) / math.sqrt(dk)
    k = r.standard_normal((B, H, T, dk)) / math.sqrt(dk)
    v = r.standard_normal((B, H, T, dv))
    x = r.standard_normal((B, H, T, dk)) * g_sigma + g_mu
    g = -np.logaddexp(0.0, -x) / g_div  # logsigmoid
    h0 = r.standard_normal((B, H, dk, dv)) * 0.3
    return q, k, v, g, h0


def _swa_inputs(seed, B=2, H=3, T=29, dk=8, dv=5, M=3):
    r = RNG(seed)
    q = r.standard_normal((B, H, T, dk))
    k = r.standard_normal((B, H, T, dk))
    v = r.standard_normal((B, H, T, dv))
    mk = r.standard_normal((H, M, dk))
    mv = r.standard_normal((H, M, dv))
    return q, k, v, mk, mv


# ----------------------------------------------------------------------------
# gated linear attention
# ----------------------------------------------------------------------------
def pin_gla_closed_form(lib):
    """Recurrent oracle == unrolled closed form with global cumulative gates."""
    q, k, v, g, h0 = _gla_inputs(1)
    o, hT = oracle.gla_fwd(q, k, v, g, h0, lib=lib)
    G = np.cumsum(g, axis=2)  # [B,H,T,dk]
    B, H, T, dk = q.shape
    ref = np.zeros_like(o)
    for b in range(B):
        for h in range(H):
            # decay factors exp(G_t - G_s) for every pair, masked to s <= t
            D = np.exp(G[b, h][:, None, :] - G[b, h][None, :, :])  # [t, s, i]
            A = np.einsum("ti,si,tsi->ts", q[b, h], k[b, h], D)
            A = np.tril(A)
            ref[b, h] = A @ v[b, h] + (q[b, h] * np.exp(G[b, h])) @ h0[b, h]
    assert _rel(o, ref) < 1e-12, _rel(o, ref)
    hT_ref = np.einsum("si,sj->ij", k[0, 0] * np.exp(G[0, 0, -1] - G[0, 0]), v[0, 0]) + \
        np.exp(G[0, 0, -1])[:, None] * h0[0, 0]
    assert _rel(hT[0, 0], hT_ref) < 1e-12


def pin_gla_unit_gates(lib):
    """g = 0 (all gates one) is causal linear attention tril(Q K^T) V."""
    q, k, v, _, _ = _gla_inputs(2, T=23)
    g = np.zeros_like(q)
    o, hT = oracle.gla_fwd(q, k, v, g, lib=lib)
    ref = np.einsum("bhts,bhsj->bhtj", np.tril(np.einsum("bhti,bhsi->bhts", q, k)), v)
    assert _rel(o, ref) < 1e-12
    assert _rel(hT, np.einsum("bhti,bhtj->bhij", k, v)) < 1e-12


def pin_gla_full_forgetting(lib):
    """g -> -inf keeps only the current token: o_t = (q_t . k_t) v_t."""
    q, k, v, _, h0 = _gla_inputs(3, T=11)
    g = np.full_like(q, -1e4)
    o, hT = oracle.gla_fwd(q, k, v, g, h0, lib=lib)
    ref = np.einsum("bhti,bhti->bht", q, k)[..., None] * v
    assert _rel(o, ref) < 1e-12
    assert _rel(hT, k[:, :, -1, :, None] * v[:, :, -1, None, :]) < 1e-12


def pin_gla_initial_state(lib):
    """With k = 0 the output is q_t^T diag(exp(G_t)) h0 (pure decay of h0)."""
    q, k, v, g, h0 = _gla_inputs(4, T=9)
    k = np.zeros_like(k)
    o, hT = oracle.gla_fwd(q, k, v, g, h0, lib=lib)
    G = np.cumsum(g, axis=2)
    ref = np.einsum("bhti,bhij->bhtj", q * np.exp(G), h0)
    assert _rel(o, ref) < 1e-12
    assert _rel(hT, np.exp(G[:, :, -1])[..., None] * h0) < 1e-12


def pin_gla_chunked_identity(lib):
    """The chunked rearrangement reproduces the recurrence for any chunk size."""
    for (g_mu, g_sigma, g_div) in ((0.0, 1.0, 16.0), (-1.0, 1.5, 1.0)):
        q, k, v, g, h0 = _gla_inputs(5, T=45, g_mu=g_mu, g_sigma=g_sigma, g_div=g_div)
        o, hT = oracle.gla_fwd(q, k, v, g, h0, lib=lib)
        for C in (1, 4, 16, 64):
            oc, hc = oracle.gla_chunked_fwd(q, k, v, g, C, h0, lib=lib)
            assert _rel(oc, o) < 1e-12, (C, _rel(oc, o))
            assert _rel(hc, hT) < 1e-12


# ----------------------------------------------------------------------------
# window + meta softmax
# ----------------------------------------------------------------------------
def _sdpa(q, k, v, mask, scale):
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x))
    out = torch.nn.functional.scaled_dot_product_attention(
        t(q), t(k), t(v), attn_mask=t(mask), scale=scale)
    return out.numpy()


def _band_mask(T, w, M):
    """Boolean [T, M+T] mask: M always-visible meta columns, then a causal band."""
    tt = np.arange(T)[:, None]
    ss = np.arange(T)[None, :]
    band = (ss <= tt) & (ss >= tt - w + 1)
    return np.concatenate([np.ones((T, M), dtype=bool), band], axis=1)


def pin_swa_full_causal(lib):
    """w >= T and M = 0 is causal softmax attention (library routine)."""
    q, k, v, _, _ = _swa_inputs(6, M=0)
    T = q.shape[2]
    scale = 0.37
    o, _ = oracle.swa_meta_fwd(q, k, v, None, None, T + 5, scale, lib=lib)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v), is_causal=True,
        scale=scale).numpy()
    assert _rel(o, ref) < 1e-12


def pin_swa_band_meta(lib):
    """Window w < T with M meta keys/values = masked softmax over [meta; keys]."""
    q, k, v, mk, mv = _swa_inputs(7)
    B, H, T, dk = q.shape
    M = mk.shape[1]
    for w in (1, 4, 9):
        scale = 1.0 / math.sqrt(dk)
        o, _ = oracle.swa_meta_fwd(q, k, v, mk, mv, w, scale, lib=lib)
        kk = np.concatenate([np.broadcast_to(mk[None], (B, H, M, dk)), k], axis=2)
        vv = np.concatenate([np.broadcast_to(mv[None], (B, H, M, mv.shape[-1])), v], axis=2)
        ref = _sdpa(q, kk, vv, _band_mask(T, w, M), scale)
        assert _rel(o, ref) < 1e-12, (w, _rel(o, ref))


def pin_swa_sinks(lib):
    """Sink-only meta tokens: zero-valued extra keys; o = o0 * exp(lse0 - lse)."""
    q, k, v, mk, _ = _swa_inputs(8)
    B, H, T, dk = q.shape
    M = mk.shape[1]
    w, scale = 6, 0.5
    o, lse = oracle.swa_meta_fwd(q, k, v, mk, None, w, scale, lib=lib)
    o0, lse0 = oracle.swa_meta_fwd(q, k, v, None, None, w, scale, lib=lib)
    kk = np.concatenate([np.broadcast_to(mk[None], (B, H, M, dk)), k], axis=2)
    vv = np.concatenate([np.zeros((B, H, M, v.shape[-1])), v], axis=2)
    assert _rel(o, _sdpa(q, kk, vv, _band_mask(T, w, M), scale)) < 1e-12
    assert _rel(o, o0 * np.exp(lse0 - lse)[..., None]) < 1e-12
    assert np.all(lse > lse0)
    # the log-sum-exp of the no-meta case for w = 1 is the single logit
    _, l1 = oracle.swa_meta_fwd(q, k, v, None, None, 1, scale, lib=lib)
    assert _rel(l1, scale * np.einsum("bhti,bhti->bht", q, k)) < 1e-12


def pin_hybrid_affine(lib):
    """o = o_gla + alpha * o_swa: alpha = 0 is the gated branch; affine in alpha."""
    q, k, v, g, h0 = _gla_inputs(9, B=1, H=3, T=21)
    r = RNG(10)
    mk = r.standard_normal((3, 2, q.shape[-1]))
    mv = r.standard_normal((3, 2, v.shape[-1]))
    o_gla, hT = oracle.gla_fwd(q, k, v, g, h0, lib=lib)
    o_swa, lse = oracle.swa_meta_fwd(q, k, v, mk, mv, 5, 0.4, lib=lib)
    for alpha in (0.0, 0.5, 2.0):
        res = oracle.hybrid_fwd(q, k, v, g, mk, mv, 5, 0.4, alpha, h0, lib=lib)
        assert _rel(res["o"], o_gla + alpha * o_swa) < 1e-12
        assert _rel(res["hT"], hT) < 1e-12 and _rel(res["lse"], lse) < 1e-12


# ----------------------------------------------------------------------------
# gradients: central finite differences
# ----------------------------------------------------------------------------
def _tiny_case(seed):
    r = RNG(seed)
    B, H, T, dk, dv, M = 1, 2, 12, 4, 3, 2
    x = {
        "q": r.standard_normal((B, H, T, dk)) * 0.5,
        "k": r.standard_normal((B, H, T, dk)) * 0.5,
        "v": r.standard_normal((B, H, T, dv)),
        "g": -np.logaddexp(0.0, -(r.standard_normal((B, H, T, dk)) - 0.5)),
        "h0": r.standard_normal((B, H, dk, dv)) * 0.5,
        "meta_k": r.standard_normal((H, M, dk)),
        "meta_v": r.standard_normal((H, M, dv)),
        "alpha": np.array(0.7),
    }
    dO = r.standard_normal((B, H, T, dv))
    dhT = r.standard_normal((B, H, dk, dv))
    return x, dO, dhT


def _hybrid_loss(lib, x, dO, dhT, w, scale):
    res = oracle.hybrid_fwd(x["q"], x["k"], x["v"], x["g"], x["meta_k"], x["meta_v"], w,
                            scale, float(x["alpha"]), x["h0"], lib=lib)
    return float(np.sum(res["o"] * dO) + np.sum(res["hT"] * dhT))


def pin_hybrid_grad_fd(lib):
    """Hand-written hybrid backward equals central differences (h = 1e-6)."""
    x, dO, dhT = _tiny_case(11)
    w, scale, eps = 3, 0.6, 1e-6
    an = oracle.hybrid_bwd(x["q"], x["k"], x["v"], x["g"], x["meta_k"], x["meta_v"], dO, w,
                           scale, float(x["alpha"]), x["h0"], dhT, lib=lib)
    names = {"q": "dq", "k": "dk", "v": "dv", "g": "dg", "h0": "dh0",
             "meta_k": "dmeta_k", "meta_v": "dmeta_v", "alpha": "dalpha"}
    for key, gname in names.items():
        base = x[key]
        num = np.zeros(np.shape(base))
        flat = num.reshape(-1)
        for idx in range(flat.size):
            xp = dict(x)
            xm = dict(x)
            bp = np.array(base, dtype=np.float64).reshape(-1).copy()
            bm = bp.copy()
            bp[idx] += eps
            bm[idx] -= eps
            xp[key] = bp.reshape(np.shape(base))
            xm[key] = bm.reshape(np.shape(base))
            flat[idx] = (_hybrid_loss(lib, xp, dO, dhT, w, scale) -
                         _hybrid_loss(lib, xm, dO, dhT, w, scale)) / (2 * eps)
        got = np.asarray(an[gname], dtype=np.float64)
        assert _rel(got, num) < 1e-6, (key, _rel(got, num))


def pin_swa_grad_fd(lib):
    """Window-only backward (sink-only and with meta values) vs differences."""
    x, dO, _ = _tiny_case(12)
    w, scale, eps = 4, 0.8, 1e-6
    for mv in (x["meta_v"], None):
        an = oracle.swa_meta_bwd(x["q"], x["k"], x["v"], x["meta_k"], mv, dO, w, scale,
                                 lib=lib)

        def loss(q, k, v, mk, mvv):
            o, _ = oracle.swa_meta_fwd(q, k, v, mk, mvv, w, scale, lib=lib)
            return float(np.sum(o * dO))

        args = [x["q"], x["k"], x["v"], x["meta_k"], mv]
        for pos, gname in enumerate(("dq", "dk", "dv", "dmeta_k", "dmeta_v")):
            if args[pos] is None:
                continue
            base = np.array(args[pos], dtype=np.float64)
            num = np.zeros(base.shape).reshape(-1)
            for idx in range(base.size):
                ap = list(args)
                am = list(args)
                bp = base.reshape(-1).copy()
                bm = bp.copy()
                bp[idx] += eps
                bm[idx] -= eps
                ap[pos] = bp.reshape(base.shape)
                am[pos] = bm.reshape(base.shape)
                num[idx] = (loss(*ap) - loss(*am)) / (2 * eps)
            assert _rel(an[gname], num.reshape(base.shape)) < 1e-6, (gname, mv is None)


def pin_gla_dg_identity(lib):
    """dg = reverse cumsum over t of (q*dq - k*dk), plus the hT term at t = T-1.

    With G the running sum of g, o and hT depend on G only through
    q_t exp(G_t), k_s exp(-G_s) and the factor exp(G_{T-1}) of hT, which
    gives dL/dG_t = q_t dq_t - k_t dk_t (+ sum_j dhT_ij hT_ij at t = T-1)."""
    q, k, v, g, h0 = _gla_inputs(13, T=19)
    r = RNG(14)
    dO = r.standard_normal(v.shape)
    dhT = r.standard_normal(h0.shape)
    res = oracle.gla_bwd(q, k, v, g, dO, h0, dhT, lib=lib)
    _, hT = oracle.gla_fwd(q, k, v, g, h0, lib=lib)
    dG = q * res["dq"] - k * res["dk"]
    dG[:, :, -1] += np.sum(dhT * hT, axis=-1)
    dg_ref = np.flip(np.cumsum(np.flip(dG, axis=2), axis=2), axis=2)
    assert _rel(res["dg"], dg_ref) < 1e-10, _rel(res["dg"], dg_ref)


# ----------------------------------------------------------------------------
# decode
# ----------------------------------------------------------------------------
def pin_decode_matches_prefill(lib):
    """Token-by-token decode from an empty state equals the prefill, including
    after the window ring wraps around (T > w)."""
    r = RNG(15)
    Bd, H, T, dk, dv, w, M = 2, 2, 13, 4, 3, 5, 2
    q = r.standard_normal((Bd, H, T, dk))
    k = r.standard_normal((Bd, H, T, dk))
    v = r.standard_normal((Bd, H, T, dv))
    g = -np.logaddexp(0.0, -r.standard_normal((Bd, H, T, dk)))
    mk = r.standard_normal((H, M, dk))
    mv = r.standard_normal((H, M, dv))
    scale, alpha = 0.5, 0.7
    pre = oracle.hybrid_fwd(q, k, v, g, mk, mv, w, scale, alpha, lib=lib)
    st = {"state": np.zeros((Bd, H, dk, dv)), "kring": np.zeros((Bd, H, w, dk)),
          "vring": np.zeros((Bd, H, w, dv)), "pos": np.zeros(Bd, dtype=np.int64)}
    outs = []
    for t in range(T):
        st = oracle.decode_step(st["state"], st["kring"], st["vring"], st["pos"],
                                q[:, :, t], k[:, :, t], v[:, :, t], g[:, :, t], mk, mv,
                                scale, alpha, lib=lib)
        outs.append(st["o"])
    dec = np.stack(outs, axis=2)
    assert _rel(dec, pre["o"]) < 1e-12, _rel(dec, pre["o"])
    assert _rel(st["state"], pre["hT"]) < 1e-12
    assert np.all(st["pos"] == T)
    # the ring holds the last w keys at slot (token mod w)
    for tok in range(T - w, T):
        assert np.array_equal(st["kring"][:, :, tok % w], k[:, :, tok])


# ----------------------------------------------------------------------------
# stage-1 distillation loss (section 2b): MSE to the teacher's attention output
# ----------------------------------------------------------------------------
def pin_mse_closed_form(lib):
    """A constant offset c between output and target gives loss c^2 and the
    gradient -2c/n everywhere; a target equal to the output gives zero."""
    r = RNG(21)
    o = r.standard_normal((2, 3, 5, 4))
    n = o.size
    for c in (0.0, 0.37, -1.5):
        loss, dO = oracle.mse_loss(o, o + c, lib=lib)
        assert abs(loss - c * c) <= 1e-12 * max(1.0, c * c), (c, loss)
        assert np.allclose(dO, -2.0 * c / n, rtol=0, atol=1e-15), c
    # a single differing element: loss = e^2 / n
    t = o.copy()
    t[1, 2, 3, 0] += 3.0
    loss, dO = oracle.mse_loss(o, t, lib=lib)
    assert abs(loss - 9.0 / n) < 1e-12
    assert abs(dO[1, 2, 3, 0] + 6.0 / n) < 1e-15 and np.count_nonzero(dO) == 1
    assert oracle.mse_loss(np.zeros((0, 4)), np.zeros((0, 4)), lib=lib)[0] == 0.0


def pin_mse_grad_fd(lib):
    """dO equals central differences of the loss with respect to o."""
    r = RNG(22)
    o = r.standard_normal((1, 2, 6, 3))
    t = r.standard_normal(o.shape)
    _, dO = oracle.mse_loss(o, t, lib=lib)
    eps = 1e-6
    num = np.zeros(o.size)
    for idx in range(o.size):
        op = o.reshape(-1).copy()
        om = op.copy()
        op[idx] += eps
        om[idx] -= eps
        num[idx] = (oracle.mse_loss(op.reshape(o.shape), t, lib=lib)[0] -
                    oracle.mse_loss(om.reshape(o.shape), t, lib=lib)[0]) / (2 * eps)
    assert _rel(dO.reshape(-1), num) < 1e-7, _rel(dO.reshape(-1), num)


def _stage1_loss(lib, x, target, w, scale):
    res = oracle.hybrid_fwd(x["q"], x["k"], x["v"], x["g"], x["meta_k"], x["meta_v"], w,
                            scale, float(x["alpha"]), x["h0"], lib=lib)
    return oracle.mse_loss(res["o"], target, lib=lib)


def pin_stage1_chain_fd(lib):
    """The stage-1 step (hybrid forward, MSE to a teacher output, hybrid
    backward fed with the loss gradient) gives the central differences of the
    loss with respect to every operator input."""
    x, _, _ = _tiny_case(23)
    target = RNG(24).standard_normal(np.shape(x["v"]))
    w, scale, eps = 4, 0.5, 1e-6
    _, dO = _stage1_loss(lib, x, target, w, scale)
    an = oracle.hybrid_bwd(x["q"], x["k"], x["v"], x["g"], x["meta_k"], x["meta_v"], dO, w,
                           scale, float(x["alpha"]), x["h0"], None, lib=lib)
    names = {"q": "dq", "k": "dk", "v": "dv", "g": "dg", "meta_k": "dmeta_k",
             "alpha": "dalpha"}
    for key, gname in names.items():
        base = np.array(x[key], dtype=np.float64)
        num = np.zeros(base.size)
        for idx in range(base.size):
            bp = base.reshape(-1).copy()
            bm = bp.copy()
            bp[idx] += eps
            bm[idx] -= eps
            xp, xm = dict(x), dict(x)
            xp[key] = bp.reshape(base.shape)
            xm[key] = bm.reshape(base.shape)
            num[idx] = (_stage1_loss(lib, xp, target, w, scale)[0] -
                        _stage1_loss(lib, xm, target, w, scale)[0]) / (2 * eps)
        got = np.asarray(an[gname], dtype=np.float64).reshape(-1)
        assert _rel(got, num) < 1e-6, (key, _rel(got, num))


# ----------------------------------------------------------------------------
# gate from its logit (section 2a: Gamma = sigma(W_gamma x))
# ----------------------------------------------------------------------------
def pin_gate_logits_closed_form(lib):
    """exp(g / scale) is the logistic function of z (written here as
    1 / (1 + e^{-z}) directly); z = 0 gives -scale log 2; far tails behave
    as -scale e^{-z} and scale z."""
    z = np.array([-40.0, -5.0, -0.5, 0.0, 0.7, 3.0, 30.0])
    for scale in (1.0, 1.0 / 16):
        g = oracle.gate_from_logits(z, scale, lib=lib)
        assert np.all(g <= 0.0)
        mid = np.abs(z) < 10
        assert np.allclose(np.exp(g[mid] / scale), 1.0 / (1.0 + np.exp(-z[mid])), rtol=1e-13)
        assert abs(g[3] + scale * np.log(2.0)) < 1e-15
        assert abs(g[-1] / scale + np.exp(-30.0)) < 1e-25
        assert abs(g[0] / scale - (-40.0)) < 1e-15


def pin_gate_logits_grad_fd(lib):
    """dz through the gate map composed with the hybrid operator equals the
    central differences of sum(o * dO) + sum(hT * dhT) with respect to z."""
    x, dO, dhT = _tiny_case(31)
    r = RNG(32)
    z = r.standard_normal(np.shape(x["g"])) * 2.0
    w, scale, s, eps = 3, 0.6, 0.25, 1e-6

    def loss(zz):
        xx = dict(x)
        xx["g"] = oracle.gate_from_logits(zz, s, lib=lib)
        return _hybrid_loss(lib, xx, dO, dhT, w, scale)

    xx = dict(x)
    xx["g"] = oracle.gate_from_logits(z, s, lib=lib)
    an = oracle.hybrid_bwd(xx["q"], xx["k"], xx["v"], xx["g"], xx["meta_k"], xx["meta_v"], dO, w,
                           scale, float(xx["alpha"]), xx["h0"], dhT, lib=lib)
    dz = oracle.dlogits(z, an["dg"], s, lib=lib).reshape(-1)
    num = np.zeros(z.size)
    for idx in range(z.size):
        zp = z.reshape(-1).copy()
        zm = zp.copy()
        zp[idx] += eps
        zm[idx] -= eps
        num[idx] = (loss(zp.reshape(z.shape)) - loss(zm.reshape(z.shape))) / (2 * eps)
    assert _rel(dz, num) < 1e-6, _rel(dz, num)


# ----------------------------------------------------------------------------
# the projections in front of the operator (section 2a: Gamma = sigma(W_gamma x),
# phi(k); reading: phi is the identity)
# ----------------------------------------------------------------------------
def _proj_x(seed, B=2, T=5, Dm=24):
    return RNG(seed).standard_normal((B, T, Dm))


def pin_projection_selection(lib):
    """One-hot weight rows pick single hidden features: q[b, h, t, i] is
    x[b, t, perm(h, i)], in the operator's [B, H, T, dk] layout."""
    H, dk, Dm = 3, 4, 24
    x = _proj_x(41, Dm=Dm)
    perm = RNG(42).permutation(Dm)[: H * dk]
    W = np.zeros((H * dk, Dm))
    W[np.arange(H * dk), perm] = 1.0
    q, k, g = oracle.qkg_projection(x, W, None, None, H, dk, lib=lib)
    assert k is None and g is None
    want = x[:, :, perm].reshape(x.shape[0], x.shape[1], H, dk).transpose(0, 2, 1, 3)
    assert np.array_equal(q, want)


def pin_projection_rank_one(lib):
    """W = a c^T (rank one) gives y = (x . c) a: keys through the identity
    feature map, gates through the logistic written out directly."""
    H, dk, Dm, s = 2, 3, 24, 0.5
    x = _proj_x(43, Dm=Dm)
    r = RNG(44)
    a, c = r.standard_normal(H * dk), r.standard_normal(Dm) * 0.3
    W = np.outer(a, c)
    _, k, g = oracle.qkg_projection(x, None, W, W, H, dk, s, lib=lib)
    xc = np.einsum("btd,d->bt", x, c)
    y = (xc[:, :, None] * a[None, None, :]).reshape(x.shape[0], x.shape[1], H, dk)
    y = y.transpose(0, 2, 1, 3)
    assert _rel(k, y) < 1e-13
    assert np.allclose(np.exp(g / s), 1.0 / (1.0 + np.exp(-y)), rtol=1e-12)


def pin_projection_zero_gate_weights(lib):
    """A zero gate projection gives sigma(0) = 1/2 everywhere: g = -scale log 2."""
    H, dk, Dm, s = 2, 4, 24, 1.0 / 16
    x = _proj_x(45, Dm=Dm)
    _, _, g = oracle.qkg_projection(x, None, None, np.zeros((H * dk, Dm)), H, dk, s, lib=lib)
    assert np.allclose(g, -s * np.log(2.0), rtol=0, atol=1e-16)


ALL_PINS = [
    pin_gla_closed_form, pin_gla_unit_gates, pin_gla_full_forgetting,
    pin_gla_initial_state, pin_gla_chunked_identity, pin_swa_full_causal,
    pin_swa_band_meta, pin_swa_sinks, pin_hybrid_affine, pin_hybrid_grad_fd,
    pin_swa_grad_fd, pin_gla_dg_identity, pin_decode_matches_prefill,
    pin_mse_closed_form, pin_mse_grad_fd, pin_stage1_chain_fd,
    pin_gate_logits_closed_form, pin_gate_logits_grad_fd, pin_projection_selection,
    pin_projection_rank_one, pin_projection_zero_gate_weights,
]
