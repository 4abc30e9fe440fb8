"""Decode-step parity: the constant-memory generation step vs the oracle, the
decode-equals-prefill identity on the GPU, and save/restore of the state."""
import math
import random

import numpy as np
import pytest
import torch

import gated_linear_sliding_chunked_b200 as L
from gated_linear_sliding_chunked_b200 import inputs as I
import oracle
from parity_util import assert_close, np64, small_problem

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("w,M,sink", [(1, 0, False), (5, 2, False), (16, 3, True),
                                      (40, 16, False)])
def test_decode_equals_prefill(dtype, w, M, sink):
    """T steps from an empty state reproduce the hybrid forward on the same
    tokens (the window wraps around the ring when T > w)."""
    Bd, H, T = 3, 2, 37
    cpu, dev = small_problem(50 + w + M, Bd, H, T, 128, 128, M, dtype)
    mk = dev["meta_k"] if M else None
    mv = dev["meta_v"] if (M and not sink) else None
    alpha = 0.7
    pre = L.hybrid_fwd(dev["q"], dev["k"], dev["v"], dev["g"], mk, mv, w=w, alpha=alpha,
                       want_hT=True)
    state = torch.zeros(Bd, H, 128, 128, device="cuda")
    kring = torch.zeros(Bd, H, w, 128, dtype=dtype, device="cuda")
    vring = torch.zeros_like(kring)
    pos = torch.zeros(Bd, dtype=torch.int64, device="cuda")
    outs = []
    for t in range(T):
        sl = lambda n: dev[n][:, :, t].contiguous()
        outs.append(L.decode_step(state, kring, vring, pos, sl("q"), sl("k"), sl("v"), sl("g"),
                                  mk, mv, alpha=alpha).clone())
    dec = torch.stack(outs, dim=2)
    x = {k: np64(v) for k, v in cpu.items()}
    ref = oracle.hybrid_fwd(x["q"], x["k"], x["v"], x["g"], x["meta_k"] if M else None,
                            x["meta_v"] if (M and not sink) else None, w, 1 / math.sqrt(128),
                            alpha)
    assert_close("decode o", dec, ref["o"], dtype)
    assert_close("decode state", state, ref["hT"], dtype)
    assert_close("prefill o", pre["o"], ref["o"], dtype)
    assert torch.all(pos.cpu() == T)


def test_decode_workload_sampled():
    """Decode workload shape (Bd=128, H=32, w=128, M=8, bf16 I/O, fp32 state)
    from a random full-window state: 6 steps on the GPU; sampled
    (sequence, head) pairs replayed in the oracle step by step."""
    wl = I.DECODE
    st = I.make_decode_state(wl, seed=0, device="cpu")
    toks = I.make_decode_tokens(wl, steps=6, seed=1, device="cpu")
    d = {k: v.cuda() for k, v in st.items()}
    outs = []
    for s in range(6):
        outs.append(L.decode_step(d["state"], d["kring"], d["vring"], d["pos"],
                                  toks["q"][s].cuda(), toks["k"][s].cuda(), toks["v"][s].cuda(),
                                  toks["g"][s].cuda(), d["meta_k"], d["meta_v"],
                                  alpha=wl.alpha).clone())
    torch.cuda.synchronize()
    seqs = [0, 77, 127]
    heads = [0, 13, 31]
    ost = {"state": np64(st["state"][seqs][:, heads]), "kring": np64(st["kring"][seqs][:, heads]),
           "vring": np64(st["vring"][seqs][:, heads]), "pos": st["pos"][seqs].numpy()}
    mk = np64(st["meta_k"][heads])
    mv = np64(st["meta_v"][heads])
    for s in range(6):
        sel = lambda t: np64(t[s][seqs][:, heads])
        ost = oracle.decode_step(ost["state"], ost["kring"], ost["vring"], ost["pos"],
                                 sel(toks["q"]), sel(toks["k"]), sel(toks["v"]), sel(toks["g"]),
                                 mk, mv, wl.scale, wl.alpha)
        assert_close(f"o step {s}", outs[s][seqs][:, heads], ost["o"], torch.bfloat16)
    assert_close("state", d["state"][seqs][:, heads], ost["state"], torch.bfloat16)
    assert np.array_equal(np64(d["kring"][seqs][:, heads]), ost["kring"])
    assert np.array_equal(np64(d["vring"][seqs][:, heads]), ost["vring"])
    assert torch.all(d["pos"].cpu() == wl.pos0 + 6)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("w", [8, 128])
def test_decode_mixed_positions(dtype, w):
    """Sequences at different positions in one batch (an empty history, a
    partly filled window, exactly full, one past full, several wraps) step
    together; every step's output is checked against the oracle's step, the
    state at the end, the rings bit for bit and pos after every step."""
    pos0 = [0, 3, w - 1, w, 5 * w + 2]
    Bd, H, M, n = len(pos0), 2, 4, 7
    cpu, dev = small_problem(400 + w, Bd, H, n, 128, 128, M, dtype)
    gen = torch.Generator().manual_seed(401 + w)
    st0 = torch.randn(Bd, H, 128, 128, generator=gen) * 0.1
    kr0 = (torch.randn(Bd, H, w, 128, generator=gen) * 0.1).to(dtype)
    vr0 = torch.randn(Bd, H, w, 128, generator=gen).to(dtype)
    state, kring, vring = st0.cuda(), kr0.cuda(), vr0.cuda()
    pos = torch.tensor(pos0, dtype=torch.int64, device="cuda")
    ost = {"state": np64(st0), "kring": np64(kr0), "vring": np64(vr0),
           "pos": np.array(pos0, dtype=np.int64)}
    x = {k: np64(v) for k, v in cpu.items()}
    for t in range(n):
        sl = lambda name: dev[name][:, :, t].contiguous()
        o = L.decode_step(state, kring, vring, pos, sl("q"), sl("k"), sl("v"), sl("g"),
                          dev["meta_k"], dev["meta_v"], alpha=0.5)
        ost = oracle.decode_step(ost["state"], ost["kring"], ost["vring"], ost["pos"],
                                 x["q"][:, :, t], x["k"][:, :, t], x["v"][:, :, t],
                                 x["g"][:, :, t], x["meta_k"], x["meta_v"],
                                 1 / math.sqrt(128), 0.5)
        assert_close(f"o step {t}", o, ost["o"], dtype)
        assert np.array_equal(pos.cpu().numpy(), ost["pos"]), (t, pos.cpu(), ost["pos"])
    assert_close("state", state, ost["state"], dtype)
    assert np.array_equal(np64(kring), ost["kring"])
    assert np.array_equal(np64(vring), ost["vring"])


def test_decode_one_launch_per_step_in_a_graph():
    """The step is one kernel launch (the position advances inside it), so a
    run of steps captures into one CUDA graph; replaying it from the same
    starting buffers gives the eager run's outputs, state, rings and pos bit
    for bit."""
    Bd, H, w, M, n = 3, 4, 16, 2, 5
    cpu, dev = small_problem(420, Bd, H, n, 128, 128, M, torch.bfloat16)
    gen = torch.Generator().manual_seed(421)
    init = [(torch.randn(Bd, H, 128, 128, generator=gen) * 0.1).cuda(),
            (torch.randn(Bd, H, w, 128, generator=gen) * 0.1).bfloat16().cuda(),
            torch.randn(Bd, H, w, 128, generator=gen).bfloat16().cuda(),
            torch.tensor([0, 9, 40], dtype=torch.int64, device="cuda")]
    toks = {k: [dev[k][:, :, t].contiguous() for t in range(n)] for k in ("q", "k", "v", "g")}
    outs = [torch.empty(Bd, H, 128, dtype=torch.bfloat16, device="cuda") for _ in range(n)]

    def steps(bufs):
        for t in range(n):
            L.decode_step(*bufs, toks["q"][t], toks["k"][t], toks["v"][t], toks["g"][t],
                          dev["meta_k"], dev["meta_v"], alpha=0.5, o=outs[t])

    eager = [x.clone() for x in init]
    steps(eager)
    eager_out = [o.clone() for o in outs]
    bufs = [x.clone() for x in init]
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        steps([x.clone() for x in init])  # warm-up off the capture
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        steps(bufs)
    for x, y in zip(bufs, init):
        x.copy_(y)
    graph.replay()
    torch.cuda.synchronize()
    for a, b in zip(outs, eager_out):
        assert torch.equal(a, b)
    for a, b in zip(bufs, eager):
        assert torch.equal(a, b)
    assert torch.equal(bufs[3].cpu(), torch.tensor([n, 9 + n, 40 + n]))


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_variable_length_prefill_then_decode(dtype):
    """Prompts of different lengths share one right-padded prefill (padding
    with k = 0 and g = 0, so the state stops at each prompt's end), the
    hand-off takes the per-sequence lengths, and the batch then decodes with
    every sequence at its own position: each sequence's outputs and final
    state match the oracle's forward over its own prompt plus the new tokens."""
    T, w, M, n, alpha, H = 150, 64, 4, 5, 0.5, 2
    lens = [150, 113, 5, 0, 64]
    Bd = len(lens)
    cpu, dev = small_problem(430, Bd, H, T + n, 128, 128, M, dtype)
    pk = cpu["k"][:, :, :T].clone()
    pg = cpu["g"][:, :, :T].clone()
    for b, l in enumerate(lens):  # padding: no key, no decay
        pk[b, :, l:] = 0
        pg[b, :, l:] = 0
    pre = {"q": dev["q"][:, :, :T].contiguous(), "k": pk.cuda(),
           "v": dev["v"][:, :, :T].contiguous(), "g": pg.cuda()}
    fwd = L.hybrid_fwd(pre["q"], pre["k"], pre["v"], pre["g"], dev["meta_k"], dev["meta_v"],
                       w=w, alpha=alpha, want_hT=True)
    state, kring, vring, pos = L.decode_prefill(pre["k"], pre["v"], fwd["hT"], w=w,
                                                lens=torch.tensor(lens))
    torch.cuda.synchronize()
    assert pos.cpu().tolist() == lens
    # decode token j of sequence b is its token lens[b] + j
    x = {k: np64(v) for k, v in cpu.items()}
    outs = []
    for j in range(n):
        idx = [l + j for l in lens]
        tok = {name: torch.stack([cpu[name][b, :, idx[b]] for b in range(Bd)]).cuda()
               for name in ("q", "k", "v", "g")}
        outs.append(L.decode_step(state, kring, vring, pos, tok["q"], tok["k"], tok["v"],
                                  tok["g"], dev["meta_k"], dev["meta_v"], alpha=alpha).clone())
    torch.cuda.synchronize()
    assert pos.cpu().tolist() == [l + n for l in lens]
    for b, l in enumerate(lens):
        sl = lambda name: x[name][b:b + 1, :, :l + n]  # its prompt, then its new tokens
        ref = oracle.hybrid_fwd(sl("q"), sl("k"), sl("v"), sl("g"), x["meta_k"], x["meta_v"],
                                w, 1 / math.sqrt(128), alpha)
        got = torch.stack([o[b] for o in outs], dim=1)[None]
        assert_close(f"decode o [seq {b}, prompt {l}]", got, ref["o"][:, :, l:], dtype)
        assert_close(f"state [seq {b}]", state[b:b + 1], ref["hT"], dtype)


def test_decode_state_save_restore_bitwise():
    Bd, H, w, M = 4, 2, 8, 2
    cpu, dev = small_problem(90, Bd, H, 12, 128, 128, M, torch.bfloat16)
    state = torch.randn(Bd, H, 128, 128, device="cuda") * 0.1
    kring = (torch.randn(Bd, H, w, 128, device="cuda") * 0.1).bfloat16()
    vring = (torch.randn(Bd, H, w, 128, device="cuda") * 0.1).bfloat16()
    pos = torch.tensor([0, 3, 8, 100], dtype=torch.int64, device="cuda")

    def run(st, kr, vr, ps, t0, t1):
        o = []
        for t in range(t0, t1):
            sl = lambda n: dev[n][:, :, t].contiguous()
            o.append(L.decode_step(st, kr, vr, ps, sl("q"), sl("k"), sl("v"), sl("g"),
                                   dev["meta_k"], dev["meta_v"], alpha=0.5).clone())
        return o

    a = [x.clone() for x in (state, kring, vring, pos)]
    run(*a, 0, 6)
    saved = [x.clone() for x in a]
    out1 = run(*a, 6, 12)
    out2 = run(*saved, 6, 12)
    for x, y in zip(out1, out2):
        assert torch.equal(x, y)
    for x, y in zip(a, saved):
        assert torch.equal(x, y)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("T,w", [(0, 8), (5, 16), (150, 64), (300, 128)])
def test_prefill_hand_off_then_decode(dtype, T, w):
    """A chunked prefill of T tokens, the hand-off (state = hT, ring = the last
    w keys and values, pos = T), then n decode steps reproduce the oracle's
    hybrid forward over all T + n tokens."""
    Bd, H, M, n, alpha = 2, 2, 4, 6, 0.5
    cpu, dev = small_problem(70 + T + w, Bd, H, T + n, 128, 128, M, dtype)
    pre = {k: dev[k][:, :, :T].contiguous() for k in ("q", "k", "v", "g")}
    if T:
        fwd = L.hybrid_fwd(pre["q"], pre["k"], pre["v"], pre["g"], dev["meta_k"], dev["meta_v"],
                           w=w, alpha=alpha, want_hT=True)
        hT = fwd["hT"]
    else:
        hT = None
    state, kring, vring, pos = L.decode_prefill(pre["k"], pre["v"], hT, w=w)
    torch.cuda.synchronize()
    assert torch.all(pos.cpu() == T)
    if T:
        assert torch.equal(state, hT)
        for t in range(max(0, T - w), T):  # ring contents: copies, bit-exact
            assert torch.equal(kring[:, :, t % w], pre["k"][:, :, t])
            assert torch.equal(vring[:, :, t % w], pre["v"][:, :, t])
    outs = []
    for t in range(T, T + n):
        sl = lambda name: dev[name][:, :, t].contiguous()
        outs.append(L.decode_step(state, kring, vring, pos, sl("q"), sl("k"), sl("v"), sl("g"),
                                  dev["meta_k"], dev["meta_v"], alpha=alpha).clone())
    dec = torch.stack(outs, dim=2)
    x = {k: np64(v) for k, v in cpu.items()}
    ref = oracle.hybrid_fwd(x["q"], x["k"], x["v"], x["g"], x["meta_k"], x["meta_v"], w,
                            1 / math.sqrt(128), alpha)
    assert_close("decode o after hand-off", dec, ref["o"][:, :, T:], dtype)
    assert_close("decode state after hand-off", state, ref["hT"], dtype)
    assert torch.all(pos.cpu() == T + n)


def _decode_configs(seed=2029):
    rng = random.Random(seed)
    out = []
    for i, T in enumerate([1, 63, 65, 128, 150, 257]):
        Bd = rng.choice([1, 2, 3, 5])
        M = rng.choice([0, 1, 4, 16])
        out.append(dict(idx=i, dtype=[torch.bfloat16, torch.float32][i % 2], T=T,
                        lens=[rng.randint(0, T) for _ in range(Bd)],
                        w=rng.choice([1, 2, 16, 64, 128, 129, 200]), M=M,
                        sink=M > 0 and rng.random() < 0.3, n=rng.choice([1, 3, 8]),
                        alpha=rng.choice([0.0, 0.5, 2.0]), H=rng.choice([1, 2, 3])))
    return out


@pytest.mark.parametrize("cfg", _decode_configs(),
                         ids=lambda c: "case{idx}-T{T}-w{w}-M{M}-Bd{}".format(len(c["lens"]), **c))
def test_decode_sweep(cfg):
    """Seeded mixed cases of the prefill hand-off with per-sequence prompt
    lengths (zero included) followed by n decode steps: windows from one key
    to wider than the ring's prompt part, meta tokens with and without
    values, several mix weights and head counts; every sequence's outputs
    and final state match the oracle's forward over its prompt and new
    tokens."""
    dtype, T, lens, w, M = cfg["dtype"], cfg["T"], cfg["lens"], cfg["w"], cfg["M"]
    sink, n, alpha, H = cfg["sink"], cfg["n"], cfg["alpha"], cfg["H"]
    Bd = len(lens)
    cpu, dev = small_problem(7600 + cfg["idx"], Bd, H, T + n, 128, 128, M, dtype)
    pk = cpu["k"][:, :, :T].clone()
    pg = cpu["g"][:, :, :T].clone()
    for b, l in enumerate(lens):  # padding: no key, no decay
        pk[b, :, l:] = 0
        pg[b, :, l:] = 0
    mk = dev["meta_k"] if M else None
    mv = dev["meta_v"] if (M and not sink) else None
    pre = {"q": dev["q"][:, :, :T].contiguous(), "k": pk.cuda(),
           "v": dev["v"][:, :, :T].contiguous(), "g": pg.cuda()}
    fwd = L.hybrid_fwd(pre["q"], pre["k"], pre["v"], pre["g"], mk, mv, w=w, alpha=alpha,
                       want_hT=True)
    state, kring, vring, pos = L.decode_prefill(pre["k"], pre["v"], fwd["hT"], w=w,
                                                lens=torch.tensor(lens))
    x = {k: np64(v) for k, v in cpu.items()}
    outs = []
    for j in range(n):
        idx = [l + j for l in lens]
        tok = {name: torch.stack([cpu[name][b, :, idx[b]] for b in range(Bd)]).cuda()
               for name in ("q", "k", "v", "g")}
        outs.append(L.decode_step(state, kring, vring, pos, tok["q"], tok["k"], tok["v"],
                                  tok["g"], mk, mv, alpha=alpha).clone())
    torch.cuda.synchronize()
    assert pos.cpu().tolist() == [l + n for l in lens]
    for b, l in enumerate(lens):
        sl = lambda name: x[name][b:b + 1, :, :l + n]
        ref = oracle.hybrid_fwd(sl("q"), sl("k"), sl("v"), sl("g"), x["meta_k"] if M else None,
                                x["meta_v"] if (M and not sink) else None, w,
                                1 / math.sqrt(128), alpha)
        got = torch.stack([o[b] for o in outs], dim=1)[None]
        assert_close(f"decode o [seq {b}, prompt {l}]", got, ref["o"][:, :, l:], dtype)
        assert_close(f"state [seq {b}]", state[b:b + 1], ref["hT"], dtype)


def test_decode_max_window():
    """The largest window the library takes (w = 1024) with the most meta
    tokens (M = 16): 1100 decode steps from an empty state, so the ring wraps,
    against the oracle's forward over the same tokens."""
    Bd, H, T, w, M = 2, 2, 1100, 1024, 16
    cpu, dev = small_problem(1024, Bd, H, T, 128, 128, M, torch.bfloat16)
    alpha = 0.6
    state = torch.zeros(Bd, H, 128, 128, device="cuda")
    kring = torch.zeros(Bd, H, w, 128, dtype=torch.bfloat16, device="cuda")
    vring = torch.zeros_like(kring)
    pos = torch.zeros(Bd, dtype=torch.int64, device="cuda")
    outs = []
    for t in range(T):
        sl = lambda n: dev[n][:, :, t].contiguous()
        outs.append(L.decode_step(state, kring, vring, pos, sl("q"), sl("k"), sl("v"), sl("g"),
                                  dev["meta_k"], dev["meta_v"], alpha=alpha).clone())
    L.lz_device_check()
    dec = torch.stack(outs, dim=2)
    x = {k: np64(v) for k, v in cpu.items()}
    ref = oracle.hybrid_fwd(x["q"], x["k"], x["v"], x["g"], x["meta_k"], x["meta_v"], w,
                            1 / math.sqrt(128), alpha)
    assert_close("decode o", dec, ref["o"], torch.bfloat16)
    assert_close("decode state", state, ref["hT"], torch.bfloat16)
    assert torch.all(pos.cpu() == T)
