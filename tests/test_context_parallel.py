"""Context parallelism: one sequence split into R contiguous segments, one per
rank, with the state fold and the window halo exchanged between ranks.

CPU: the exchange logic with the oracle's arithmetic, as two gloo processes
(torch.distributed) and as threads, against the oracle over the whole
sequence.  GPU: the CUDA library's kernels for every step, the segments run as
threads of one process on one GPU (each exchange completes on the host before
the next launch), against the oracle over the whole sequence."""
import math
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from gated_linear_sliding_chunked_b200 import context_parallel as CP
import oracle
from parity_util import assert_close, np64, small_problem

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ALPHA = 0.5


def _problem(seed, T, w, M, dtype=torch.float64, device="cpu"):
    cpu, _ = small_problem(seed, 2, 2, T, 128, 128, M, torch.float32, train=True, h0=True,
                           device="cpu")
    cast = {k: (v.to(dtype) if k not in ("g", "h0", "dhT") else v.to(torch.float64 if
            dtype == torch.float64 else torch.float32)) for k, v in cpu.items()}
    return cpu, {k: v.to(device) for k, v in cast.items()}


def _segment(x, r, Ts):
    return {k: (v[:, :, r * Ts:(r + 1) * Ts].contiguous() if k in ("q", "k", "v", "g", "dO")
                else v) for k, v in x.items()}


def _run_rank(comm, ops, x, Ts, w):
    s = _segment(x, comm.rank, Ts)
    o, hT, ctx = CP.cp_forward(comm, ops, s["q"], s["k"], s["v"], s["g"], s["meta_k"],
                               s["meta_v"], w=w, alpha=ALPHA, h0=s["h0"])
    gr = CP.cp_backward(comm, ops, ctx, s["dO"], s["dhT"])
    return {"o": o, "hT": hT, **gr}


def _reference(x, w):
    xs = {k: np64(v) for k, v in x.items()}
    f = oracle.hybrid_fwd(xs["q"], xs["k"], xs["v"], xs["g"], xs["meta_k"], xs["meta_v"], w,
                          1 / math.sqrt(128), ALPHA, xs["h0"])
    b = oracle.hybrid_bwd(xs["q"], xs["k"], xs["v"], xs["g"], xs["meta_k"], xs["meta_v"],
                          xs["dO"], w, 1 / math.sqrt(128), ALPHA, xs["h0"], xs["dhT"])
    return f, b


def _check(res, f, b, tol_fn):
    cat = lambda name: np.concatenate([np64(r[name]) for r in res], axis=2)
    tol_fn("o", cat("o"), f["o"])
    tol_fn("hT", np64(res[-1]["hT"]), f["hT"])
    for name in ("dq", "dk", "dv", "dg"):
        tol_fn(name, cat(name), b[name])
    tol_fn("dh0", np64(res[0]["dh0"]), b["dh0"])
    for name in ("dmeta_k", "dmeta_v"):
        for r in res:  # every rank holds the sum over ranks
            tol_fn(name, np64(r[name]), b[name])


def _exact(name, got, ref):
    err = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert err <= 1e-10, f"{name}: rel-L2 {err:.3e}"


@pytest.mark.parametrize("R,T,w", [(2, 96, 16), (3, 90, 30), (4, 64, 1)])
def test_threads_with_oracle_arithmetic(R, T, w):
    """R ranks as threads, every step from the oracle: the split operator
    equals the oracle's operator over the whole sequence."""
    from cp_oracle_ops import OracleOps
    _, x = _problem(600 + R, T, w, 3)
    res = CP.run_threads(R, lambda comm: _run_rank(comm, OracleOps(), x, T // R, w))
    f, b = _reference(x, w)
    _check(res, f, b, _exact)


def test_segment_shorter_than_the_halo_is_refused():
    from cp_oracle_ops import OracleOps
    _, x = _problem(610, 40, 30, 2)
    with pytest.raises(ValueError, match="shorter than w - 1"):
        CP.run_threads(2, lambda comm: _run_rank(comm, OracleOps(), x, 20, 30))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _gloo_rank(rank, world, port, T, w, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import datetime
    import torch.distributed as dist
    from cp_oracle_ops import OracleOps
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        _, x = _problem(620, T, w, 4)
        res = _run_rank(CP.DistComm(), OracleOps(), x, T // world, w)
        out.put((rank, {k: (None if v is None else v.numpy()) for k, v in res.items()}))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_with_oracle_arithmetic():
    """Two processes over torch.distributed (gloo): all-gathers of the
    segment summaries, the halo sent forward and its gradient sent back, the
    meta gradients summed; the result equals the oracle over the sequence."""
    world, port, T, w = 2, _free_port(), 80, 24
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_gloo_rank, args=(r, world, port, T, w, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = [{k: (None if v is None else torch.from_numpy(v)) for k, v in got[r].items()}
           for r in range(world)]
    _, x = _problem(620, T, w, 4)
    f, b = _reference(x, w)
    _check(res, f, b, _exact)


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("R,T,w,M", [(2, 384, 64, 4), (3, 390, 128, 8), (2, 200, 1, 0)])
def test_segments_on_one_gpu_match_the_oracle(dtype, R, T, w, M):
    """Every step on the GPU through the library (segment decays, folds, row
    copies, the gated and window passes), the R segments as threads that
    take turns on one GPU; compared with the oracle over the whole sequence
    at the path's bars (1e-5 fp32, 2e-2 bf16)."""
    import gated_linear_sliding_chunked_b200 as L
    L.load()
    cpu, x = _problem(640 + R + w, T, w, M, dtype=dtype, device="cuda")
    xr = {k: v for k, v in x.items()}
    if not M:
        xr["meta_k"] = xr["meta_v"] = None
    res = CP.run_threads(R, lambda comm: _run_rank(comm, CP.LibraryOps(), xr, T // R, w))
    torch.cuda.synchronize()
    xc = {k: v.cpu() for k, v in x.items()}
    if not M:
        xc["meta_k"] = xc["meta_v"] = None
    f, b = _reference(xc, w)
    names = ["o", "hT", "dq", "dk", "dv", "dg", "dh0"] + (["dmeta_k", "dmeta_v"] if M else [])
    cat = lambda name: np.concatenate([np64(r[name]) for r in res], axis=2)
    got = {"o": cat("o"), "hT": np64(res[-1]["hT"]), "dh0": np64(res[0]["dh0"])}
    for name in ("dq", "dk", "dv", "dg"):
        got[name] = cat(name)
    for name in ("dmeta_k", "dmeta_v"):
        if M:
            got[name] = np64(res[0][name])
    ref = {**f, **b}
    for name in names:
        assert_close(f"{name} [R={R}]", got[name], ref[name], dtype)
