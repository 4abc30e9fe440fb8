"""Context parallelism of the hybrid operator: one long sequence over R ranks.

Rank r holds tokens [r*Ts, (r+1)*Ts) of every (batch, head).  The gated
branch's state update S_t = diag(exp(g_t)) S_{t-1} + k_t v_t^T (Lizard
technical summary, section 2a) is linear, so a segment maps the state it
receives to diag(E) h + S (E: its gate product per key dim, S: its final
state from a zero start).  The window branch needs the last w - 1 keys and
values of the previous segment.  The exchange per layer:

forward
  1. every rank: E_r (segment decay) and S_r (gated pass from a zero state);
  2. all-gather (E, S); the state entering segment r is the fold of the
     pairs of segments 0 .. r-1 over the sequence's h0;
  3. every rank: the gated pass again from that state (outputs and the state
     after the segment: the sequence's final state on the last rank);
  4. the last w - 1 keys / values go to the next rank (a halo); the window
     branch runs over [halo; segment] and its first w - 1 outputs are
     dropped; o = o_gla + alpha * o_swa.
backward
  1. every rank: G_r, the gradient of its own outputs with respect to the
     state it received (a gated backward with dhT = 0);
  2. all-gather G; the state gradient leaving segment r is the reverse fold
     of the (E, G) pairs of segments r+1 .. R-1 over the sequence's dhT;
  3. every rank: the gated backward with that dhT (dh0 of rank 0 is the
     sequence's); the window backward over [halo; segment] with dO = 0 on
     the halo rows; the halo rows' key / value gradients go back to the
     previous rank and are added to its last w - 1 rows;
  4. meta-token gradients: summed over ranks.

The arithmetic (decays, folds, passes, row copies and sums) runs in the
CUDA library (lz_cp_segment_decay, lz_cp_fold, lz_cp_rows and the operator's
entry points); this module only orders the calls and moves tensors between
ranks through a `Comm`: `DistComm` (torch.distributed: NCCL between GPUs,
gloo on CPU) or `ThreadComm` (ranks as threads of one process, which lets
one GPU run every segment in turn).  Each step's inputs are taken from
exchanges the host has already completed, so no kernel ever waits on
another rank's kernel.

Requirements: every segment has the same length Ts >= w - 1 (the halo then
comes from the previous rank alone); the gates are fp32 log-gates.  The
sum over ranks of dalpha is not formed here.
"""
from __future__ import annotations

import threading

import torch


# --------------------------------------------------------------------------
# communication between ranks
# --------------------------------------------------------------------------
class DistComm:
    """Exchanges over torch.distributed (any backend; the default group)."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)

    def all_gather(self, t):
        """[world, *t.shape]: every rank's t in rank order."""
        t = t.contiguous()
        parts = [torch.empty_like(t) for _ in range(self.world)]
        self.dist.all_gather(parts, t, group=self.group)
        return torch.stack(parts)

    def _shift(self, t, step):
        t = t.contiguous()
        src, dst = self.rank - step, self.rank + step
        ops = []
        out = None
        if 0 <= src < self.world:
            out = torch.empty_like(t)
            ops.append(self.dist.P2POp(self.dist.irecv, out, src, self.group))
        if 0 <= dst < self.world:
            ops.append(self.dist.P2POp(self.dist.isend, t, dst, self.group))
        if ops:
            for req in self.dist.batch_isend_irecv(ops):
                req.wait()
        return out

    def shift_forward(self, t):
        """Sends t to rank + 1; returns what rank - 1 sent (None on rank 0)."""
        return self._shift(t, 1)

    def shift_backward(self, t):
        """Sends t to rank - 1; returns what rank + 1 sent (None on the last
        rank)."""
        return self._shift(t, -1)

    def all_reduce_sum(self, t):
        t = t.clone()
        self.dist.all_reduce(t, op=self.dist.ReduceOp.SUM, group=self.group)
        return t


class _Hub:
    def __init__(self, world):
        self.world = world
        self.barrier = threading.Barrier(world)
        self.slots = [None] * world


class ThreadComm:
    """Ranks as threads of one process (one per segment), meeting at a
    barrier for every exchange.  Tensors are handed over by reference; the
    threads share the device's default stream, so a tensor read by another
    rank was produced by work enqueued before the barrier."""

    def __init__(self, hub: _Hub, rank: int):
        self.hub, self.rank, self.world = hub, rank, hub.world

    @staticmethod
    def group(world):
        hub = _Hub(world)
        return [ThreadComm(hub, r) for r in range(world)]

    def _exchange(self, t):
        h = self.hub
        h.slots[self.rank] = t
        h.barrier.wait()
        got = list(h.slots)
        h.barrier.wait()
        return got

    def all_gather(self, t):
        return torch.stack([x.contiguous() for x in self._exchange(t)])

    def shift_forward(self, t):
        got = self._exchange(t)
        return got[self.rank - 1] if self.rank > 0 else None

    def shift_backward(self, t):
        got = self._exchange(t)
        return got[self.rank + 1] if self.rank + 1 < self.world else None

    def all_reduce_sum(self, t):
        got = self._exchange(t)
        acc = got[0].clone()
        for x in got[1:]:
            acc += x
        return acc


def run_threads(world, fn):
    """Runs fn(comm) for every rank of a ThreadComm group on its own thread;
    returns the results in rank order (re-raises the first failure)."""
    comms = ThreadComm.group(world)
    res, err = [None] * world, [None] * world

    def body(r):
        try:
            res[r] = fn(comms[r])
        except BaseException as e:  # noqa: BLE001 - handed back to the caller
            err[r] = e
            comms[r].hub.barrier.abort()

    ts = [threading.Thread(target=body, args=(r,)) for r in range(world)]
    for t in ts:
        t.start()
    for t in ts:
        t.join()
    for e in err:
        if e is not None and not isinstance(e, threading.BrokenBarrierError):
            raise e
    for e in err:
        if e is not None:
            raise e
    return res


# --------------------------------------------------------------------------
# the library's kernels
# --------------------------------------------------------------------------
class LibraryOps:
    """The CUDA library's entry points, in the form the exchange uses."""

    def __init__(self):
        import gated_linear_sliding_chunked_b200 as L
        self.L = L

    def segment_decay(self, g):
        return self.L.segment_decay(g)

    def fold(self, E_all, X_all, r, direction, init):
        return self.L.cp_fold(E_all, X_all, r, direction, init)

    def rows(self, dst, dst_off, n, A=None, a_off=0, a_scale=1.0, B=None, b_off=0):
        return self.L.cp_rows(dst, dst_off, n, A, a_off, a_scale, B, b_off)

    def gla_fwd(self, q, k, v, g, h0):
        return self.L.gla_fwd(q, k, v, g, h0, want_hT=True)

    def gla_bwd(self, q, k, v, g, dO, h0, dhT):
        return self.L.gla_bwd(q, k, v, g, dO, h0, dhT, want_dh0=True)

    def swa_fwd(self, q, k, v, meta_k, meta_v, w, scale):
        return self.L.swa_meta_fwd(q, k, v, meta_k, meta_v, w=w, scale=scale)

    def swa_bwd(self, q, k, v, meta_k, meta_v, lse, dO, w, scale, o):
        return self.L.swa_meta_bwd(q, k, v, meta_k, meta_v, lse, dO, w=w, scale=scale, o=o)


# --------------------------------------------------------------------------
# the split operator
# --------------------------------------------------------------------------
def _with_halo(ops, halo, x, hw, zero_halo=False):
    """[halo; x] along the token axis (zeros in place of the halo rows when
    zero_halo)."""
    B, H, Ts, d = x.shape
    out = torch.empty(B, H, hw + Ts, d, dtype=x.dtype, device=x.device)
    ops.rows(out, 0, hw, None if zero_halo else halo)
    ops.rows(out, hw, Ts, x)
    return out


def cp_forward(comm, ops, q, k, v, g, meta_k, meta_v, *, w, alpha, scale=None, h0=None):
    """Forward of this rank's segment (q, k, v [B, H, Ts, d], g fp32 [B, H,
    Ts, dk]; meta tokens and h0 the same on every rank).  Returns (o, hT,
    ctx): o the segment's outputs, hT the state after the segment (the
    sequence's final state on the last rank), ctx what the backward needs."""
    B, H, Ts, dk = q.shape
    r, R = comm.rank, comm.world
    hw = min(w - 1, Ts) if r > 0 else 0  # halo rows this rank receives
    if R > 1 and Ts < w - 1:
        raise ValueError(f"context parallel: segments of {Ts} tokens are shorter than w - 1 = "
                         f"{w - 1}")
    scale = scale if scale is not None else dk ** -0.5
    E = ops.segment_decay(g)
    _, S = ops.gla_fwd(q, k, v, g, None)
    E_all, S_all = comm.all_gather(E), comm.all_gather(S)
    h_in = ops.fold(E_all, S_all, r, 0, h0)
    o, hT = ops.gla_fwd(q, k, v, g, h_in)
    # the halo: this segment's last w - 1 keys and values go to the next rank
    nt = min(w - 1, Ts)
    tails = torch.empty(2, B, H, nt, dk, dtype=k.dtype, device=k.device)
    ops.rows(tails[0], 0, nt, k, a_off=Ts - nt)
    ops.rows(tails[1], 0, nt, v, a_off=Ts - nt)
    halo = comm.shift_forward(tails)
    if hw:
        Xq = _with_halo(ops, None, q, hw, zero_halo=True)
        Xk = _with_halo(ops, halo[0], k, hw)
        Xv = _with_halo(ops, halo[1], v, hw)
    else:
        Xq, Xk, Xv = q, k, v
    o_win, lse = ops.swa_fwd(Xq, Xk, Xv, meta_k, meta_v, w, scale)
    ops.rows(o, 0, Ts, o_win, hw, alpha, o, 0)  # o = o_gla + alpha * o_swa
    ctx = {"q": q, "k": k, "v": v, "g": g, "meta_k": meta_k, "meta_v": meta_v, "Xq": Xq,
           "Xk": Xk, "Xv": Xv, "o_win": o_win, "lse": lse, "h_in": h_in, "E_all": E_all,
           "hw": hw, "w": w, "alpha": alpha, "scale": scale}
    return o, hT, ctx


def cp_backward(comm, ops, ctx, dO, dhT=None):
    """Backward of this rank's segment given dL/do of its outputs and the
    sequence's dL/dhT (used by the last rank; None = 0).  Returns dq, dk, dv,
    dg of the segment, dh0 (the sequence's, on rank 0), and the meta-token
    gradients summed over all ranks."""
    q, k, v, g = ctx["q"], ctx["k"], ctx["v"], ctx["g"]
    B, H, Ts, dk = q.shape
    r = comm.rank
    hw, w, alpha, scale = ctx["hw"], ctx["w"], ctx["alpha"], ctx["scale"]
    # gated branch: the state gradient leaving this segment, then its backward
    G = ops.gla_bwd(q, k, v, g, dO, ctx["h_in"], None)["dh0"]
    G_all = comm.all_gather(G)
    dhT_r = ops.fold(ctx["E_all"], G_all, r, 1, dhT)
    gr = ops.gla_bwd(q, k, v, g, dO, ctx["h_in"], dhT_r)
    # window branch over [halo; segment], dO = 0 on the halo rows
    dOw = torch.empty(B, H, hw + Ts, dO.shape[-1], dtype=dO.dtype, device=dO.device)
    ops.rows(dOw, 0, hw, None)
    ops.rows(dOw, hw, Ts, dO, 0, alpha)
    wr = ops.swa_bwd(ctx["Xq"], ctx["Xk"], ctx["Xv"], ctx["meta_k"], ctx["meta_v"], ctx["lse"],
                     dOw, w, scale, ctx["o_win"])
    dq, dkk, dvv = gr["dq"], gr["dk"], gr["dv"]
    ops.rows(dq, 0, Ts, wr["dq"], hw, 1.0, dq, 0)
    ops.rows(dkk, 0, Ts, wr["dk"], hw, 1.0, dkk, 0)
    ops.rows(dvv, 0, Ts, wr["dv"], hw, 1.0, dvv, 0)
    # the halo rows' key / value gradients belong to the previous rank
    nt = min(w - 1, Ts)
    back = torch.empty(2, B, H, nt, dk, dtype=k.dtype, device=k.device)
    ops.rows(back[0], 0, nt, wr["dk"] if hw else None)
    ops.rows(back[1], 0, nt, wr["dv"] if hw else None)
    got = comm.shift_backward(back)
    if got is not None and nt:
        ops.rows(dkk, Ts - nt, nt, got[0], 0, 1.0, dkk, Ts - nt)
        ops.rows(dvv, Ts - nt, nt, got[1], 0, 1.0, dvv, Ts - nt)
    out = {"dq": dq, "dk": dkk, "dv": dvv, "dg": gr["dg"], "dh0": gr["dh0"] if r == 0 else None}
    for name in ("dmeta_k", "dmeta_v"):
        out[name] = comm.all_reduce_sum(wr[name]) if wr.get(name) is not None else None
    return out
