"""The multi-GPU host logic of bench.py on CPU: two gloo ranks (the path
shards into independent replicas; the only collectives are the barrier and
the max / sum over ranks of the timing)."""
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    w, r, local = bench.dist_env()
    assert (w, r, local) == (world, rank, rank)
    bench.init_dist(w, backend="gloo", timeout_s=60)
    try:
        bench.barrier()
        dev = torch.device("cpu")
        ms_max, value = bench.aggregate_step(2.0 + rank, 1000, dev)  # rank 1 is the slow one
        total = bench.sum_over_ranks(rank + 1, dev)
        out.put((rank, ms_max, value, total))
    finally:
        dist.destroy_process_group()


def test_two_ranks_aggregate_over_the_slowest_rank():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=5) for _ in range(world))
    for rank, ms_max, value, total in res:
        assert ms_max == 3.0                               # max over ranks
        assert value == pytest.approx(2 * 1000 / 3.0e-3)   # all ranks' tokens / slowest time
        assert total == 3.0


def test_one_rank_is_the_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert not dist.is_initialized()
    assert bench.aggregate_step(4.0, 500, torch.device("cpu")) == (4.0, 500 / 4.0e-3)


def test_reference_arm_prints_on_rank_zero_only():
    """Under torchrun the other ranks of `--impl reference` exit 0 without
    work or output."""
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "1"],
                       env=env, capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""
