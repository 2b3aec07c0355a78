"""bench.py's multi-rank plumbing on CPU: two gloo ranks, the whole-job
value is all ranks' bytes over the slowest rank's time, and every rank
agrees on it (the collective steps are the same on every rank)."""
import os
import socket
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    w, r, _ = bench.dist_init()
    assert (w, r) == (world, rank)
    # rank r moved (r + 1) GB in (r + 1) * 0.5 s
    gbs, t = bench.aggregate((rank + 1) * 1e9, (rank + 1) * 0.5, w)
    q.put((rank, gbs, t))
    dist.destroy_process_group()


def test_two_rank_aggregation():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get() for _ in range(2))
    for _, gbs, t in res:
        assert t == pytest.approx(1.0)          # slowest rank's time
        assert gbs == pytest.approx(3.0)        # (1 + 2) GB / 1 s


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    gbs, t = bench.aggregate(2e9, 0.5, 1)
    assert gbs == pytest.approx(4.0) and t == 0.5


def test_reference_arm_under_two_ranks():
    """bench.py --impl reference under torchrun with 2 CPU ranks (gloo): rank 0
    alone times the oracle and prints the one JSON line; the other rank exits
    0 without work."""
    import json
    import subprocess
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--config", "opt_tiny_f32", "--steps", "2", "--warmup", "3"]
    out = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT,
                         env={**os.environ, "CUDA_VISIBLE_DEVICES": ""})
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["steps"] >= 1
