"""bench.py's multi-rank plumbing on CPU: two gloo ranks.

Every (sequence, head) is independent, so ranks decode their own replicas
with no data collective; the only cross-rank steps are the barrier and the
max over ranks of the timed duration, which these tests exercise.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    r, w = bench.dist_init("gloo")
    bench.barrier()
    t = 1.5 + r                                    # rank r "took" 1.5 + r seconds
    tmax = bench.reduce_max(t)
    val = bench.weak_scaling_value(1000.0, w, tmax)
    bench.barrier()
    import torch.distributed as dist
    dist.destroy_process_group()
    q.put((r, w, tmax, val))


@pytest.mark.parametrize("world", [2])
def test_max_over_ranks_and_weak_scaling(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r, w, tmax, val in res:
        assert w == world
        assert tmax == 1.5 + (world - 1)           # every rank sees the slowest rank's time
        assert val == 1000.0 * world / tmax


def test_single_process_defaults():
    import bench
    assert bench.reduce_max(3.25) == 3.25
    assert bench.weak_scaling_value(10.0, 1, 2.0) == 5.0


def test_reference_arm_under_two_ranks():
    """bench.py --impl reference launched as two ranks: rank 0 alone runs the
    oracle on the host and prints one line; the other rank exits 0 silently."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           "bench.py", "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"]
    res = subprocess.run(cmd, cwd=root, capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["value"] > 0 and rec["e2e"]["h2d_bytes_per_step"] == 0
