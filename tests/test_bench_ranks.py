"""Multi-rank aggregation of bench.py on CPU: two gloo ranks (one process per rank, as torchrun
starts them) each report their own time; every rank must get the slowest one, and the whole-job
rate divides the units of all ranks by it. GPUs run replicas, so this max-over-ranks step is the
only exchange between ranks."""
import datetime
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank: int, world: int, port: int, times, q) -> None:
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        slowest = bench.max_over_ranks(times[rank], world, "cpu")
        q.put((rank, slowest, bench.whole_job_rate(512 * 5, world, slowest)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("times", [(0.75, 1.25), (2.0, 0.5)])
def test_max_over_ranks_gloo(times):
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, times, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    slowest = max(times)
    for rank, m, rate in got:
        assert m == slowest
        assert rate == pytest.approx(2 * 512 * 5 / slowest)


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.whole_job_rate(100, 1, 2.0) == 50.0


def test_reference_arm_under_torchrun_two_ranks():
    """`--impl reference` launched like the GPU arm (torchrun, two ranks; gloo on this host): rank 0
    alone runs the oracle and prints the one JSON line, the other rank exits 0 without work."""
    import json
    import subprocess
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py", "--impl", "reference",
           "--gpus", "2", "--model", "tiny", "--prompt", "16", "--decode", "32", "--steps", "2", "--warmup", "3"]
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="", OMP_NUM_THREADS="2")
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
