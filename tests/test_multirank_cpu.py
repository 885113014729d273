"""The multi-process path of bench.py on CPU ranks (gloo, world size 2).

The decode stacks are independent replicas on every rank (no data-path
collective); what the ranks share is host logic: the device time of a run is
the maximum over ranks (one all-reduce), the whole-job value is every rank's
work over that time, and the reference arm runs on rank 0 alone.  These
checks run that logic across two processes without a GPU.
"""

import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    mine = 2.0 + 3.0 * rank                      # rank 1 is the slower one
    worst = bench.max_over_ranks(mine, dist)
    e2e = bench.max_over_ranks(10.0 - rank, dist)   # a second reduction, same order on every rank
    value = bench.replica_throughput(world, 1e9, 4, worst)
    dist.barrier()
    dist.destroy_process_group()
    out.put((rank, worst, e2e, value))


def test_max_over_ranks_and_replica_throughput_on_two_gloo_ranks():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, worst, e2e, value in got:
        assert worst == 5.0                      # the slowest rank's time, on every rank
        assert e2e == 10.0
        assert value == pytest.approx(2 * 1e9 * 4 / 5e-3)


def test_reference_arm_prints_one_line_from_rank_zero():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes", "1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "1", "--cpu-seconds", "0.2",
           "--workload", "single_512"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle"


def test_bench_refuses_a_gpu_count_that_disagrees_with_the_launch():
    # --gpus N must match the ranks the launcher started (WORLD_SIZE); alone it would run one replica
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "2", "--impl", "reference"],
                       cwd=root, env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 2
    assert "WORLD_SIZE=1" in r.stderr and "torch.distributed.run" in r.stderr
