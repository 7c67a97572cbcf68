"""The multi-rank (replicas) form of bench.py on CPU: two gloo ranks.

bench.py --gpus N runs N independent replicas, each on its own batch of tokens.  The
only collectives are the timing barrier and the max over ranks of the measured time.
These tests drive that host logic, and the reference arm under torchrun, with two
processes on the CPU.
"""
import datetime
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    from routing_dispatch_expert_moe_b200 import inputs as I
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        r, lr, w = bench.env_rank()
        total = bench.max_over_ranks(100.0 + 50.0 * rank)          # rank 1 is the slow one
        value = bench.job_throughput(8192, w, 10, total)
        cfg = I.small_config("replica", T=64, d=64, E=8, k=2, F=64)
        x = np.asarray(I.gen_x(cfg, seed=bench.replica_seed(rank)), np.float64)
        cs = torch.tensor([float(np.abs(x).sum()), float(x[0, 0])], dtype=torch.float64)
        got = [torch.zeros(2, dtype=torch.float64) for _ in range(w)]
        dist.all_gather(got, cs)
        q.put((rank, r, lr, w, total, value, [g.tolist() for g in got]))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time_and_own_batches():
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, r, lr, w, total, value, sums in res:
        assert (r, lr, w) == (rank, rank, 2)
        assert total == 150.0                                       # max over ranks, on every rank
        assert value == pytest.approx(8192 * 2 * 10 / 0.150)        # all ranks' tokens / slowest time
        assert sums[0] != sums[1]                                   # each replica has its own batch
    assert res[0][6] == res[1][6]                                   # and every rank sees the same


def test_reference_arm_under_torchrun_prints_one_line_from_rank_0():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "2", "--warmup", "3", "--workload", "c1_tiny", "--ref-tokens", "8"]
    env = dict(os.environ, OMP_NUM_THREADS="1")
    out = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600, env=env)
    assert out.returncode == 0, out.stderr[-3000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, out.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["steps"] == 2
    assert d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
