"""The N>1 host logic of bench.py on CPU: two gloo ranks.

The decode path shards by whole sequences ("replicas only": each rank owns its
own batch, no collective on the data path), so the only cross-rank steps are
the timing reductions: the job's time is the slowest rank's, its throughput
the positions of all ranks over that time. The reference arm under torchrun
runs on rank 0 alone; the other ranks exit without work.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, ws, port, q):
    import datetime

    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=ws, timeout=datetime.timedelta(seconds=60))
    try:
        # rank r attends 1000 * (r + 1) positions in 10 * (r + 1) ms
        positions, ms = 1000.0 * (rank + 1), 10.0 * (rank + 1)
        value, elapsed_max = bench.aggregate(positions, ms, ws)
        mx = bench.max_over_ranks(float(rank), ws)
        sm = bench.sum_over_ranks(float(rank + 1), ws)
        bench.barrier(ws)
        q.put((rank, value, elapsed_max, mx, sm))
    finally:
        dist.destroy_process_group()


def test_two_rank_reductions():
    ws = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, ws, port, q)) for r in range(ws)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(ws))
    for rank, value, elapsed_max, mx, sm in got:
        assert elapsed_max == 20.0            # slowest rank
        assert value == pytest.approx(3000.0 / 0.020)
        assert mx == 1.0 and sm == 3.0


def test_reference_arm_under_torchrun_prints_once():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "2", "--warmup", "1", "--workload", "tiny"]
    env = dict(os.environ, OMP_NUM_THREADS="2")
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
