"""The N>1 host logic of bench.py on CPU: two gloo ranks.

The decode path shards by whole sequences ("replicas only": each rank owns its
own batch, no collective on the data path), so the only cross-rank steps are
the timing reductions: the job's time is the slowest rank's, its throughput
the positions of all ranks over that time. The reference arm under torchrun
runs on rank 0 alone; the other ranks exit without work.

Context-parallel decode of long sequences has one exchange: the all-gather of
every rank's softmax partials (cp.gather_partials). Its host logic -- the
shard plan covering every INT4 page exactly once, the gather in rank order,
the exact merge -- runs here on two gloo ranks with the oracle's partials.
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


def _cp_rank_main(rank, ws, port, q):
    import datetime

    import numpy as np
    import torch
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import oracle as O
    from compressed_kv_cache_kv4_b200 import cp, synth

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=ws, timeout=datetime.timedelta(seconds=60))
    try:
        wl = synth.workload("qwen8b", B=3)
        wl.lens = np.array([2049, 600, 150], np.int32)
        wl.Hq, wl.Hkv, wl.D, wl.seed = 8, 2, 64, 61
        wl.softmax_scale = 0.125
        k, v, off = synth.gen_kv(wl)
        qq = synth.gen_q(wl)
        sh = O.shape(wl.B, wl.Hq, wl.Hkv, wl.D, wl.sink, wl.recent)
        kb = synth.bf16_bits(synth.pad_batch(k, off, range(wl.B)))
        vb = synth.bf16_bits(synth.pad_batch(v, off, range(wl.B)))
        qd = qq.float().numpy().astype(np.float64)
        pb, pe = cp.shard_pages(wl.lens, ws, wl.sink, wl.recent)
        G = wl.Hq // wl.Hkv
        log2e = 1.0 / np.log(2.0)
        # this rank's partials: INT4 positions of its page range, plus the INT8
        # positions on the last rank, from the oracle's dequantised rows
        part = np.zeros((wl.B, wl.Hq, wl.D + 4), np.float32)
        for b in range(wl.B):
            L = int(wl.lens[b])
            pos = np.arange(int(pb[rank, b]) * 16, int(pe[rank, b]) * 16)
            pos = pos[(pos >= wl.sink) & (pos < L - wl.recent)]
            if rank == ws - 1:
                p8 = np.arange(L)
                pos = np.concatenate([pos, p8[(p8 < wl.sink) | (p8 >= L - wl.recent)]])
            for h in range(wl.Hkv):
                kh, vh = O.dequant_rows(sh, kb, vb, wl.lens, b, h)
                for g in range(G):
                    hq = h * G + g
                    if pos.size == 0:
                        part[b, hq, 0] = -np.inf
                        continue
                    m, l, o = O.attend_rows(qd[b, hq], kh[pos], vh[pos], wl.softmax_scale)
                    part[b, hq, 0], part[b, hq, 1], part[b, hq, 4:] = m * log2e, l, o
        gathered = cp.gather_partials(torch.as_tensor(part)).numpy().astype(np.float64)
        assert gathered.shape == (ws, wl.B, wl.Hq, wl.D + 4)
        assert np.array_equal(gathered[rank], part.astype(np.float64))      # rank order
        full = O.decode(sh, synth.bf16_bits(qq), kb, vb, wl.lens, wl.softmax_scale)
        err = 0.0
        for b in range(wl.B):
            for hq in range(wl.Hq):
                ms, ls, os_ = gathered[:, b, hq, 0] / log2e, gathered[:, b, hq, 1], gathered[:, b, hq, 4:]
                keep = ls > 0
                out = O.merge(ms[keep], ls[keep], os_[keep])
                err = max(err, float(np.abs(out - full[b, hq]).max()))
        # every INT4 page of every sequence lies in exactly one shard
        first, end = cp.int4_pages(wl.lens, wl.sink, wl.recent)
        cover = all(np.array_equal(np.concatenate([np.arange(pb[r, b], pe[r, b]) for r in range(ws)]),
                                   np.arange(first[b], end[b])) for b in range(wl.B))
        q.put((rank, err, cover))
    finally:
        dist.destroy_process_group()


def test_two_rank_context_parallel_exchange():
    ws = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_cp_rank_main, args=(r, ws, port, q)) for r in range(ws)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(300)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(ws))
    for rank, err, cover in got:
        assert cover
        assert err <= 1e-5, err       # fp32 partials, fp64 merge
