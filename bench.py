"""Benchmark of the KV4-RL decode-attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl kv4|reference] [--workload NAME]

One step = one decode step of one attention layer for the whole batch:
kv4_append of one new token per sequence (INT4 page + INT8 side cache), then
kv4_decode_attn (plan, split-K worker kernel over the INT4 pages and INT8
units, exact merge). Metric: KV positions attended per second (sum over
sequences of the context length), and algorithmic HBM GB/s.

Steady state: the cache is prefilled to L0 - 64 positions; step s appends
position L0 - 64 + (s mod 64) and attends over L0 - 63 + (s mod 64) positions,
so the context lengths stay at the workload's distribution however many steps
run. Inputs of all 64 cycle steps are generated on the device before timing;
the cache (hundreds of MB) exceeds the 126 MB L2, so no L2 flush is needed.

Multi-GPU: one process per GPU (torchrun), each with its own batch (its own
seed); no collective on the data path ("replicas only", weak scaling). The
timed region is bracketed by a barrier and a device synchronise; the time is
the max over ranks.

--impl reference times the fp64 C oracle on this machine's host cores on a
bounded sample of the same workload (the reference arm of the comparison).
"""
import argparse
import hashlib
import json
import math
import os
import re
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

CYCLE = 64


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2048)
    ap.add_argument("--warmup", type=int, default=64)
    ap.add_argument("--impl", default="kv4", choices=["kv4", "reference"])
    ap.add_argument("--workload", default="qwen8b", choices=["qwen8b", "async", "long", "evict", "tiny"])
    ap.add_argument("--no-secondary", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--page-evict-only", action="store_true",
                    help="time only kv4_evict_pages on the eviction workload and print its figures")
    ap.add_argument("--learner-only", action="store_true",
                    help="time only smd_masked_attn on the learner workload and print its figures")
    ap.add_argument("--topk-only", action="store_true",
                    help="print only kv_topk_retain on the evict workload at a 10%% budget (the ncu capture's command)")
    ap.add_argument("--masked-only", action="store_true",
                    help="print only the masked decode paths on the evict workload at a 10%% budget "
                         "(the ncu capture's command)")
    ap.add_argument("--prefill-only", action="store_true",
                    help="print only the prefill append of the qwen8b prompt (the ncu capture's command)")
    ap.add_argument("--sink", type=int, default=None, help="override the INT8 sink size (0 = pure INT4)")
    ap.add_argument("--recent", type=int, default=None, help="override the INT8 recent window")
    return ap.parse_args()


# ---------------------------------------------------------------------------- distributed
def dist_setup(args):
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        if args.impl == "kv4":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=300))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, ws):
    if ws == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x, ws):
    if ws == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def aggregate(positions, elapsed_ms, ws):
    """Whole-job throughput: positions attended on all ranks / the slowest rank's time."""
    elapsed_max = max_over_ranks(elapsed_ms, ws)
    return sum_over_ranks(positions, ws) / (elapsed_max / 1e3), elapsed_max


# ---------------------------------------------------------------------------- clocks
class ClockSampler:
    """SM clock and throttle reasons sampled through NVML while the timed region runs."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown", 0x1: "gpu_idle",
               0x2: "applications_clocks_setting", 0x100: "display_clock_setting"}

    def __init__(self, index, period=0.005):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period, self.index, self.ok = period, index, False
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # pragma: no cover
            self.err = str(e)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": len(self.samples), "source": "nvml"}
        return {"sm_mhz": float(np.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples), "source": "nvml"}


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(path))
        return float(d["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs, STREAM-style copy)"
    except Exception:
        return 6650.0, "fallback (6.65 TB/s, earlier measurement on this pool)"


# ---------------------------------------------------------------------------- ncu traffic
PROFILE = os.path.join(ROOT, "profiles", "decode_kernel_qwen8b.json")
KERNEL_SOURCES = ["kv4_decode.cu", "kv4_common.cuh", "kv4_internal.h"]


def kernel_source_hash():
    """sha256 of the decode kernel's sources with comments and whitespace removed."""
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        src = open(os.path.join(ROOT, "compressed_kv_cache_kv4_b200", "csrc", f)).read()
        src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
        src = re.sub(r"//[^\n]*", " ", src)
        h.update(" ".join(src.split()).encode())
    return h.hexdigest()


def ncu_traffic(wbytes):
    """DRAM bytes (read + write) of one decode worker launch from the committed
    ncu figures (profiles/decode_kernel_qwen8b.json), scaled from the captured
    launch's algorithmic bytes to `wbytes`. None if the figures are absent or
    the kernel sources have changed since the capture."""
    try:
        d = json.load(open(PROFILE))
        if d.get("kernel_sources_sha256") != kernel_source_hash():
            return None
        return int(round(float(d["dram_bytes_per_launch"]) * wbytes / float(d["algorithmic_bytes_of_captured_launch"])))
    except (OSError, KeyError, ValueError, TypeError):
        return None


# ---------------------------------------------------------------------------- byte accounting
def region_counts(lens, sink, recent):
    """Per sequence: INT4-attended positions, INT8-attended positions, INT4 pages."""
    lens = np.asarray(lens, np.int64)
    n8 = np.minimum(lens, sink) + np.maximum(0, lens - np.maximum(sink, lens - recent))
    n4 = lens - n8
    hi = lens - recent
    pages = np.where(hi > sink, (hi + 15) // 16 - sink // 16, 0)
    return n4, n8, pages


def worker_bytes(lens, wl):
    """Algorithmic bytes the split-K worker kernel must read for one decode:
    INT4 codes + scales (D + D/8 bytes per position and KV head: 144 at D=128),
    INT8 codes + scales (2 (D + 2): 260), page-table entries of the INT4 pages,
    and the query."""
    n4, n8, pages = region_counts(lens, wl.sink, wl.recent)
    D, H = wl.D, wl.Hkv
    b4 = int(n4.sum()) * H * (D + D // 8)
    b8 = int(n8.sum()) * H * 2 * (D + 2)
    bpt = int(pages.sum()) * 4
    bq = wl.B * wl.Hq * D * 2
    return b4 + b8 + bpt + bq


def step_bytes(lens, wl):
    """Worker bytes + output + append (new K/V in, INT4 and INT8 rows out)."""
    D, H = wl.D, wl.Hkv
    out = wl.B * wl.Hq * D * 2
    append = wl.B * H * (2 * D * 2 + 2 * (D // 2 + 2 * D // 32) + 2 * (D + 2))
    return worker_bytes(lens, wl) + out + append


# ---------------------------------------------------------------------------- kv4 arm
def build_kv4(wl, L0, extra, seed_off, sink=None, recent=None):
    import compressed_kv_cache_kv4_b200 as K
    from compressed_kv_cache_kv4_b200 import synth
    sink = wl.sink if sink is None else sink
    recent = wl.recent if recent is None else recent
    pt, npages = synth.gen_page_table(wl, np.asarray(L0, np.int64) + extra)
    cache = K.KV4Cache(wl.Hkv, wl.D, wl.B, npages, sink, recent)
    ptd = torch.as_tensor(pt, device="cuda")
    return cache, ptd, pt, npages


def prefill(cache, wl, lens_pre, ptd, purpose=1):
    from compressed_kv_cache_kv4_b200 import synth
    k, v, off = synth.gen_kv(wl, device="cuda", lens=lens_pre, purpose=purpose)
    cache.append(k, v, torch.as_tensor(off.astype(np.int32), device="cuda"),
                 torch.zeros(wl.B, dtype=torch.int32, device="cuda"), ptd)
    torch.cuda.synchronize()
    return k, v, off


class Steady:
    """A workload in steady state: the cache is prefilled to L0 - 64 positions
    and step s appends position L0 - 64 + (s mod 64) of every sequence and
    attends over L0 - 63 + (s mod 64) positions, so the lengths keep the
    workload's distribution however many steps run. The inputs of all 64
    cycle steps are resident on the device."""

    def __init__(self, wl, rank=0):
        import compressed_kv_cache_kv4_b200 as K
        from compressed_kv_cache_kv4_b200 import synth
        self.wl = wl
        L0 = wl.lens.astype(np.int64)
        self.lens_pre = np.maximum(L0 - CYCLE, 0).astype(np.int32)
        self.cache, self.ptd, self.pt_np, self.npages = build_kv4(wl, L0, CYCLE, rank)
        self.kpre, self.vpre, self.offpre = prefill(self.cache, wl, self.lens_pre, self.ptd)
        self.step_k, self.step_v, self.step_q, self.lens_old, self.lens_new = [], [], [], [], []
        for c in range(CYCLE):
            kn, vn = synth.gen_step_kv(wl, c, device="cuda")
            self.step_k.append(kn.contiguous())
            self.step_v.append(vn.contiguous())
            self.step_q.append(synth.gen_q(wl, step=c, device="cuda"))
            self.lens_old.append(torch.as_tensor(self.lens_pre + c, dtype=torch.int32, device="cuda"))
            self.lens_new.append(torch.as_tensor(self.lens_pre + c + 1, dtype=torch.int32, device="cuda"))
        self.out = torch.empty((wl.B, wl.Hq, wl.D), dtype=torch.bfloat16, device="cuda")
        self.ws_buf = self.cache.workspace(wl.B, wl.Hq)
        self.K = K

    def step(self, s):
        c = s % CYCLE
        self.K.kv4_append(self.cache.handle, self.step_k[c], self.step_v[c], None, self.lens_old[c], self.ptd)
        self.K.kv4_decode_attn(self.cache.handle, self.step_q[c], self.lens_new[c], self.ptd, self.wl.softmax_scale,
                               self.ws_buf, self.out)

    def positions(self, steps):
        """KV positions attended by the given steps (sum over sequences of the length)."""
        base = int(self.lens_pre.astype(np.int64).sum())
        return float(sum(base + self.wl.B * (s % CYCLE + 1) for s in steps))

    def mean_lens(self):
        return self.lens_pre.astype(np.int64) + CYCLE // 2

    def check(self, what):
        st, bits = self.cache.get_error()
        assert st == self.K.KV4_OK, ("device error " + what, st, bits)

    def timed(self, s0, steps, ws, sampler=None):
        """Device time (ms, this rank) of `steps` consecutive steps from s0,
        bracketed by a barrier and a device synchronise."""
        stream = torch.cuda.current_stream()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(ws)
        torch.cuda.synchronize()
        ctx = sampler if sampler is not None else _Null()
        with ctx:
            e0.record(stream)
            for s in range(s0, s0 + steps):
                self.step(s)
            e1.record(stream)
            torch.cuda.synchronize()
        barrier(ws)
        return e0.elapsed_time(e1)

    def worker_pass(self, n):
        """The decode worker kernel of n consecutive steps, each launch timed with
        CUDA events on its stream (a pass of its own: an event between two kernels
        keeps the second from starting early under programmatic dependent
        launch, so the throughput steps carry none). Returns per-launch us."""
        K = self.K
        K.kv4_timing_enable(n, 1)
        for s in range(n):
            self.step(s)
        torch.cuda.synchronize()
        ms = K.kv4_timing_read_each(0, n)
        K.kv4_timing_disable()
        return [1e3 * x for x in ms]

    def e2e(self, n, ws):
        """The same steps through the public API with host buffers: every step
        uploads its k_new, v_new and q from pinned memory and downloads its output.
        Copies run on a second stream with two buffer sets, so step s+1's upload
        and step s's download overlap the kernels of step s."""
        K, wl = self.K, self.wl
        hk = [t.cpu().pin_memory() for t in self.step_k]
        hv = [t.cpu().pin_memory() for t in self.step_v]
        hq = [t.cpu().pin_memory() for t in self.step_q]
        dk = [torch.empty_like(self.step_k[0]) for _ in range(2)]
        dv = [torch.empty_like(self.step_v[0]) for _ in range(2)]
        dq = [torch.empty_like(self.step_q[0]) for _ in range(2)]
        dout = [torch.empty((wl.B, wl.Hq, wl.D), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
        hout = [torch.empty((wl.B, wl.Hq, wl.D), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        comp = torch.cuda.current_stream()
        copy = torch.cuda.Stream()
        in_ready = [torch.cuda.Event() for _ in range(2)]
        done = [torch.cuda.Event() for _ in range(2)]
        out_copied = [torch.cuda.Event() for _ in range(2)]

        def upload(s):
            i, c = s % 2, s % CYCLE
            with torch.cuda.stream(copy):
                dk[i].copy_(hk[c], non_blocking=True)
                dv[i].copy_(hv[c], non_blocking=True)
                dq[i].copy_(hq[c], non_blocking=True)
                in_ready[i].record(copy)

        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(ws)
        torch.cuda.synchronize()
        e0.record(comp)
        copy.wait_event(e0)
        upload(0)
        for s in range(n):
            i, c = s % 2, s % CYCLE
            comp.wait_event(in_ready[i])
            if s >= 2:
                comp.wait_event(out_copied[i])
            K.kv4_append(self.cache.handle, dk[i], dv[i], None, self.lens_old[c], self.ptd)
            K.kv4_decode_attn(self.cache.handle, dq[i], self.lens_new[c], self.ptd, wl.softmax_scale, self.ws_buf,
                              dout[i])
            done[i].record(comp)
            if s + 1 < n:
                if s >= 1:
                    copy.wait_event(done[(s + 1) % 2])
                upload(s + 1)
            copy.wait_event(done[i])
            with torch.cuda.stream(copy):
                hout[i].copy_(dout[i], non_blocking=True)
                out_copied[i].record(copy)
        comp.wait_event(out_copied[(n - 1) % 2])
        e1.record(comp)
        torch.cuda.synchronize()
        ms = max_over_ranks(e0.elapsed_time(e1), ws)
        positions = sum_over_ranks(self.positions(range(n)), ws)
        h2d = (self.step_k[0].numel() + self.step_v[0].numel() + self.step_q[0].numel()) * 2
        return {"value": positions / (ms / 1e3), "unit": "KV positions/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": dout[0].numel() * 2, "steps": n,
                "overlap": "uploads and downloads on a second stream, two buffer sets"}

    def bf16(self, n=50):
        """The bf16 paged kernel on the same K/V at the prefilled lengths: worker
        kernel per launch (median) and whole call."""
        K, wl = self.K, self.wl
        pages = torch.zeros((self.npages, wl.Hkv, 2, 16, wl.D), dtype=torch.bfloat16, device="cuda")
        for b in range(wl.B):
            L = int(self.lens_pre[b])
            p = torch.arange(L, device="cuda")
            pid = self.ptd[b][p // 16].long()
            slot = (p % 16).long()
            pages[pid, :, 0, slot, :] = self.kpre[int(self.offpre[b]): int(self.offpre[b]) + L]
            pages[pid, :, 1, slot, :] = self.vpre[int(self.offpre[b]): int(self.offpre[b]) + L]
        lens_t = torch.as_tensor(self.lens_pre, dtype=torch.int32, device="cuda")
        o = torch.empty((wl.B, wl.Hq, wl.D), dtype=torch.bfloat16, device="cuda")
        wsb = torch.zeros(K.bf16_paged_workspace_bytes(wl.B, wl.Hq, wl.Hkv, wl.D), dtype=torch.uint8, device="cuda")
        fn = lambda: K.bf16_paged_decode_attn(self.step_q[0], pages, self.ptd, lens_t, wl.softmax_scale, wsb, o,
                                              wl.Hkv)
        call, _ = time_calls(fn, n)
        K.kv4_timing_enable(n, 1)
        for _ in range(n):
            fn()
        torch.cuda.synchronize()
        kern = float(np.median(K.kv4_timing_read_each(1, n)))
        K.kv4_timing_disable()
        pos = int(self.lens_pre.astype(np.int64).sum())
        nbytes = pos * wl.Hkv * 4 * wl.D + int(((self.lens_pre + 15) // 16).sum()) * 4 + wl.B * wl.Hq * wl.D * 2
        peak, _ = peaks()
        del pages
        return {"positions_per_s": pos / (call / 1e3), "call_us": call * 1e3, "worker_us_median": kern * 1e3,
                "worker_gbs": nbytes / (kern / 1e3) / 1e9, "frac_of_peak": nbytes / (kern / 1e3) / 1e9 / peak}

    def close(self):
        self.cache.close()
        for name in ("kpre", "vpre", "step_k", "step_v", "step_q", "out", "ws_buf", "ptd"):
            setattr(self, name, None)
        torch.cuda.empty_cache()


class _Null:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        return False


def roofline(st, worker_us, peak, peak_src):
    """Roofline object of the decode worker kernel: algorithmic bytes at the
    cycle's mean lengths over the median of per-launch event timings."""
    wbytes = worker_bytes(st.mean_lens(), st.wl)
    med = float(np.median(worker_us))
    achieved = wbytes / (med / 1e6) / 1e9
    return {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4), "traffic": None, "kernel": "kv4_decode_kernel (page-major workers)",
            "algorithmic_bytes_per_launch": wbytes, "launches": len(worker_us), "median_us": med,
            "mean_us": float(np.mean(worker_us)), "peak_source": peak_src}


def measure_workload(name, steps=128, warmup=16, ws=1, rank=0, bf16=True):
    """Steady-state figures of one workload: positions/s of whole steps, the
    worker kernel against the roofline, end to end with host buffers, and the
    bf16 kernel on the same data."""
    from compressed_kv_cache_kv4_b200 import synth
    wl = synth.workload(name)
    st = Steady(wl, rank)
    for s in range(warmup):
        st.step(s)
    ms = st.timed(warmup, steps, ws)
    st.check(name)
    peak, src = peaks()
    rf = roofline(st, st.worker_pass(max(64, CYCLE)), peak, src)
    res = {"workload": workload_config(wl)["workload"], "positions_per_step": st.positions(range(steps)) / steps,
           "ms_per_step": ms / steps, "positions_per_s": st.positions(range(warmup, warmup + steps)) / (ms / 1e3),
           "worker_us_median": rf["median_us"], "worker_gbs": rf["achieved"], "worker_frac_of_peak": rf["frac"],
           "worker_launches": rf["launches"], "e2e": st.e2e(64, ws)}
    if bf16:
        res["bf16"] = st.bf16()
        res["kv4_speedup_over_bf16_worker"] = res["bf16"]["worker_us_median"] / rf["median_us"]
    st.check(name)
    st.close()
    return res


def run_kv4(args, ws, rank):
    from compressed_kv_cache_kv4_b200 import synth

    dev = torch.cuda.current_device()
    wl = synth.workload(args.workload)
    if args.sink is not None:
        wl.sink = args.sink
    if args.recent is not None:
        wl.recent = args.recent
    wl.seed += 7919 * rank                      # each rank its own batch (same length law)
    st = Steady(wl, rank)
    for s in range(args.warmup):
        st.step(s)
    torch.cuda.synchronize()
    st.check("before timing")
    # clocks sampled over every measured part: the timed steps, the worker's
    # per-launch pass and the end-to-end steps
    clk = ClockSampler(dev)
    with clk:
        elapsed_ms = st.timed(args.warmup, args.steps, ws)
        st.check("in timed region")
        worker_us = st.worker_pass(max(64, CYCLE))
        e2e = st.e2e(max(64, min(args.steps, 512)), ws)
    st.check("after e2e")
    positions = st.positions(range(args.warmup, args.warmup + args.steps))
    value, elapsed_max = aggregate(positions, elapsed_ms, ws)
    peak, peak_src = peaks()
    rf = roofline(st, worker_us, peak, peak_src)
    rf["traffic"] = ncu_traffic(rf["algorithmic_bytes_per_launch"])
    sbytes = step_bytes(st.mean_lens(), wl)
    res = {
        "elapsed_ms": elapsed_max, "ms_per_step": elapsed_max / args.steps, "value": value,
        "positions_per_step": positions / args.steps, "clocks": clk.summary(),
        "step_gbs": sbytes / (elapsed_max / args.steps / 1e3) / 1e9,
        "worker_avg_us": rf["mean_us"], "roofline": rf,
        "gpu_launches": 3 * args.steps,   # per step: append, decode workers, merge
    }
    # e2e through host buffers: per step H2D of (k_new, v_new, q) from pinned memory, D2H of the output
    res["e2e"] = e2e
    if rank == 0 and not args.no_secondary and args.workload == "qwen8b":
        res["secondary"] = secondary(st)
    if rank == 0 and not args.no_cpu:
        res["cpu_baseline"] = cpu_baseline(wl, st.kpre, st.vpre, st.offpre, st.lens_pre)
        if "secondary" in res:   # the oracle beside the other measured rows
            res["cpu_baseline"]["rows"] = cpu_rows()
    st.close()
    if rank == 0 and not args.no_secondary and args.workload == "qwen8b":
        # the other four workloads in steady state, each next to the bf16 kernel on its data
        res["secondary"]["workloads"] = {name: measure_workload(name) for name in ("async", "long", "evict", "tiny")}
        res["secondary"]["context_parallel"] = cp_secondary()
    return wl, res


def cp_secondary(n_shards=(2, 4, 8), steps=50):
    """Context-parallel decode of the long workload (4 x 131072 positions) on
    this GPU: each page-range shard decoded by kv4_decode_partials, one after
    another, and the partials merged by kv4_merge_partials. On N GPUs each rank
    runs one shard and all-gathers (D + 4) * 4 bytes per (sequence, query head)
    before the merge; that exchange is not measured here (one GPU)."""
    import compressed_kv_cache_kv4_b200 as K
    from compressed_kv_cache_kv4_b200 import cp, synth
    wl = synth.workload("long")
    cache, ptd, _, _ = build_kv4(wl, wl.lens, 0, 0)
    k, v, _ = prefill(cache, wl, wl.lens, ptd)
    del k, v
    q = synth.gen_q(wl, device="cuda")
    lens = torch.as_tensor(wl.lens, device="cuda")
    ws = cache.workspace(wl.B, wl.Hq)
    o = torch.empty((wl.B, wl.Hq, wl.D), dtype=torch.bfloat16, device="cuda")
    single, _ = time_calls(lambda: K.kv4_decode_attn(cache.handle, q, lens, ptd, wl.softmax_scale, ws, o), steps)
    res = {"workload": "long: B=4, L=131072, 32/8 heads, D=128", "single_call_us": single * 1e3,
           "partial_bytes_per_rank": wl.B * wl.Hq * (wl.D + 4) * 4, "exchange": "not measured (one GPU)"}
    for n in n_shards:
        pb, pe = cp.shard_pages(wl.lens, n, wl.sink, wl.recent)
        pbt = [torch.as_tensor(pb[r], device="cuda") for r in range(n)]
        pet = [torch.as_tensor(pe[r], device="cuda") for r in range(n)]
        parts = torch.empty((n, wl.B, wl.Hq, wl.D + 4), dtype=torch.float32, device="cuda")
        per = []
        for r in range(n):
            t, _ = time_calls(lambda: K.kv4_decode_partials(cache.handle, q, lens, ptd, wl.softmax_scale, ws, parts[r],
                                                            pbt[r], pet[r], with_int8=(r == n - 1)), steps)
            per.append(t * 1e3)
        merge, _ = time_calls(lambda: K.kv4_merge_partials(parts, o), steps)
        res["%d_shards" % n] = {"shard_call_us": per, "max_shard_us": max(per), "merge_us": merge * 1e3,
                                "step_us_if_one_gpu_per_shard": max(per) + merge * 1e3}
    st, bits = cache.get_error()
    res["device_error"] = bits
    cache.close()
    return res


def time_calls(fn, n, kind=None):
    import compressed_kv_cache_kv4_b200 as K
    for _ in range(5):
        fn()
    torch.cuda.synchronize()
    if kind is not None:
        K.kv4_timing_enable(n)
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(n):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    call_ms = e0.elapsed_time(e1) / n
    kern_ms = None
    if kind is not None:
        t, c = K.kv4_timing_read(kind)
        K.kv4_timing_disable()
        kern_ms = t / max(c, 1)
    return call_ms, kern_ms


def secondary(st):
    """Comparisons on the qwen8b data: decode only, pure INT4 (no INT8
    protection), the bf16 kernel, the prefill append, the eviction path (top-k +
    masked decode, page eviction) and the learner-side attention."""
    import compressed_kv_cache_kv4_b200 as K
    wl, cache, ptd = st.wl, st.cache, st.ptd
    lens_pre, kpre, vpre, offpre = st.lens_pre, st.kpre, st.vpre, st.offpre
    out = {}
    peak, _ = peaks()
    lens_t = torch.as_tensor(lens_pre, dtype=torch.int32, device="cuda")
    pos = int(lens_pre.astype(np.int64).sum())
    q0 = st.step_q[0]
    o = torch.empty((wl.B, wl.Hq, wl.D), dtype=torch.bfloat16, device="cuda")
    ws_buf = cache.workspace(wl.B, wl.Hq)

    # protected KV4, decode only, at lens_pre
    call, kern = time_calls(lambda: K.kv4_decode_attn(cache.handle, q0, lens_t, ptd, wl.softmax_scale, ws_buf, o),
                            200, kind=0)
    wb = worker_bytes(lens_pre, wl)
    out["kv4_decode_only"] = {"positions_per_s": pos / (call / 1e3), "call_us": call * 1e3, "worker_us": kern * 1e3,
                              "worker_gbs": wb / (kern / 1e3) / 1e9, "frac_of_peak": wb / (kern / 1e3) / 1e9 / peak}

    # pure KV4 (sink = recent = 0): the throughput ratio the KV4-RL review quotes (~94%)
    pure, _, _, _ = build_kv4(wl, wl.lens.astype(np.int64), CYCLE, 0, sink=0, recent=0)
    pure.append(kpre, vpre, torch.as_tensor(offpre.astype(np.int32), device="cuda"),
                torch.zeros(wl.B, dtype=torch.int32, device="cuda"), ptd)
    wsp = pure.workspace(wl.B, wl.Hq)
    callp, kernp = time_calls(lambda: K.kv4_decode_attn(pure.handle, q0, lens_t, ptd, wl.softmax_scale, wsp, o),
                              200, kind=0)
    out["pure_kv4_decode_only"] = {"positions_per_s": pos / (callp / 1e3), "call_us": callp * 1e3,
                                   "worker_us": kernp * 1e3,
                                   "protected_over_pure": (pos / (call / 1e3)) / (pos / (callp / 1e3))}
    pure.close()
    del pure

    # bf16 paged kernel on the same K/V
    out["bf16_decode_only"] = st.bf16(100)
    out["bf16_decode_only"]["kv4_speedup"] = out["bf16_decode_only"]["call_us"] / (call * 1e3)

    # prefill: append of every prompt position (rewrites the same bytes each call)
    offs_t = torch.as_tensor(offpre.astype(np.int32), device="cuda")
    zeros = torch.zeros(wl.B, dtype=torch.int32, device="cuda")
    callp, _ = time_calls(lambda: cache.append(kpre, vpre, offs_t, zeros, ptd), 20)
    T = int(offpre[-1])
    n8 = int(np.minimum(lens_pre, wl.sink + wl.recent).astype(np.int64).sum())
    pbytes = T * wl.Hkv * (4 * wl.D + 18 * wl.D // 16) + n8 * wl.Hkv * 2 * (wl.D + 2) + (wl.B + 1) * 4
    out["prefill_append"] = {"tokens": T, "us": callp * 1e3, "tokens_per_s": T / (callp / 1e3),
                             "gbs": pbytes / (callp / 1e3) / 1e9, "frac_of_peak": pbytes / (callp / 1e3) / 1e9 / peak}

    # eviction workload: top-k (per KV head) + masked decode at 10/30/50/90/100%
    out["evict"] = evict_secondary()
    # learner-side attention under the recorded shadow mask
    out["smd_learner"] = learner_secondary()
    return out


def topk_only(permille=100, reps=20):
    """kv_topk_retain alone on the evict workload's scores (B = 64 x 8 rows of
    16384 positions), each launch timed after a 256 MB read flushes L2."""
    import compressed_kv_cache_kv4_b200 as K
    from compressed_kv_cache_kv4_b200 import synth
    wl = synth.workload("evict")
    k, v, off = synth.gen_kv(wl, device="cuda", lens=wl.lens)
    del v
    scores = synth.gen_scores(wl, k, off, device="cuda")
    del k
    lens = torch.as_tensor(wl.lens, device="cuda")
    L = int(wl.lens.max())
    mask = torch.zeros((wl.B, wl.Hkv, (L + 31) // 32), dtype=torch.int32, device="cuda")
    count = torch.zeros((wl.B, wl.Hkv), dtype=torch.int32, device="cuda")
    flush = torch.ones(256 << 20, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    ms = []
    for r in range(reps + 3):
        flush.max()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        K.kv_topk_retain(scores, lens, permille, mask, count, max_len=L)
        e1.record(stream)
        torch.cuda.synchronize()
        if r >= 3:
            ms.append(e0.elapsed_time(e1))
    med = float(np.median(ms))
    nbytes = wl.B * wl.Hkv * (L * 4 + (L + 31) // 32 * 4)
    return {"rows": wl.B * wl.Hkv, "L": L, "permille": permille, "us_l2_flushed": med * 1e3,
            "gbs": nbytes / (med / 1e3) / 1e9, "retained": int(count.sum().item())}


def masked_only(permille=100, reps=20):
    """Masked decode on the evict workload under a kv_topk_retain mask: the page
    path (kv4_decode_attn with the mask) and the gathered path
    (kv4_decode_attn_masked), each call timed with CUDA events."""
    import compressed_kv_cache_kv4_b200 as K
    from compressed_kv_cache_kv4_b200 import synth
    wl = synth.workload("evict")
    cache, ptd, _, _ = build_kv4(wl, wl.lens, 0, 0)
    k, v, off = prefill(cache, wl, wl.lens, ptd)
    scores = synth.gen_scores(wl, k, off, device="cuda")
    del k, v
    torch.cuda.empty_cache()   # the prompt's K/V are not needed again
    q = synth.gen_q(wl, device="cuda")
    lens = torch.as_tensor(wl.lens, device="cuda")
    L = int(wl.lens.max())
    mask = torch.zeros((wl.B, wl.Hkv, (ptd.shape[1] * 16 + 31) // 32), dtype=torch.int32, device="cuda")
    K.kv_topk_retain(scores, lens, permille, mask, None, max_len=L)
    o = torch.empty((wl.B, wl.Hq, wl.D), dtype=torch.bfloat16, device="cuda")
    ws = cache.workspace(wl.B, wl.Hq)
    page, _ = time_calls(lambda: K.kv4_decode_attn(cache.handle, q, lens, ptd, wl.softmax_scale, ws, o,
                                                   retain_mask=mask), reps)
    gath, _ = time_calls(lambda: cache.decode_masked(q, lens, ptd, wl.softmax_scale, mask, L * permille // 1000,
                                                     out=o), reps)
    unm, _ = time_calls(lambda: K.kv4_decode_attn(cache.handle, q, lens, ptd, wl.softmax_scale, ws, o), reps)
    st = cache.get_error()[0]
    cache.close()
    return {"permille": permille, "page_path_us": page * 1e3, "gathered_us": gath * 1e3, "unmasked_us": unm * 1e3,
            "device_error": st}


def prefill_only(reps=20):
    """The prefill append of the qwen8b prompt (lengths L0 - 64) alone."""
    from compressed_kv_cache_kv4_b200 import synth
    wl = synth.workload("qwen8b")
    lens_pre = np.maximum(wl.lens.astype(np.int64) - CYCLE, 0).astype(np.int32)
    cache, ptd, _, _ = build_kv4(wl, wl.lens, CYCLE, 0)
    k, v, off = prefill(cache, wl, lens_pre, ptd)
    offs_t = torch.as_tensor(off.astype(np.int32), device="cuda")
    zeros = torch.zeros(wl.B, dtype=torch.int32, device="cuda")
    call, _ = time_calls(lambda: cache.append(k, v, offs_t, zeros, ptd), reps)
    st = cache.get_error()[0]
    cache.close()
    return {"positions": int(off[-1]), "us": call * 1e3, "device_error": st}


def evict_secondary(steps=50, page_only=False):
    import compressed_kv_cache_kv4_b200 as K
    from compressed_kv_cache_kv4_b200 import synth
    wl = synth.workload("evict")
    cache, ptd, pt_np, npages = build_kv4(wl, wl.lens, 0, 0)
    k, v, off = prefill(cache, wl, wl.lens, ptd)
    scores = synth.gen_scores(wl, k, off, device="cuda")
    del k, v
    q = synth.gen_q(wl, device="cuda")
    lens = torch.as_tensor(wl.lens, device="cuda")
    L = int(wl.lens.max())
    if page_only:
        o = torch.empty((wl.B, wl.Hq, wl.D), dtype=torch.bfloat16, device="cuda")
        res = {"page_evict": page_evict_secondary(wl, cache, scores, lens, ptd, q, o, cache.workspace(wl.B, wl.Hq))}
        res["device_error"] = cache.get_error()[1]
        cache.close()
        return res
    mstride = (ptd.shape[1] * 16 + 31) // 32
    mask = torch.zeros((wl.B, wl.Hkv, mstride), dtype=torch.int32, device="cuda")
    count = torch.zeros((wl.B, wl.Hkv), dtype=torch.int32, device="cuda")
    o = torch.empty((wl.B, wl.Hq, wl.D), dtype=torch.bfloat16, device="cuda")
    wsb = cache.workspace(wl.B, wl.Hq)
    res = {}
    flush = torch.ones(256 << 20, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    def topk_flushed(permille, reps=20):
        """kv_topk_retain timed alone after a 256 MB read evicts the scores from L2."""
        ms = []
        for r in range(reps + 3):
            flush.max()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda._sleep(100000)   # the GPU stays busy until the launch below is queued
            e0.record(stream)
            K.kv_topk_retain(scores, lens, permille, mask, count, max_len=L)
            e1.record(stream)
            torch.cuda.synchronize()
            if r >= 3:
                ms.append(e0.elapsed_time(e1))
        return float(np.median(ms))

    for permille in (100, 300, 500, 900, 1000):
        tk, _ = time_calls(lambda: K.kv_topk_retain(scores, lens, permille, mask, count, max_len=L), steps)
        tkf = topk_flushed(permille)
        call, kern = time_calls(lambda: K.kv4_decode_attn(cache.handle, q, lens, ptd, wl.softmax_scale, wsb, o,
                                                          retain_mask=mask), steps, kind=0)
        kept = int(count.sum().item()) / wl.Hkv
        # the gathered path: retained INT4 rows packed into compact pages, then decoded
        bound = L * permille // 1000
        callg, _ = time_calls(lambda: cache.decode_masked(q, lens, ptd, wl.softmax_scale, mask, bound, out=o), steps)
        res["%d" % permille] = {"topk_us": tk * 1e3, "topk_us_l2_flushed": tkf * 1e3,
                                "masked_decode_us": call * 1e3, "worker_us": kern * 1e3,
                                "masked_gather_decode_us": callg * 1e3,
                                "retained_positions_per_s": kept / ((tk + call) / 1e3),
                                "topk_gbs": wl.B * wl.Hkv * L * 4 / (tk / 1e3) / 1e9,
                                "topk_gbs_l2_flushed": wl.B * wl.Hkv * L * 4 / (tkf / 1e3) / 1e9}
    call, kern = time_calls(lambda: K.kv4_decode_attn(cache.handle, q, lens, ptd, wl.softmax_scale, wsb, o), steps,
                            kind=0)
    res["unmasked_decode_us"] = call * 1e3
    del flush
    res["page_evict"] = page_evict_secondary(wl, cache, scores, lens, ptd, q, o, wsb)
    st, bits = cache.get_error()
    res["device_error"] = bits
    cache.close()
    return res


def page_evict_bytes(wl, lens, pt_stride, permille, nring):
    """Algorithmic bytes of one kv4_evict_pages launch: the candidate pages'
    scores, the page-table row read and written, the free list and lengths,
    and the ring pages of every head read and written when they rotate."""
    total = 0
    for L in np.asarray(lens, np.int64):
        n = (L + 15) // 16
        jlo = 1 if wl.sink > 0 else 0
        nc = max(0, max(jlo, (L - wl.recent) // 16) - jlo)
        ksel = min(max(n * permille // 1000 - (n - nc), 0), nc)
        e = nc - ksel
        total += 8 + 4
        if e == 0:
            continue
        n, nc, ksel, e = int(n), int(nc), int(ksel), int(e)
        total += (nc * 16 * wl.Hkv * 4 if ksel > 0 else 0) + 2 * pt_stride * 4 + e * 4
        if nring and e % nring:
            total += 2 * wl.Hkv * nring * (32 * wl.D + 64)
    return total


def page_evict_secondary(wl, cache, scores, lens, ptd, q, o, wsb, reps=20):
    """kv4_evict_pages on the eviction workload: each launch timed alone with
    CUDA events, after the cache state is restored and L2 is flushed by a read
    of 256 MB (the inputs fit in L2), with a spin on the stream ahead of the start event so
    that host-side launch work is not timed; then decode on the compacted
    cache."""
    import compressed_kv_cache_kv4_b200 as K
    peak, _ = peaks()
    lens0, pt0, side0 = lens.clone(), ptd.clone(), cache.side.clone()
    flush = torch.ones(256 << 20, dtype=torch.uint8, device="cuda")
    freed = torch.empty_like(ptd)
    cnt = torch.empty_like(lens)
    stream = torch.cuda.current_stream()
    nring = wl.recent // 16
    out = {}
    for permille in (100, 500):
        ms = []
        for r in range(reps + 3):
            lens.copy_(lens0)
            ptd.copy_(pt0)
            cache.side.copy_(side0)
            flush.max()                  # reads 256 MB: L2 holds clean flush lines only
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda._sleep(100000)   # keeps the GPU busy until the launch below is queued
            e0.record(stream)
            K.kv4_evict_pages(cache.handle, scores, permille, lens, ptd, freed, cnt)
            e1.record(stream)
            torch.cuda.synchronize()
            if r >= 3:
                ms.append(e0.elapsed_time(e1))
        t = float(np.mean(ms))
        nbytes = int(page_evict_bytes(wl, wl.lens, ptd.shape[1], permille, nring))
        kept = int(lens.sum().item())
        call, _ = time_calls(lambda: K.kv4_decode_attn(cache.handle, q, lens, ptd, wl.softmax_scale, wsb, o), 20)
        out["%d" % permille] = {"us": t * 1e3, "gbs": nbytes / (t / 1e3) / 1e9,
                                "frac_of_peak": nbytes / (t / 1e3) / 1e9 / peak,
                                "algorithmic_bytes": nbytes, "pages_freed": int(cnt.sum().item()),
                                "positions_after": kept, "decode_after_us": call * 1e3}
    lens.copy_(lens0)
    ptd.copy_(pt0)
    cache.side.copy_(side0)
    del flush
    return out


def bf16_peak():
    try:
        d = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
        return float(d["bf16_tflops"]), "measured (MEASURED_PEAKS.json bf16_tflops, cuBLAS burst)"
    except Exception:
        return 1590.0, "fallback (1.59 PFLOP/s, earlier measurement on this pool)"


def mask_popcount(mask):
    """Set bits of an int32 mask tensor (on its device)."""
    x = mask.to(torch.int64) & 0xFFFFFFFF
    x = x - ((x >> 1) & 0x55555555)
    x = (x & 0x33333333) + ((x >> 2) & 0x33333333)
    x = (x + (x >> 4)) & 0x0F0F0F0F
    return int((((x * 0x01010101) & 0xFFFFFFFF) >> 24).sum().item())


def learner_secondary(steps=20):
    """smd_masked_attn on the learner workload (4 sequences x 8192 positions,
    32/8 heads, D = 128, the recorded-eviction mask, ~46% of keys kept).
    Inputs (q 268 MB, K/V 134 MB, mask 134 MB) exceed L2."""
    import compressed_kv_cache_kv4_b200 as K
    from compressed_kv_cache_kv4_b200 import synth
    wl = synth.workload("learner")
    T = int(wl.lens.max())
    q, k, v = synth.gen_learner_qkv(wl, T, device="cuda")
    mask = synth.gen_shadow_mask(wl, T, device="cuda")
    out = torch.empty((wl.B, T, wl.Hq, wl.D), dtype=torch.bfloat16, device="cuda")
    peak, peak_src = bf16_peak()
    res = {}
    for name, m in (("shadow_mask", mask), ("dense_causal", None)):
        call, _ = time_calls(lambda: K.smd_masked_attn(q, k, v, wl.softmax_scale, out, mask=m), steps)
        pairs = mask_popcount(mask) if m is not None else wl.B * wl.Hkv * T * (T + 1) // 2
        dense_pairs = wl.B * wl.Hkv * T * (T + 1) // 2
        flops = 4.0 * wl.D * wl.G * pairs                 # q.k and p.v per visible (query, key) pair
        dense_flops = 4.0 * wl.D * wl.G * dense_pairs     # what the kernel computes (no block is empty)
        res[name] = {"ms": call, "visible_pairs": pairs, "tflops_algorithmic": flops / (call / 1e3) / 1e12,
                     "tflops_dense_causal": dense_flops / (call / 1e3) / 1e12,
                     "frac_of_bf16_peak": dense_flops / (call / 1e3) / 1e12 / peak,
                     "tokens_per_s": wl.B * T / (call / 1e3)}
    res["peak_tflops"] = peak
    res["peak_source"] = peak_src
    del q, k, v, mask, out
    torch.cuda.empty_cache()
    return res


# ---------------------------------------------------------------------------- CPU oracle
def oracle_build_flags():
    from oracle import build as ob
    return "gcc " + " ".join(ob.FLAGS)


def cpu_model():
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def oracle_threads():
    try:
        import ctypes
        g = ctypes.CDLL(None)
        f = g.omp_get_max_threads
        return int(f())
    except Exception:
        return int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))


def oracle_sample(wl, seqs, k, v, off, lens_pre, q, head=None):
    """One oracle pass (cache byte image + fp64 decode) over the given sequences;
    with `head`, over that KV head only (its G query heads). Returns the time and
    the KV positions covered (a single head counts 1/Hkv of each position)."""
    import oracle as O
    from compressed_kv_cache_kv4_b200 import synth
    qs, hkv, hq = q[seqs], wl.Hkv, wl.Hq
    if head is not None:
        G = wl.Hq // wl.Hkv
        k, v = k[:, head: head + 1], v[:, head: head + 1]
        qs, hkv, hq = qs[:, head * G: (head + 1) * G], 1, G
    kp, vp = synth.pad_batch(k, off, seqs), synth.pad_batch(v, off, seqs)
    kb, vb, qb = synth.bf16_bits(kp), synth.bf16_bits(vp), synth.bf16_bits(qs)
    lens = np.asarray(lens_pre)[seqs].astype(np.int32)
    sh = O.shape(len(seqs), hq, hkv, wl.D, wl.sink, wl.recent)
    npg = [(int(L) + 15) // 16 for L in lens]
    table = np.full((len(seqs), max(npg)), -1, np.int32)
    pos = 0
    for i, n in enumerate(npg):
        table[i, :n] = np.arange(pos, pos + n, dtype=np.int32)
        pos += n
    t0 = time.perf_counter()
    O.write_cache(sh, kb, vb, lens, table, max(pos, 1))
    O.decode(sh, qb, kb, vb, lens, wl.softmax_scale)
    covered = float(lens.astype(np.int64).sum()) * (1.0 if head is None else 1.0 / wl.Hkv)
    return time.perf_counter() - t0, covered


def cpu_baseline(wl, k, v, off, lens_pre, budget_s=20.0):
    import oracle as O
    from compressed_kv_cache_kv4_b200 import synth
    O.lib()
    q = synth.gen_q(wl, device="cuda").cpu()
    kc, vc = k.cpu(), v.cpu()
    total_t, total_pos, seqs_done, b = 0.0, 0, [], 0
    while total_t < budget_s and b < wl.B:
        chunk = list(range(b, min(b + 8, wl.B)))
        t, p = oracle_sample(wl, chunk, kc, vc, off, lens_pre, q)
        total_t += t
        total_pos += p
        seqs_done += chunk
        b += 8
    return {"value": total_pos / total_t, "unit": "KV positions/s", "cores": oracle_threads(), "kind": "oracle",
            "sample": "%d of %d sequences of the %s workload (%d positions): oracle cache image + fp64 decode, "
                      "%.1f s" % (len(seqs_done), wl.B, wl.name, total_pos, total_t),
            "build": oracle_build_flags(), "cpu": cpu_model()}


def cpu_rows():
    """The oracle timed beside the eviction and learner rows, on the host cores:
    page-granular eviction on the whole eviction workload (64 sequences of
    16384 positions, 8 KV heads, 10% of pages kept; seeded uniform scores stand
    in for the H2O-style ones, the oracle's work does not depend on the values),
    and the learner attention under the shadow mask on one sequence of 1024
    positions with the learner heads (32/8, D = 128)."""
    import oracle as O
    from compressed_kv_cache_kv4_b200 import synth
    out = {}
    wl = synth.workload("evict")
    L = int(wl.lens.max())
    rng = np.random.default_rng(1005)
    scores = rng.random((wl.B, wl.Hkv, L), dtype=np.float32)
    npg = L // 16
    pt = np.arange(wl.B * npg, dtype=np.int32).reshape(wl.B, npg)
    t0 = time.perf_counter()
    _, _, _, cnt, _ = O.evict_pages(scores, wl.lens, pt, None, wl.D, 100, wl.sink, wl.recent)
    dt = time.perf_counter() - t0
    out["page_evict"] = {"us": dt * 1e6, "pages_freed": int(cnt.sum()),
                         "sample": "all 64 sequences, 10% of pages kept, fp64 page sums and a full sort"}
    wl = synth.workload("learner", B=1, T=1024)
    T = 1024
    q, k, v = synth.gen_learner_qkv(wl, T)
    mask = synth.gen_shadow_mask(wl, T).numpy().view(np.uint32)
    qb, kb, vb = synth.bf16_bits(q), synth.bf16_bits(k), synth.bf16_bits(v)
    t0 = time.perf_counter()
    O.masked_attn(qb, kb, vb, wl.softmax_scale, mask=mask)
    dt = time.perf_counter() - t0
    pairs = int(sum(bin(int(w)).count("1") for w in mask.reshape(-1)))
    out["smd_learner"] = {"s": dt, "tflops_algorithmic": 4.0 * wl.D * wl.G * pairs / dt / 1e12,
                          "sample": "1 sequence x 1024 positions, 32/8 heads, D = 128, shadow mask "
                                    "(%d visible pairs), fp64" % pairs}
    out["cores"] = oracle_threads()
    return out


def run_reference(args, ws, rank):
    """The oracle as the reference arm: each step one bounded sample of the workload."""
    import oracle as O
    from compressed_kv_cache_kv4_b200 import synth
    wl = synth.workload(args.workload)
    L0 = wl.lens.astype(np.int64)
    lens_pre = np.maximum(L0 - CYCLE, 0).astype(np.int32) + CYCLE // 2
    k, v, off = synth.gen_kv(wl, device="cpu", lens=lens_pre)
    q = synth.gen_q(wl)
    O.lib()
    # Size the per-step sample so warm-up + steps fit in about two minutes: whole
    # sequences when one fits the per-step budget, else (sequence, KV head)
    # pairs, as many as the budget allows (the oracle's cache writer is serial,
    # so a sample's time grows with its size).
    budget = 120.0 / max(1, args.steps + args.warmup)
    t_seq, _ = oracle_sample(wl, [0], k, v, off, lens_pre, q)
    if t_seq <= budget:
        head_mode, per_step = False, max(1, min(wl.B, int(budget / max(t_seq, 1e-6))))
    else:
        t_pair, _ = oracle_sample(wl, [0], k, v, off, lens_pre, q, head=0)
        head_mode, per_step = True, max(1, min(wl.B, int(budget / max(t_pair, 1e-6))))
    total_t, total_pos = 0.0, 0.0
    for s in range(args.warmup + args.steps):
        seqs = [(s * per_step + i) % wl.B for i in range(per_step)]
        if head_mode:
            t, p = oracle_sample(wl, seqs, k, v, off, lens_pre, q, head=s % wl.Hkv)
        else:
            t, p = oracle_sample(wl, seqs, k, v, off, lens_pre, q)
        if s >= args.warmup:
            total_t += t
            total_pos += p
    value = total_pos / total_t
    line = {"metric": "decode-attn KV positions/s and achieved HBM GB/s (% of B200 peak), 8B-like GQA",
            "impl": "reference", "value": value, "unit": "KV positions/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_t / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(wl),
            "cpu_baseline": {"value": value, "unit": "KV positions/s",
                             "cores": min(oracle_threads(), per_step * (1 if head_mode else wl.Hkv)),
                             "kind": "oracle",
                             "sample": "%d %s per step of the %s workload: oracle cache image + fp64 decode"
                                       % (per_step, "(sequence, KV head) pair(s)" if head_mode else "sequence(s)",
                                          wl.name),
                             "build": oracle_build_flags(), "cpu": cpu_model()},
            "e2e": {"value": value, "unit": "KV positions/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


def workload_config(wl):
    return {"workload": "%s: B=%d, Hq=%d, Hkv=%d, D=%d, L %s, sink %d, recent %d, INT4 group 32, 16-token pages"
                        % (wl.name, wl.B, wl.Hq, wl.Hkv, wl.D, length_desc(wl), wl.sink, wl.recent),
            "B": wl.B, "Hq": wl.Hq, "Hkv": wl.Hkv, "head_dim": wl.D, "mean_len": float(wl.lens.mean()),
            "l2": "inputs exceed L2 (no flush)", "parallelism": "replicas (one batch per GPU)"}


def length_desc(wl):
    return {"qwen8b": "~U[1024,8192]", "async": "lognormal(median 4096, sigma 1) clipped [256,32768]",
            "long": "131072", "evict": "16384", "tiny": "(200, 37)"}.get(wl.name, "?")


def main():
    args = parse()
    ws, rank, local = dist_setup(args)
    if args.impl == "reference":
        if rank == 0:
            run_reference(args, ws, rank)
        return
    if args.page_evict_only:
        if rank == 0:
            print(json.dumps(evict_secondary(page_only=True)), flush=True)
        return
    if args.learner_only:
        if rank == 0:
            print(json.dumps(learner_secondary()), flush=True)
        return
    if args.topk_only:
        if rank == 0:
            print(json.dumps(topk_only()), flush=True)
        return
    if args.prefill_only:
        if rank == 0:
            print(json.dumps(prefill_only()), flush=True)
        return
    if args.masked_only:
        if rank == 0:
            print(json.dumps(masked_only()), flush=True)
        return
    wl, res = run_kv4(args, ws, rank)
    if rank == 0:
        line = {"metric": "decode-attn KV positions/s and achieved HBM GB/s (% of B200 peak), 8B-like GQA",
                "value": res["value"], "unit": "KV positions/s", "n_gpus": ws, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": res["ms_per_step"], "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "int4/int8 codes; bf16+fp16 mma, f32 accumulate",
                "data": "synthetic", "config": workload_config(wl), "roofline": res["roofline"],
                "cpu_baseline": res.get("cpu_baseline"), "e2e": res["e2e"], "gpu_launches": res["gpu_launches"],
                "clocks": res["clocks"], "step_hbm_gbs": res["step_gbs"], "worker_avg_us": res["worker_avg_us"],
                "positions_per_step": res["positions_per_step"], "secondary": res.get("secondary")}
        print(json.dumps(line))
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
