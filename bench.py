#!/usr/bin/env python
"""Throughput of the approximate-then-correct low-bit KV decode-attention step.

One step = jfa_decode_scores + jfa_decode_finish (top-k, correction and merge
in one cluster kernel) over every sequence and head of one decode layer (the Llama-3.1-8B-shaped K3V2 layer by
default: batch 4, 32 query / 8 KV heads, 32768 cached tokens, top-k 256).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--host-resident] [--impl jfa|reference]

Prints one JSON line (rank 0).  Under torchrun each rank runs its own replica
of the workload on its own GPU (weak scaling; the per-(sequence, KV head)
problems are independent, so there is no data-path collective).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode attn: cached KV tokens/s on 1 B200 and % of HBM roofline (K3V2, K4V4)"
L2_BYTES = 126 << 20      # B200 L2


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=None)
    ap.add_argument("--host-resident", action="store_true",
                    help="exact bf16 rows in pinned host memory (zero-copy gather)")
    ap.add_argument("--impl", default="jfa", choices=["jfa", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-rounds", type=int, default=3,
                    help="rounds of the oracle baseline (one segment per host process each)")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the other workloads and variants (the per_config lines)")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--only-fp4", action="store_true",
                    help="print only the NVFP4 step lines (one JSON line per workload)")
    ap.add_argument("--only-channel", action="store_true",
                    help="print only the critical-channel step line of the workload")
    ap.add_argument("--only-onebit", action="store_true",
                    help="print only the 1-bit dense-attention line of the workload")
    return ap.parse_args(argv)


def workload_of(args):
    import workloads as W
    return W.WORKLOADS[args.workload or W.DEFAULT_WORKLOAD]


# ---------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------
def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return rank, world, local


def dist_init(world: int, backend: str):
    import datetime

    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))


def max_over_ranks(x: float, world: int, device=None) -> float:
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------------------
# roofline bookkeeping
# ---------------------------------------------------------------------------
def bytes_per_token(w) -> int:
    """Packed codes + fp16 scales/zeros per (token, KV head)."""
    return 128 * w.key_bits // 8 + 8 + 128 * w.val_bits // 8 + 16


def scan_alg_bytes(w) -> int:
    n_seg = w.batch * w.kv_heads
    return n_seg * w.n_quant * bytes_per_token(w) + w.batch * w.heads * 128 * 2


def step_alg_bytes(w) -> int:
    """Codes + scales, gathered top-k rows, tail rows, q and out."""
    n_seg = w.batch * w.kv_heads
    tail = w.ctx - w.n_quant
    keff = min(w.topk, w.n_quant)
    return (n_seg * (w.n_quant * bytes_per_token(w) + (keff + tail) * 512)
            + w.batch * w.heads * 128 * (2 + 4))


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def kernel_hash() -> str:
    h = hashlib.sha256()
    for f in ("scores.cu", "jfa_common.cuh", "jfa_approx.cuh", "jfa_internal.cuh"):
        with open(os.path.join(ROOT, "bit_kv_cache_jfa_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str):
    """DRAM bytes per scan launch from the committed ncu summary, if it was
    taken on the current scan kernel source (else None)."""
    p = os.path.join(ROOT, "profiles", "scan_traffic.txt")
    if not os.path.exists(p):
        return None
    kh = kernel_hash()
    with open(p) as f:
        for line in f:
            parts = line.split()
            if len(parts) >= 3 and not line.startswith("#") and parts[0] == kh \
                    and parts[1] == workload:
                return float(parts[2])
    return None


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class Clocks:
    """SM clock and clock-event reasons sampled during the timed region: NVML
    polled from a thread every ~2 ms (read-only queries), else nvidia-smi."""

    # NVML clock-event reason bits
    REASONS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
               "hw_thermal_slowdown": 0x40}

    def __init__(self, index: int, enabled: bool):
        self.samples, self.max_mhz, self.reasons = [], 0.0, set()
        self.thread = self.proc = self.path = None
        self.stop_flag = False
        if not enabled:
            return
        try:
            import threading
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))

            def poll():
                while not self.stop_flag:
                    self.samples.append(float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)))
                    bits = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                    for n, v in self.REASONS.items():
                        if bits & v:
                            self.reasons.add(n)
                    time.sleep(0.002)

            self.thread = threading.Thread(target=poll, daemon=True)
            self.thread.start()
            return
        except Exception:
            self.thread = None
        fd, self.path = tempfile.mkstemp(prefix="jfa_clocks_", suffix=".csv")
        os.close(fd)
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={index}", f"--query-gpu={q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.thread is not None:
            self.stop_flag = True
            self.thread.join(timeout=5)
            if not self.samples:
                return None
            return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                    "reasons": sorted(self.reasons), "samples": len(self.samples),
                    "source": "nvml"}
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                p = [x.strip() for x in line.split(",")]
                if len(p) < 9:
                    continue
                try:
                    sm.append(float(p[1]))
                    mx = max(mx, float(p[2]))
                except ValueError:
                    continue
                for n, v in zip(names, p[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "source": "nvidia-smi"}


# ---------------------------------------------------------------------------
# CPU oracle timing (baseline legs only): the oracle as it stands, one
# (sequence, KV head) segment per process, processes started with `spawn`
# ---------------------------------------------------------------------------
def _bf16_bits(t) -> "object":
    """bf16 tensor -> its raw 16-bit patterns as a numpy int16 array (cheap to pickle)."""
    import torch
    return t.contiguous().view(torch.int16).numpy()


def _oracle_worker(jobs, barrier, results, n_rounds: int):
    """One host core: per round, pack its segment (untimed), wait for the
    other workers, then time the oracle's decode step on it."""
    for var in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
        os.environ[var] = "1"
    sys.path.insert(0, ROOT)
    import numpy as np
    import oracle.jfa_oracle as O

    def f64(bits):
        return (bits.astype(np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)

    for r in range(n_rounds):
        job = jobs.get()
        t0 = t1 = 0.0
        if job is not None:
            q, k, v, ctx, kb, vb, topk, scale = job
            kk, vv = f64(k)[None, None], f64(v)[None, None]
            cache = O.pack_cache(kk, vv, ctx, kb, vb)
            qq = f64(q)[None]
        barrier.wait()
        if job is not None:
            t0 = time.time()
            O.decode_step(qq, kk, vv, cache, topk, scale)
            t1 = time.time()
        results.put((r, t0, t1, job is not None))
        barrier.wait()


def time_oracle_pool(w, n_rounds: int, kv_fn, workers: int | None = None):
    """Time the oracle's decode step on `workers` host processes at once, one
    segment each per round (packing untimed), for n_rounds rounds.  Returns
    (tokens/s of a full step, segments timed, seconds in the timed windows,
    workers, per-round windows).  A round's window runs from the first
    worker's start to the last worker's end; a full step (batch * kv_heads
    segments) is extrapolated from the segments per second in the windows."""
    import multiprocessing as mp

    import workloads as W
    n_seg = w.batch * w.kv_heads
    if workers is None:
        workers = max(1, min(os.cpu_count() or 1, n_seg, 32))
    ctx = mp.get_context("spawn")
    jobs, results = ctx.Queue(), ctx.Queue()
    barrier = ctx.Barrier(workers)
    procs = [ctx.Process(target=_oracle_worker, args=(jobs, barrier, results, n_rounds),
                         daemon=True) for _ in range(workers)]
    for pr in procs:
        pr.start()
    q = W.gen_q(w)
    g = w.group
    order = W.sample_segments(w, n_seg, seed=1)
    memo, memo_bytes = {}, 0
    i = 0
    for r in range(n_rounds):
        for _ in range(workers):
            b, h = order[i % n_seg]
            i += 1
            job = memo.get((b, h))
            if job is None:
                k, v = kv_fn(b, h)
                job = (_bf16_bits(q[b, h * g:(h + 1) * g]), _bf16_bits(k), _bf16_bits(v), w.ctx,
                       w.key_bits, w.val_bits, w.topk, W.default_scale(w))
                if memo_bytes < (2 << 30):   # segments recur across rounds: keep them
                    memo[(b, h)] = job
                    memo_bytes += job[1].nbytes + job[2].nbytes
            jobs.put(job)
    windows, done = [], 0
    for r in range(n_rounds):
        rs = [results.get(timeout=600) for _ in range(workers)]
        t0 = min(x[1] for x in rs if x[3])
        t1 = max(x[2] for x in rs if x[3])
        windows.append(t1 - t0)
        done += sum(1 for x in rs if x[3])
    for pr in procs:
        pr.join(timeout=60)
    spent = sum(windows)
    step_s = spent / done * n_seg
    return w.batch * w.ctx / step_s, done, spent, workers, windows


# ---------------------------------------------------------------------------
# reference arm: the oracle itself, timed on the host cores
# ---------------------------------------------------------------------------
def run_reference(args, w):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    import workloads as W
    rounds = args.warmup + args.steps
    _, _, _, workers, windows = time_oracle_pool(
        w, rounds, lambda bb, hh: W.gen_segment(w, bb, hh))
    n_seg = w.batch * w.kv_heads
    per_round = min(workers, n_seg)
    # each step: one round of `workers` segments in parallel, extrapolated to
    # the n_seg segments of a full step
    times = [win / per_round * n_seg for win in windows[args.warmup:]]
    step_s = statistics.mean(times)
    value = w.batch * w.ctx / step_s
    sample = (f"per step, {per_round} of the {n_seg} (sequence, KV head) segments of "
              f"{w.ctx} tokens, one per host process in parallel, extrapolated to a full step")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": step_s * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(w, args),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": workers,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def config_of(w, args, host_resident=None):
    host = args.host_resident if host_resident is None else host_resident
    return {"workload": w.name, "batch": w.batch, "heads": w.heads, "kv_heads": w.kv_heads,
            "ctx": w.ctx, "format": w.fmt, "topk": w.topk,
            "exact_rows": "pinned_host" if host else "hbm",
            "parallelism": f"replicas x{args.gpus}"}


# ---------------------------------------------------------------------------
# the CUDA path
# ---------------------------------------------------------------------------
class Setup:
    """A workload resident on the device: R copies of the packed cache (and of
    the exact rows the correction gathers), together larger than L2, so steps
    that rotate over them read their inputs from HBM without an L2 flush."""

    def __init__(self, w, dev, host_resident: bool):
        import torch

        import bit_kv_cache_jfa_b200 as jfa
        import workloads as W
        self.w, self.dev, self.host = w, dev, host_resident
        self.q = W.gen_q(w).to(dev)
        k_all, v_all = W.gen_kv_device(w, dev, W.gen_q(w))
        probe = jfa.KVCache(w.batch, w.heads, w.kv_heads, w.ctx, w.key_bits, w.val_bits, device=dev)
        self.packed_bytes = probe.layout.groups_bytes
        self.n_copies = 1 + -(-L2_BYTES // max(1, self.packed_bytes))
        del probe
        self.ws = None
        self.copies = []
        for c in range(self.n_copies):
            cache = jfa.KVCache(w.batch, w.heads, w.kv_heads, w.ctx, w.key_bits, w.val_bits,
                                device=dev)
            if self.ws is None:
                self.ws = jfa.Workspace(cache, w.topk, device=dev)
            cache.append(k_all, v_all, self.ws)
            if host_resident:
                ke, ve = k_all.cpu().pin_memory(), v_all.cpu().pin_memory()
            else:
                ke, ve = (k_all, v_all) if c == 0 else (k_all.clone(), v_all.clone())
            self.copies.append((cache, cache.geom(), cache.struct(), ke, ve))
        del k_all, v_all
        torch.cuda.synchronize()
        self.out = torch.empty(w.batch, w.heads, 128, dtype=torch.float32, device=dev)
        self.idx = torch.empty(w.batch, w.kv_heads, w.topk, dtype=torch.int32, device=dev)
        self.stream = torch.cuda.current_stream(dev)
        self.sp = self.stream.cuda_stream
        self.scale = W.default_scale(w)
        self.geom = self.copies[0][1]

    def l2_note(self) -> str:
        return (f"not flushed: the timed steps rotate over {self.n_copies} copies of the packed "
                f"cache and of the exact rows ({self.n_copies} x "
                f"{self.packed_bytes / 2**20:.0f} MiB packed > 126 MB L2), so every step reads "
                f"its inputs from HBM")

    def step(self, i):
        from bit_kv_cache_jfa_b200 import _lib
        _, g, cs, ke, ve = self.copies[i % self.n_copies]
        _lib.check(_lib.jfa_decode_scores(g, cs, self.q, self.scale, self.ws.buf, self.sp),
                   "scores")
        _lib.check(_lib.jfa_decode_finish(g, cs, self.q, self.scale, self.w.topk, self.idx, ke,
                                          ve, int(self.host), self.ws.buf, self.out, self.sp),
                   "finish")

    def step3(self, i):
        from bit_kv_cache_jfa_b200 import _lib
        _, g, cs, ke, ve = self.copies[i % self.n_copies]
        _lib.check(_lib.jfa_decode_scores(g, cs, self.q, self.scale, self.ws.buf, self.sp),
                   "scores")
        _lib.check(_lib.jfa_topk(g, self.w.topk, self.ws.buf, self.idx, self.sp), "topk")
        _lib.check(_lib.jfa_correct_merge(g, cs, self.q, self.scale, self.idx, self.w.topk, ke, ve,
                                          int(self.host), self.ws.buf, self.out, self.sp),
                   "correct_merge")

    def step_blocks(self, i, n_blocks):
        """A step with 128-token block selection: scores, jfa_topk_blocks,
        jfa_correct_merge on the chosen blocks' tokens."""
        from bit_kv_cache_jfa_b200 import _lib
        _, g, cs, ke, ve = self.copies[i % self.n_copies]
        k = n_blocks * 128
        _lib.check(_lib.jfa_decode_scores(g, cs, self.q, self.scale, self.ws.buf, self.sp),
                   "scores")
        _lib.check(_lib.jfa_topk_blocks(g, n_blocks, self.ws.buf, self.idx_blocks, self.sp),
                   "topk_blocks")
        _lib.check(_lib.jfa_correct_merge(g, cs, self.q, self.scale, self.idx_blocks, k, ke, ve,
                                          int(self.host), self.ws.buf, self.out, self.sp),
                   "correct_merge")

    def check_flag(self):
        from bit_kv_cache_jfa_b200 import _lib
        st, flag = _lib.jfa_check_error(self.geom, self.ws.buf, self.sp)
        if flag:
            raise RuntimeError(f"device error flag {flag:#x}")

    def timed(self, fn, steps: int, warmup: int) -> float:
        """ms per call of fn(i): warm-up calls, then `steps` calls back to back
        between one pair of CUDA events on the launching stream."""
        import torch
        for i in range(warmup):
            fn(i)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(self.stream)
        for i in range(steps):
            fn(i)
        e1.record(self.stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / steps

    def scan_ms(self, steps: int) -> float:
        """The scan kernel alone, over the same rotation, on a workspace of its
        own (scan-only launches leave the selection histogram for a finishing
        kernel to consume)."""
        import bit_kv_cache_jfa_b200 as jfa
        from bit_kv_cache_jfa_b200 import _lib
        ws_scan = jfa.Workspace(self.copies[0][0], self.w.topk, device=self.dev)

        def scan(i):
            _, g, cs, _, _ = self.copies[i % self.n_copies]
            _lib.check(_lib.jfa_decode_scores(g, cs, self.q, self.scale, ws_scan.buf, self.sp),
                       "scores")
        ms = self.timed(scan, steps, 3)
        del ws_scan
        return ms

    def summary(self, step_ms: float, scan_ms: float) -> dict:
        w = self.w
        peak, _ = measured_peaks()
        scan_gbs = scan_alg_bytes(w) / (scan_ms / 1e3) / 1e9
        step_gbs = step_alg_bytes(w) / (step_ms / 1e3) / 1e9
        return {"us_per_step": step_ms * 1e3, "tokens_per_s": w.batch * w.ctx / (step_ms / 1e3),
                "scan_us": scan_ms * 1e3, "scan_frac": scan_gbs / peak,
                "step_frac": step_gbs / peak, "step_alg_bytes": step_alg_bytes(w)}


def block_alg_bytes(w, n_blocks: int) -> int:
    """Step bytes with block selection: codes + scales, the chosen blocks'
    exact rows, tail rows, q and out."""
    n_seg = w.batch * w.kv_heads
    tail = w.ctx - w.n_quant
    rows = min(n_blocks * 128, w.n_quant)
    return (n_seg * (w.n_quant * bytes_per_token(w) + (rows + tail) * 512)
            + w.batch * w.heads * 128 * (2 + 4))


def per_config_line(args, dev, name: str, host: bool, n_blocks: int = 0) -> dict:
    import torch

    import workloads as W
    w = W.WORKLOADS[name]
    st = Setup(w, dev, host)
    steps = max(20, min(args.steps, 200))
    if n_blocks:
        st.idx_blocks = torch.empty(w.batch, w.kv_heads, n_blocks * 128, dtype=torch.int32,
                                    device=dev)
        step_ms = st.timed(lambda i: st.step_blocks(i, n_blocks), steps, max(3, args.warmup))
        st.check_flag()
        peak, _ = measured_peaks()
        alg = block_alg_bytes(w, n_blocks)
        d = {"workload": name, "selection": f"{n_blocks} blocks of 128 tokens",
             "exact_rows": "pinned_host" if host else "hbm", "steps": steps,
             "us_per_step": step_ms * 1e3, "tokens_per_s": w.batch * w.ctx / (step_ms / 1e3),
             "step_frac": alg / (step_ms / 1e3) / 1e9 / peak, "step_alg_bytes": alg,
             "calls": "jfa_decode_scores + jfa_topk_blocks + jfa_correct_merge"}
        del st
        torch.cuda.empty_cache()
        return d
    scan_ms = st.scan_ms(steps)
    step_ms = st.timed(st.step, steps, max(3, args.warmup))
    st.check_flag()
    d = {"workload": name, "exact_rows": "pinned_host" if host else "hbm", "steps": steps,
         **st.summary(step_ms, scan_ms)}
    if host:
        # bytes the step gathers across the host link: the top-k rows of every
        # segment (the tail rows sit in the cache's device tail buffer)
        keff = min(w.topk, w.n_quant)
        link = w.batch * w.kv_heads * keff * 512
        d["host_link_bytes_per_step"] = link
    del st
    torch.cuda.empty_cache()
    return d


def per_config_append(args, dev, name: str) -> dict:
    """A decode loop with the append inside the step: every step appends one
    token per sequence at its own position (jfa_append_decode_step: the
    append kernel, flushing full tails into groups, then the scan and the
    finishing kernel).  Two copies of the cache (together larger than L2)
    alternate, each growing by one token per step it runs."""
    import numpy as np
    import torch

    import bit_kv_cache_jfa_b200 as jfa
    from bit_kv_cache_jfa_b200 import _lib
    import workloads as W
    w = W.WORKLOADS[name]
    steps = max(20, min(args.steps, 200))
    warm = max(3, args.warmup)
    grow = (steps + warm) // 2 + 2
    cap = 64 * -(-(w.ctx + grow) // 64)
    k_all, v_all = W.gen_kv_device(w, dev, W.gen_q(w))
    copies = []
    ws = None
    for c in range(2):
        cache = jfa.KVCache(w.batch, w.heads, w.kv_heads, cap, w.key_bits, w.val_bits, device=dev)
        if ws is None:
            ws = jfa.Workspace(cache, w.topk, device=dev)
        cache.append(k_all, v_all, ws)
        ke = torch.zeros(w.batch, w.kv_heads, cap, 128, dtype=torch.bfloat16, device=dev)
        ve = torch.zeros_like(ke)
        ke[:, :, :w.ctx], ve[:, :, :w.ctx] = k_all, v_all
        copies.append([cache, ke, ve, np.full(w.batch, w.ctx, dtype=np.int32)])
    del k_all, v_all
    q = W.gen_q(w).to(dev)
    kn = torch.randn(w.batch, w.kv_heads, 128, device=dev).to(torch.bfloat16)
    vn = torch.randn(w.batch, w.kv_heads, 128, device=dev).to(torch.bfloat16)
    out = torch.empty(w.batch, w.heads, 128, dtype=torch.float32, device=dev)
    idx = torch.empty(w.batch, w.kv_heads, w.topk, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    scale = W.default_scale(w)

    def step(i):
        cache, ke, ve, lens = copies[i % 2]
        _lib.check(_lib.jfa_append_decode_step(cache.geom(), lens, cache.struct(), kn, vn, ke, ve,
                                               q, scale, w.topk, idx, 0, ws.buf, out,
                                               stream.cuda_stream), "append_decode_step")
        lens += 1

    for i in range(warm):
        step(i)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for i in range(steps):
        step(i)
    e1.record(stream)
    torch.cuda.synchronize()
    st, flag = _lib.jfa_check_error(copies[0][0].geom(), ws.buf, stream.cuda_stream)
    if flag:
        raise RuntimeError(f"device error flag {flag:#x}")
    ms = e0.elapsed_time(e1) / steps
    peak, _ = measured_peaks()
    alg = step_alg_bytes(w)
    d = {"workload": name, "selection": "top-k tokens, one token appended per sequence per step",
         "exact_rows": "hbm", "steps": steps, "us_per_step": ms * 1e3,
         "tokens_per_s": w.batch * w.ctx / (ms / 1e3), "step_frac": alg / (ms / 1e3) / 1e9 / peak,
         "calls": "jfa_append_decode_step (append kernel, scan, finishing kernel)",
         "lengths": f"{w.ctx} .. {int(copies[0][3][0])} tokens per sequence (64-token "
                    f"boundaries crossed: tails flushed into groups inside the step)"}
    del copies, ws
    torch.cuda.empty_cache()
    return d


FP4_RECORD_BYTES = 9232    # NVFP4 keys of 128 tokens: codes, block scales, group scales


def fp4_scan_bytes(w) -> int:
    """Bytes the FP4 scan must read: every record of the N_q quantized
    tokens (codes 64 B, block scales 8 B, group scales 1/16 B per token) and
    the selection score it writes per token."""
    n_seg = w.batch * w.kv_heads
    return n_seg * (-(-w.n_quant // 128) * FP4_RECORD_BYTES + w.n_quant * 4)


def fp4_step_bytes(w, n_blocks: int) -> int:
    """FP4 step: the scan's bytes, the chosen blocks' exact K and V rows, the
    tail rows, q and out."""
    n_seg = w.batch * w.kv_heads
    tail = w.ctx - w.n_quant
    rows = min(n_blocks * 128, w.n_quant)
    return fp4_scan_bytes(w) + n_seg * (rows + tail) * 512 + w.batch * w.heads * 128 * (2 + 4)


def per_config_fp4(args, dev, name: str, n_blocks: int) -> dict:
    """The NVFP4 step (Jet-QSparse abstract): jfa_fp4_decode_step = query
    quantization, the tcgen05 FP4 scan, 128-token block selection and the
    exact attention over the chosen blocks and the tail.  Copies of the key
    pool (together larger than L2) and of the exact rows rotate."""
    import torch

    import bit_kv_cache_jfa_b200 as jfa
    from bit_kv_cache_jfa_b200 import _lib
    import workloads as W
    w = W.WORKLOADS[name]
    cap = 128 * -(-w.ctx // 128)
    k_all, v_all = W.gen_kv_device(w, dev, W.gen_q(w))
    q = W.gen_q(w).to(dev)
    probe = jfa.FP4KeyPool(w.batch, w.heads, w.kv_heads, cap, device=dev)
    n_copies = 1 + -(-L2_BYTES // probe.pool.numel())
    ws = jfa.Workspace(probe, 64, device=dev)
    del probe
    copies = []
    for c in range(n_copies):
        pool = jfa.FP4KeyPool(w.batch, w.heads, w.kv_heads, cap, device=dev)
        ke = torch.zeros(w.batch, w.kv_heads, cap, 128, dtype=torch.bfloat16, device=dev)
        ve = torch.zeros_like(ke)
        ke[:, :, :w.ctx], ve[:, :, :w.ctx] = k_all, v_all
        pool.sync(ke, w.ctx, ws)
        copies.append((pool, pool.geom(w.ctx), ke, ve))
    del k_all, v_all
    out = torch.empty(w.batch, w.heads, 128, dtype=torch.float32, device=dev)
    idx = torch.empty(w.batch, w.kv_heads, n_blocks * 128, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    sp = stream.cuda_stream
    scale = W.default_scale(w)

    def step(i):
        pool, g, ke, ve = copies[i % n_copies]
        _lib.check(_lib.jfa_fp4_decode_step(g, pool.pool, q, scale, n_blocks, idx, ke, ve, 0,
                                            ws.buf, out, sp), "fp4_decode_step")

    def scan(i):
        pool, g, _, _ = copies[i % n_copies]
        _lib.check(_lib.jfa_fp4_scores(g, pool.pool, q, scale, ws.buf, sp), "fp4_scores")

    def timed(fn, steps, warm):
        for i in range(warm):
            fn(i)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(stream)
        for i in range(steps):
            fn(i)
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / steps

    steps = max(20, min(args.steps, 200))
    warm = max(3, args.warmup)
    ms = timed(step, steps, warm)
    scan_ms = timed(scan, steps, warm)
    st, flag = _lib.jfa_check_error(copies[0][1], ws.buf, sp)
    if flag:
        raise RuntimeError(f"device error flag {flag:#x}")
    peak, _ = measured_peaks()
    alg = fp4_step_bytes(w, n_blocks)
    d = {"workload": name, "format": "NVFP4 keys, exact bf16 rows",
         "selection": f"{n_blocks} blocks of 128 tokens", "exact_rows": "hbm", "steps": steps,
         "us_per_step": ms * 1e3, "tokens_per_s": w.batch * w.ctx / (ms / 1e3),
         "step_frac": alg / (ms / 1e3) / 1e9 / peak, "step_alg_bytes": alg,
         "scan_us": scan_ms * 1e3,
         "scan_frac": fp4_scan_bytes(w) / (scan_ms / 1e3) / 1e9 / peak,
         "scan_note": "jfa_fp4_scores: query records + the tcgen05 scan (two launches)",
         "copies": n_copies,
         "calls": "jfa_fp4_decode_step (query records, FP4 scan, block selection, sparse "
                  "exact attention)"}
    del copies, ws
    torch.cuda.empty_cache()
    return d


def per_config_channel(args, dev, name: str, r: int) -> dict:
    """Critical-channel selection (TailorKV review): jfa_channel_decode_step =
    scores over the r most important channels of a channel-major key copy,
    top-k, exact attention over the chosen tokens and the tail.  Copies of
    the channel-major keys and of the exact rows rotate (together > L2)."""
    import torch

    import bit_kv_cache_jfa_b200 as jfa
    from bit_kv_cache_jfa_b200 import _lib
    import workloads as W
    w = W.WORKLOADS[name]
    cap = 64 * -(-w.ctx // 64)
    k_all, v_all = W.gen_kv_device(w, dev, W.gen_q(w))
    q = W.gen_q(w).to(dev)
    n_seg = w.batch * w.kv_heads
    scan_bytes = n_seg * w.n_quant * 2 * r
    n_copies = 1 + -(-L2_BYTES // max(1, n_seg * w.n_quant * 2 * 128))
    copies = []
    ws = None
    for c in range(n_copies):
        keys = jfa.ChannelKeys(w.batch, w.heads, w.kv_heads, cap, device=dev)
        if ws is None:
            ws = jfa.Workspace(keys, w.topk, device=dev)
        ke = torch.zeros(w.batch, w.kv_heads, cap, 128, dtype=torch.bfloat16, device=dev)
        ve = torch.zeros_like(ke)
        ke[:, :, :w.ctx], ve[:, :, :w.ctx] = k_all, v_all
        keys.sync(ke, w.ctx)
        copies.append((keys, keys.geom(w.ctx), ke, ve))
    del k_all, v_all
    out = torch.empty(w.batch, w.heads, 128, dtype=torch.float32, device=dev)
    idx = torch.empty(w.batch, w.kv_heads, w.topk, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    sp = stream.cuda_stream
    scale = W.default_scale(w)

    def step(i):
        keys, g, ke, ve = copies[i % n_copies]
        _lib.check(_lib.jfa_channel_decode_step(g, keys.k_t, keys.k_max, q, scale, r, w.topk, idx,
                                                ke, ve, 0, ws.buf, out, sp), "channel_step")

    def scan(i):
        keys, g, _, _ = copies[i % n_copies]
        _lib.check(_lib.jfa_channel_scores(g, keys.k_t, keys.k_max, q, scale, r, ws.buf, sp),
                   "channel_scores")

    def timed(fn, steps, warm):
        for i in range(warm):
            fn(i)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(stream)
        for i in range(steps):
            fn(i)
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / steps

    steps = max(20, min(args.steps, 200))
    warm = max(3, args.warmup)
    ms = timed(step, steps, warm)
    scan_ms = timed(scan, steps, warm)
    st, flag = _lib.jfa_check_error(copies[0][1], ws.buf, sp)
    if flag:
        raise RuntimeError(f"device error flag {flag:#x}")
    peak, _ = measured_peaks()
    tail = w.ctx - w.n_quant
    alg = (scan_bytes + n_seg * (min(w.topk, w.n_quant) + tail) * 512
           + w.batch * w.heads * 128 * (2 + 4))
    d = {"workload": name, "format": f"bf16 channel-major keys, {r} critical channels",
         "selection": f"top-{w.topk} tokens", "exact_rows": "hbm", "steps": steps,
         "us_per_step": ms * 1e3, "tokens_per_s": w.batch * w.ctx / (ms / 1e3),
         "step_frac": alg / (ms / 1e3) / 1e9 / peak, "step_alg_bytes": alg,
         "scan_us": scan_ms * 1e3, "scan_frac": scan_bytes / (scan_ms / 1e3) / 1e9 / peak,
         "copies": n_copies,
         "calls": "jfa_channel_decode_step (channel scores, top-k, sparse exact attention)"}
    del copies, ws
    torch.cuda.empty_cache()
    return d


def per_config_onebit(args, dev, name: str) -> dict:
    """1-bit KV cache with dense attention (TailorKV review): jfa_onebit_attend
    over every quantized token and the exact tail.  Copies of the pool
    (together larger than L2) rotate."""
    import torch

    import bit_kv_cache_jfa_b200 as jfa
    from bit_kv_cache_jfa_b200 import _lib
    import workloads as W
    w = W.WORKLOADS[name]
    cap = 64 * -(-w.ctx // 64)
    k_all, v_all = W.gen_kv_device(w, dev, W.gen_q(w))
    q = W.gen_q(w).to(dev)
    n_seg = w.batch * w.kv_heads
    rec_bytes = n_seg * (w.n_quant // 64) * 3584
    n_copies = 1 + -(-L2_BYTES // max(1, rec_bytes))
    ke = torch.zeros(w.batch, w.kv_heads, cap, 128, dtype=torch.bfloat16, device=dev)
    ve = torch.zeros_like(ke)
    ke[:, :, :w.ctx], ve[:, :, :w.ctx] = k_all, v_all
    del k_all, v_all
    copies = []
    ws = None
    for c in range(n_copies):
        cache = jfa.OneBitCache(w.batch, w.heads, w.kv_heads, cap, device=dev)
        if ws is None:
            ws = jfa.Workspace(cache, 64, device=dev)
        cache.sync(ke, ve, w.ctx, ws)
        copies.append((cache, cache.geom(w.ctx)))
    out = torch.empty(w.batch, w.heads, 128, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    sp = stream.cuda_stream
    scale = W.default_scale(w)

    def step(i):
        cache, g = copies[i % n_copies]
        _lib.check(_lib.jfa_onebit_attend(g, cache.pool, q, scale, ke, ve, 0, ws.buf, out, sp),
                   "onebit_attend")

    steps = max(20, min(args.steps, 200))
    for i in range(max(3, args.warmup)):
        step(i)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for i in range(steps):
        step(i)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    st, flag = _lib.jfa_check_error(copies[0][1], ws.buf, sp)
    if flag:
        raise RuntimeError(f"device error flag {flag:#x}")
    peak, _ = measured_peaks()
    alg = rec_bytes + n_seg * (w.ctx - w.n_quant) * 512 + w.batch * w.heads * 128 * (2 + 4)
    d = {"workload": name, "format": "1-bit keys and values (3584 B per 64 tokens), exact tail",
         "selection": "none: dense attention over every token", "exact_rows": "hbm",
         "steps": steps, "us_per_step": ms * 1e3, "tokens_per_s": w.batch * w.ctx / (ms / 1e3),
         "step_frac": alg / (ms / 1e3) / 1e9 / peak, "step_alg_bytes": alg, "copies": n_copies,
         "calls": "jfa_onebit_attend (one launch)"}
    del copies, ws
    torch.cuda.empty_cache()
    return d


def run_jfa(args, w):
    import torch

    import bit_kv_cache_jfa_b200 as jfa
    from bit_kv_cache_jfa_b200 import _lib

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist_init(world, "nccl")
    jfa.load()

    st = Setup(w, dev, args.host_resident)
    # the scan kernel alone (the roofline object), before the step loop: in
    # the same loop after the step loops some processes measured it ~35 %
    # slower than inside the step, others not; that figure is reported too
    scan_avg = st.scan_ms(args.steps)
    for i in range(max(3, args.warmup)):
        st.step(i)
    torch.cuda.synchronize()
    st.check_flag()

    # timed steps: K decode steps back to back (the call sequence of a step,
    # nothing between the calls), one event pair around all of them
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = Clocks(local, not args.no_clocks)
    barrier(world)
    torch.cuda.synchronize()
    wall0 = time.perf_counter()
    e0.record(st.stream)
    for i in range(args.steps):
        st.step(i)
    e1.record(st.stream)
    torch.cuda.synchronize()
    barrier(world)
    wall = time.perf_counter() - wall0
    clk = clocks.stop()
    ms = e0.elapsed_time(e1) / args.steps
    ms_max = max_over_ranks(ms, world, dev)

    # the same steps as the three separate calls (scores, top-k, correct+merge)
    unfused_ms = st.timed(st.step3, args.steps, 3)
    scan_after = st.scan_ms(args.steps)

    # end to end through the public API, two ways; every step takes q from
    # pinned host memory (the step's first kernel copies it across the host
    # link into the workspace) and the finishing kernel writes out straight
    # into pinned host memory:
    #  - eager: one jfa_decode_step C-ABI call per step (decode_step);
    #  - graph: the step captured once per cache copy (DecodeGraph) and replayed
    q_host = st.q.cpu().pin_memory()
    out_host = torch.empty(st.out.shape, dtype=st.out.dtype).pin_memory()

    def eager_step(i):
        cache, _, _, ke, ve = st.copies[i % st.n_copies]
        jfa.decode_step(cache, q_host, w.topk, ke, ve, st.ws, scale=st.scale, out=out_host,
                        idx=st.idx, exact_on_host=bool(st.host), stream=st.sp)

    eager_ms = st.timed(eager_step, args.steps, max(3, args.warmup))
    graphs = [jfa.DecodeGraph(cache, q_host, w.topk, ke, ve, st.ws, scale=st.scale, out=out_host,
                              idx=st.idx, exact_on_host=bool(st.host))
              for cache, _, _, ke, ve in st.copies]

    def graph_step(i):
        graphs[i % st.n_copies].replay()

    graph_ms = st.timed(graph_step, args.steps, max(3, args.warmup))
    e2e_max = max_over_ranks(min(eager_ms, graph_ms), world, dev)
    e2e_api = "graph replay (DecodeGraph.replay)" if graph_ms <= eager_ms else \
        "eager C-ABI call per step (jfa_decode_step)"
    st.check_flag()
    del graphs

    per_config = []
    if not args.no_per_config and world == 1:
        for name, host in (("llama8b_k4v4_128k", False), ("llama8b_k4v4_128k", True),
                           ("qwen30b_k3v2_32k", False), ("llama70b_k3v2_32k_b8", False),
                           ("llama70b_k4v4_128k_b8", False), ("llama70b_k3v2_8k_b1", False)):
            if name == w.name and host == args.host_resident:
                continue
            per_config.append(per_config_line(args, dev, name, host))
        per_config.append(per_config_line(args, dev, "llama8b_k4v4_128k", False, n_blocks=64))
        per_config.append(per_config_append(args, dev, w.name))
        for name in ("qwen30b_k3v2_32k", "llama8b_k4v4_128k"):
            per_config.append(per_config_fp4(args, dev, name, 64))
        per_config.append(per_config_channel(args, dev, w.name, 16))
        per_config.append(per_config_onebit(args, dev, w.name))

    tokens = w.batch * w.ctx
    value = world * tokens / (ms_max / 1e3)
    peak, peak_kind = measured_peaks()
    summ = st.summary(ms, scan_avg)
    launches = jfa.jfa_decode_step_launches(st.geom, w.topk)

    line = None
    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            k0, v0 = st.copies[0][3], st.copies[0][4]
            kv_cpu = lambda b, h: (k0[b, h].cpu(), v0[b, h].cpu())
            rounds = max(1, args.cpu_rounds)
            val, n, spent, workers, _ = time_oracle_pool(w, rounds, kv_cpu)
            cpu = {"value": val, "unit": "tokens/s", "cores": workers, "kind": "oracle",
                   "sample": f"{n} (sequence, KV head) segments of {w.ctx} tokens, {workers} "
                             f"at a time on {workers} host processes ({rounds} rounds, "
                             f"{spent:.2f} s in the timed windows), extrapolated to the "
                             f"{w.batch * w.kv_heads} segments of a full step"}
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32", "data": "synthetic", "config": config_of(w, args),
            "l2": st.l2_note(),
            "roofline": {"bound": "hbm", "kernel": "scan_kernel (jfa_decode_scores)",
                         "achieved": summ["scan_frac"] * peak, "peak": peak,
                         "peak_kind": peak_kind, "unit": "GB/s", "frac": summ["scan_frac"],
                         "traffic": recorded_traffic(w.name),
                         "alg_bytes_per_launch": scan_alg_bytes(w),
                         "us_per_launch": scan_avg * 1e3,
                         "us_per_launch_after_step_loops": scan_after * 1e3},
            "step_roofline": {"achieved": summ["step_frac"] * peak, "peak": peak, "unit": "GB/s",
                              "frac": summ["step_frac"], "alg_bytes_per_step": step_alg_bytes(w)},
            "cpu_baseline": cpu,
            "e2e": {"value": world * tokens / (e2e_max / 1e3), "unit": "tokens/s",
                    "ms_per_step": e2e_max, "api": e2e_api,
                    "eager_ms_per_step": eager_ms, "graph_ms_per_step": graph_ms,
                    "h2d_bytes_per_step": st.q.numel() * st.q.element_size(),
                    "d2h_bytes_per_step": st.out.numel() * st.out.element_size()},
            "unfused": {"ms_per_step": unfused_ms,
                        "calls": "jfa_decode_scores + jfa_topk + jfa_correct_merge"},
            "per_config": per_config,
            "gpu_launches": launches * args.steps,
            "clocks": clk,
            "wall_s_timed_region": wall,
        }
        print(json.dumps(line), flush=True)
    barrier(world)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def main():
    args = parse()
    w = workload_of(args)
    if args.impl == "reference":
        return run_reference(args, w)
    if args.only_channel:
        import torch
        dev = torch.device("cuda", dist_env()[2])
        torch.cuda.set_device(dev)
        print(json.dumps(per_config_channel(args, dev, w.name, 16)), flush=True)
        return 0
    if args.only_onebit:
        import torch
        dev = torch.device("cuda", dist_env()[2])
        torch.cuda.set_device(dev)
        print(json.dumps(per_config_onebit(args, dev, w.name)), flush=True)
        return 0
    if args.only_fp4:
        import torch
        dev = torch.device("cuda", dist_env()[2])
        torch.cuda.set_device(dev)
        names = [args.workload] if args.workload else ["qwen30b_k3v2_32k", "llama8b_k4v4_128k"]
        for name in names:
            print(json.dumps(per_config_fp4(args, dev, name, 64)), flush=True)
        return 0
    return run_jfa(args, w)


if __name__ == "__main__":
    sys.exit(main())
