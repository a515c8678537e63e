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
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-clocks", action="store_true")
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
# CPU oracle timing (baseline leg only)
# ---------------------------------------------------------------------------
def oracle_cores() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def time_oracle(w, seconds: float, kv_fn, segs=None):
    """Time the oracle's decode step on whole (sequence, KV head) segments of
    the workload (packing untimed) until about `seconds` of CPU work or the
    end of `segs`; returns (tokens/s in the metric's unit, segments, seconds)."""
    import oracle.jfa_oracle as O
    import workloads as W
    q = W.gen_q(w)
    if segs is None:
        segs = W.sample_segments(w, w.batch * w.kv_heads, seed=1)
    g = w.group
    done, spent = 0, 0.0
    for (b, h) in segs:
        k, v = kv_fn(b, h)
        kk = k.double().numpy()[None, None]
        vv = v.double().numpy()[None, None]
        qq = q[b:b + 1, h * g:(h + 1) * g].double().numpy()
        cache = O.pack_cache(kk, vv, w.ctx, w.key_bits, w.val_bits)
        t0 = time.perf_counter()
        O.decode_step(qq, kk, vv, cache, w.topk, W.default_scale(w))
        spent += time.perf_counter() - t0
        done += 1
        if spent >= seconds:
            break
    # one full step covers batch * kv_heads segments of ctx tokens each
    step_s = spent / done * (w.batch * w.kv_heads)
    return w.batch * w.ctx / step_s, done, spent


# ---------------------------------------------------------------------------
# reference arm: the oracle itself, timed on the host cores
# ---------------------------------------------------------------------------
def run_reference(args, w):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    import workloads as W
    times = []
    n_seg = w.batch * w.kv_heads
    for i in range(args.warmup + args.steps):
        seg = divmod(i % n_seg, w.kv_heads)
        val, n, s = time_oracle(w, 0.0, lambda bb, hh: W.gen_segment(w, bb, hh), segs=[seg])
        if i >= args.warmup:
            times.append(w.batch * w.ctx / val)     # seconds per full step (extrapolated)
    step_s = statistics.mean(times)
    value = w.batch * w.ctx / step_s
    cores = oracle_cores()
    sample = (f"one (sequence, KV head) segment of {w.ctx} tokens per step, extrapolated to "
              f"the {w.batch * w.kv_heads} segments of a full step")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": step_s * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(w, args),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def config_of(w, args, n_copies=0, packed_bytes=0):
    return {"workload": w.name, "batch": w.batch, "heads": w.heads, "kv_heads": w.kv_heads,
            "ctx": w.ctx, "format": w.fmt, "topk": w.topk,
            "exact_rows": "pinned_host" if args.host_resident else "hbm",
            "l2": (f"not flushed: the timed steps rotate over {n_copies} copies of the packed "
                   f"cache and of the exact rows ({n_copies} x {packed_bytes / 2**20:.0f} MiB "
                   f"packed > 126 MB L2), so every step reads its inputs from HBM")
                  if n_copies else "host run",
            "parallelism": f"replicas x{args.gpus}"}


# ---------------------------------------------------------------------------
# the CUDA path
# ---------------------------------------------------------------------------
def run_jfa(args, w):
    import torch

    import bit_kv_cache_jfa_b200 as jfa
    from bit_kv_cache_jfa_b200 import _lib
    import workloads as W

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist_init(world, "nccl")
    jfa.load()

    q = W.gen_q(w).to(dev)
    k_all, v_all = W.gen_kv_device(w, dev, W.gen_q(w))
    # R copies of the cache (and of the exact rows the correction gathers),
    # together larger than L2: the timed steps rotate over them, so every
    # step reads its inputs from HBM without an L2 flush between steps
    probe = jfa.KVCache(w.batch, w.heads, w.kv_heads, w.ctx, w.key_bits, w.val_bits, device=dev)
    packed_bytes = probe.layout.groups_bytes
    n_copies = 1 + -(-L2_BYTES // max(1, packed_bytes))
    del probe
    ws = None
    copies = []
    for c in range(n_copies):
        cache = jfa.KVCache(w.batch, w.heads, w.kv_heads, w.ctx, w.key_bits, w.val_bits, device=dev)
        if ws is None:
            ws = jfa.Workspace(cache, w.topk, device=dev)
        cache.append(k_all, v_all, ws)
        if args.host_resident:
            ke, ve = k_all.cpu().pin_memory(), v_all.cpu().pin_memory()
        else:
            ke, ve = (k_all, v_all) if c == 0 else (k_all.clone(), v_all.clone())
        copies.append((cache, cache.geom(), cache.struct(), ke, ve))
    del k_all, v_all
    torch.cuda.synchronize()
    out = torch.empty(w.batch, w.heads, 128, dtype=torch.float32, device=dev)
    idx = torch.empty(w.batch, w.kv_heads, w.topk, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    sp = stream.cuda_stream
    scale = W.default_scale(w)
    host = 1 if args.host_resident else 0
    geom = copies[0][1]

    def step(i, wsb=None):
        _, g, cs, ke, ve = copies[i % n_copies]
        _lib.check(_lib.jfa_decode_scores(g, cs, q, scale, ws.buf, sp), "scores")
        _lib.check(_lib.jfa_decode_finish(g, cs, q, scale, w.topk, idx, ke, ve,
                                          host, ws.buf, out, sp), "finish")

    for i in range(max(3, args.warmup)):
        step(i)
    torch.cuda.synchronize()
    st, flag = _lib.jfa_check_error(geom, ws.buf, sp)
    if flag:
        raise RuntimeError(f"device error flag {flag:#x}")

    # timed steps: K decode steps back to back (the call sequence of a step,
    # nothing between the calls), one event pair around all of them
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = Clocks(local, not args.no_clocks)
    barrier(world)
    torch.cuda.synchronize()
    wall0 = time.perf_counter()
    e0.record(stream)
    for i in range(args.steps):
        step(i)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    wall = time.perf_counter() - wall0
    clk = clocks.stop()
    ms = e0.elapsed_time(e1) / args.steps
    ms_max = max_over_ranks(ms, world, dev)

    # the same steps as the three separate calls (scores, top-k, correct+merge)
    # instead of the fused finishing kernel, for reference
    def step3(i):
        _, g, cs, ke, ve = copies[i % n_copies]
        _lib.check(_lib.jfa_decode_scores(g, cs, q, scale, ws.buf, sp), "scores")
        _lib.check(_lib.jfa_topk(g, w.topk, ws.buf, idx, sp), "topk")
        _lib.check(_lib.jfa_correct_merge(g, cs, q, scale, idx, w.topk, ke, ve, host, ws.buf, out,
                                          sp), "correct_merge")

    for i in range(3):
        step3(i)
    u0, u1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    u0.record(stream)
    for i in range(args.steps):
        step3(i)
    u1.record(stream)
    torch.cuda.synchronize()
    unfused_ms = u0.elapsed_time(u1) / args.steps

    # the scan kernel alone (roofline): its own launches back to back over the
    # same rotation, on a workspace of its own (scan-only launches leave the
    # selection histogram for a finishing kernel to consume)
    ws_scan = jfa.Workspace(copies[0][0], w.topk, device=dev)
    for i in range(3):
        _, g, cs, _, _ = copies[i % n_copies]
        _lib.check(_lib.jfa_decode_scores(g, cs, q, scale, ws_scan.buf, sp), "scores")
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s0.record(stream)
    for i in range(args.steps):
        _, g, cs, _, _ = copies[i % n_copies]
        _lib.check(_lib.jfa_decode_scores(g, cs, q, scale, ws_scan.buf, sp), "scores")
    s1.record(stream)
    torch.cuda.synchronize()
    scan_avg = s0.elapsed_time(s1) / args.steps
    del ws_scan

    # end to end through the public API: every step copies q in from pinned
    # host memory and replays the step captured in a CUDA graph (one per
    # cache copy, captured before the timed region), whose finishing kernel
    # writes its output straight into pinned host memory (out may be
    # host-resident)
    q_host = q.cpu().pin_memory()
    out_host = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    graphs = [jfa.DecodeGraph(cache, q, w.topk, ke, ve, ws, scale=scale, out=out_host, idx=idx,
                              exact_on_host=bool(host))
              for cache, _, _, ke, ve in copies]

    def e2e_step(i):
        q.copy_(q_host, non_blocking=True)
        graphs[i % n_copies].replay()

    for i in range(max(3, args.warmup)):
        e2e_step(i)
    x0, x1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    x0.record(stream)
    for i in range(args.steps):
        e2e_step(i)
    x1.record(stream)
    torch.cuda.synchronize()
    e2e_avg = x0.elapsed_time(x1) / args.steps
    e2e_max = max_over_ranks(e2e_avg, world, dev)

    st, flag = _lib.jfa_check_error(geom, ws.buf, sp)
    if flag:
        raise RuntimeError(f"device error flag {flag:#x}")

    tokens = w.batch * w.ctx
    value = world * tokens / (ms_max / 1e3)
    peak, peak_kind = measured_peaks()
    achieved = scan_alg_bytes(w) / (scan_avg / 1e3) / 1e9
    step_gbs = step_alg_bytes(w) / (ms / 1e3) / 1e9
    launches = jfa.jfa_decode_step_launches(geom, w.topk)

    line = None
    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            k_exact, v_exact = copies[0][3], copies[0][4]
            kv_cpu = lambda b, h: (k_exact[b, h].cpu(), v_exact[b, h].cpu())
            val, n, spent = time_oracle(w, args.cpu_seconds, kv_cpu)
            cpu = {"value": val, "unit": "tokens/s", "cores": oracle_cores(), "kind": "oracle",
                   "sample": f"{n} of {w.batch * w.kv_heads} (sequence, KV head) segments "
                             f"({w.ctx} tokens each) in {spent:.1f} s, extrapolated to a "
                             f"full step"}
            try:  # the same oracle on one core (numpy's BLAS pool limited to 1 thread)
                from threadpoolctl import threadpool_limits
                with threadpool_limits(limits=1):
                    v1, n1, s1 = time_oracle(w, args.cpu_seconds / 2, kv_cpu)
                cpu["one_core"] = {"value": v1, "cores": 1,
                                   "sample": f"{n1} segments in {s1:.1f} s, extrapolated"}
            except ImportError:
                pass
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32", "data": "synthetic", "config": config_of(w, args, n_copies, packed_bytes),
            "roofline": {"bound": "hbm", "kernel": "scan_kernel (jfa_decode_scores)",
                         "achieved": achieved, "peak": peak, "peak_kind": peak_kind,
                         "unit": "GB/s", "frac": achieved / peak,
                         "traffic": recorded_traffic(w.name),
                         "alg_bytes_per_launch": scan_alg_bytes(w),
                         "us_per_launch": scan_avg * 1e3},
            "step_roofline": {"achieved": step_gbs, "peak": peak, "unit": "GB/s",
                              "frac": step_gbs / peak, "alg_bytes_per_step": step_alg_bytes(w)},
            "cpu_baseline": cpu,
            "e2e": {"value": world * tokens / (e2e_max / 1e3), "unit": "tokens/s",
                    "ms_per_step": e2e_max,
                    "h2d_bytes_per_step": q.numel() * q.element_size(),
                    "d2h_bytes_per_step": out.numel() * out.element_size()},
            "unfused": {"ms_per_step": unfused_ms,
                        "calls": "jfa_decode_scores + jfa_topk + jfa_correct_merge"},
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
    return run_jfa(args, w)


if __name__ == "__main__":
    sys.exit(main())
