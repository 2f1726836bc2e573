#!/usr/bin/env python3
"""Benchmark of the fused chunked KL-distillation loss (forward + backward).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--config 8k]

One step = ckl_forward + ckl_backward over one batch of the named workload
(default: the 8K student head, T=8192, d=3072, V=128256, K=100, chunk=1024,
5 % trailing padding), inputs resident in HBM.  With N > 1 (launched by
torch.distributed.run) every rank runs its own batch (weak scaling, no
collective on the data path); the time is the max over ranks.  Rank 0 prints
one JSON line.

``--impl reference`` times the fp64 CPU oracle instead (the only reference
implementation there is), on a bounded sample of rows per step.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "fused KL fwd+bwd tokens/s and TFLOP/s (% bf16 peak) @ T=8K,V=128256,d=3072"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--config", default="8k")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--dp-allreduce", action="store_true",
                    help="also time the data-parallel step: loss and dW all-reduced over the "
                         "ranks with NCCL, overlapped with the backward slab by slab")
    ap.add_argument("--no-single-pass", action="store_true",
                    help="skip timing the single-pass entry point (ckl_forward_backward)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--memory-sweep", action="store_true",
                    help="measure workspace and peak device memory vs T at the 256K shape")
    ap.add_argument("--topk", action="store_true",
                    help="time the teacher top-K cache producer (T=8192, V=128256, K=100)")
    ap.add_argument("--f32", action="store_true",
                    help="time the fp32-input entry points (tf32 tensor cores) on the workload")
    ap.add_argument("--compare", action="store_true",
                    help="peak memory and time vs T: dense / forward-chunked PyTorch losses "
                         "against the fused library, at the 32K shape")
    return ap.parse_args(argv)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def workload_desc(c):
    m = c["mask"]
    masked = 0 if m is None else int((m == 0).sum())
    return (f"{c['name']}: T={c['T']} d={c['d']} V={c['V']} K={c['K']} chunk={c['chunk']}, "
            f"{masked} positions masked, synthetic (seeded N(0,1) H, N(0,0.02) W, Zipf(1.1) "
            f"teacher ids, sorted N(0,2) teacher log-probs)")


def kernel_source_hash() -> str:
    """Hash of the sources of the tensor-core kernels and their launches (all
    CUDA sources but the top-K producer's); ncu traffic figures are valid only
    for it."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "chunked_kl_loss_ckl_b200", "csrc")
    for f in sorted(x for x in os.listdir(csrc) if x != "ckl_topk.cuh"):
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of ``kernel`` from profiles/traffic.json, or None
    when absent or taken on other kernel sources."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        t = json.load(f)
    if t.get("source_hash") != kernel_source_hash():
        return None
    e = t.get("kernels", {}).get(workload, {}).get(kernel)
    return None if e is None else float(e["dram_bytes_per_launch"])


def flops_per_token(c):
    return 8.0 * c["d"] * c["V"]


def backward_blocks(T, V, plan):
    """(rows, cols) of each block of the backward, in order (row chunks of
    plan[0] rows, each swept in plan[2] vocabulary slabs of plan[1] columns)."""
    Cr, Sv, n = plan
    out = []
    for r0 in range(0, T, Cr):
        for s in range(n):
            out.append((min(Cr, T - r0), min(Sv, V - s * Sv)))
    return out


def backward_launches(T, V, plan):
    """Tensor-core launches of one forward + backward per kernel: the logits
    once, and per backward block its dZ and its dH + dW."""
    nb = len(backward_blocks(T, V, plan))
    return {"fwd_gemm": 1, "bwd_dz": nb, "bwd_dhdw": nb}


def kernel_flops_per_step(T, d, V, plan):
    """FLOPs of one forward + backward per tensor-core kernel: the logits 2 T V
    d, each block's recomputed logits 2 rows cols d and its dH + dW 4 rows cols
    d (8 d V per token in all)."""
    blocks = backward_blocks(T, V, plan)
    return {"fwd_gemm": 2.0 * T * V * d, "bwd_dz": sum(2.0 * r * c * d for r, c in blocks),
            "bwd_dhdw": sum(4.0 * r * c * d for r, c in blocks)}


# ----------------------------------------------------------------- distributed
def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Max of a per-rank float over the process group (identity when alone)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(base: int, rank: int) -> int:
    """Each rank draws its own batch (weak scaling)."""
    return base + 1000 * rank


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """SM clock, power and clock-event reasons of one GPU, sampled on a host
    thread every ``period_s`` through NVML (or ``nvidia-smi -lms`` when NVML
    is unavailable), each sample stamped with ``time.perf_counter()``.
    ``stop(t0, t1)`` summarises only the samples taken inside [t0, t1], the
    host interval that brackets the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_uuid: str | None, period_s: float = 0.02):
        import threading
        self.samples = []          # (t, sm MHz, max sm MHz, power W or None, reasons)
        self.source = None
        self._stop = threading.Event()
        self._thread = None
        self.proc = None
        try:
            import pynvml
            pynvml.nvmlInit()
            h = (pynvml.nvmlDeviceGetHandleByUUID(gpu_uuid.encode()) if gpu_uuid
                 else pynvml.nvmlDeviceGetHandleByIndex(0))
            bits = {"hw_slowdown": pynvml.nvmlClocksEventReasonHwSlowdown,
                    "hw_thermal_slowdown": pynvml.nvmlClocksEventReasonHwThermalSlowdown,
                    "sw_thermal_slowdown": pynvml.nvmlClocksEventReasonSwThermalSlowdown,
                    "sw_power_cap": pynvml.nvmlClocksEventReasonSwPowerCap}
            smax = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))

            def poll():
                while not self._stop.is_set():
                    t = time.perf_counter()
                    try:
                        sm = float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM))
                        pw = pynvml.nvmlDeviceGetPowerUsage(h) / 1e3
                        r = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                        self.samples.append((t, sm, smax, pw,
                                             {n for n, b in bits.items() if r & b}))
                    except Exception:
                        pass
                    self._stop.wait(period_s)

            self.source = f"NVML, every {int(period_s * 1e3)} ms"
            self._thread = threading.Thread(target=poll, daemon=True)
            self._thread.start()
            return
        except Exception:
            pass
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
               "-lms", str(max(10, int(period_s * 1e3)))]
        if gpu_uuid:
            cmd += ["-i", gpu_uuid]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
        except OSError:
            return
        self.source = f"nvidia-smi -lms {max(10, int(period_s * 1e3))}"

        def read():
            for line in self.proc.stdout:
                t = time.perf_counter()
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm, smax = float(parts[1]), float(parts[2])
                except ValueError:
                    continue
                try:
                    pw = float(parts[3])
                except ValueError:
                    pw = None
                self.samples.append((t, sm, smax, pw, {n for n, v in zip(self.NAMES, parts[5:9])
                                                        if v.lower() == "active"}))

        import threading
        self._thread = threading.Thread(target=read, daemon=True)
        self._thread.start()

    def stop(self, t0: float | None = None, t1: float | None = None):
        self._stop.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self._thread is not None:
            self._thread.join(timeout=5)
        return summarise_clocks(self.samples, t0, t1, self.source)


def summarise_clocks(samples, t0=None, t1=None, source=None):
    """Median / min SM clock, median power and the reasons seen, over the
    samples with t0 <= t <= t1 (all of them when no window is given)."""
    inside = [s for s in samples if (t0 is None or s[0] >= t0) and (t1 is None or s[0] <= t1)]
    if not inside:
        return None
    sm = [s[1] for s in inside]
    pw = [s[3] for s in inside if s[3] is not None]
    reasons = set()
    for s in inside:
        reasons |= s[4]
    return {"sm_mhz": statistics.median(sm), "sm_min_mhz": min(sm),
            "sm_max_mhz": max(s[2] for s in inside),
            "power_w": round(statistics.median(pw), 1) if pw else None,
            "samples": len(inside), "reasons": sorted(reasons),
            "window_s": None if t0 is None or t1 is None else round(t1 - t0, 3),
            "source": f"{source}; only samples inside the timed region"}


def cpu_description():
    """(model name, logical CPUs this process may run on)."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.lower().startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    try:
        n = len(os.sched_getaffinity(0))
    except AttributeError:
        n = os.cpu_count() or 1
    return model, n


# ----------------------------------------------------------------- CPU oracle
def cpu_oracle_sample(c, target_s: float, rows: int | None = None):
    """Times the fp64 oracle on the first ``rows`` tokens of the workload.

    Calibrates ``rows`` so the timed run takes about ``target_s`` seconds
    unless ``rows`` is given.  Returns (tokens/s, rows, seconds, threads).
    """
    import oracle
    try:
        from threadpoolctl import threadpool_info
        threads = max((i.get("num_threads", 1) for i in threadpool_info()
                       if i.get("user_api") == "blas"), default=1)
    except Exception:
        threads = os.cpu_count() or 1

    def run(r):
        m = None if c["mask"] is None else c["mask"][:r]
        t0 = time.perf_counter()
        oracle.chunked(c["H"][:r], c["W"], c["idx"][:r], c["logp"][:r], m, chunk=r)
        return time.perf_counter() - t0

    if rows is None:
        # fixed cost (widening W to fp64) + per-row cost, from two probes
        t16, t48 = run(16), run(48)
        per_row = max((t48 - t16) / 32.0, 1e-4)
        fixed = max(t16 - 16 * per_row, 0.0)
        rows = int(min(4096, max(16, (target_s - fixed) / per_row)))
    dt = run(rows)
    return rows / dt, rows, dt, threads


# ----------------------------------------------------------------- ours
def bench_ours(args):
    import torch
    ws_n, rank, local = dist_env()
    if args.gpus != ws_n and ws_n > 1:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={ws_n}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws_n > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180),
                                device_id=dev)

    import chunked_kl_loss_ckl_b200 as ckl
    from ckl_synth import CONFIGS, make_config, student_topk_torch

    # the GPT-OSS-shaped teacher ids come from the student's own top-200
    # logits: input preparation, done with torch on the GPU before timing
    topk = student_topk_torch if CONFIGS[args.config].get("neighbourhood") else None
    c = make_config(args.config, seed=rank_seed(args.seed, rank), student_topk=topk)
    T, d, V, K, chunk = c["T"], c["d"], c["V"], c["K"], c["chunk"]
    to = lambda a, dt: torch.from_numpy(a).to(dev)
    H = to(c["H"].view(np.int16), None).view(torch.bfloat16)
    W = to(c["W"].view(np.int16), None).view(torch.bfloat16)
    idx = to(c["idx"], None)
    logp = to(c["logp"], None)
    mask = None if c["mask"] is None else to(c["mask"], None)
    ws = ckl.new_workspace(T, d, V, K, chunk, dev)
    loss = torch.empty(1, dtype=torch.float32, device=dev)
    lse = torch.empty(T, dtype=torch.float32, device=dev)
    dH = torch.empty(T, d, dtype=torch.bfloat16, device=dev)
    dW = torch.empty(V, d, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(trace=None):
        ckl.forward(H, W, idx, logp, mask, chunk, workspace=ws, trace=trace, out_loss=loss,
                    out_lse=lse)
        ckl.backward(H, W, idx, logp, mask, lse, chunk=chunk, dW=dW, accumulate_dW=False,
                     workspace=ws, trace=trace, out_dH=dH)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    rc, word = ckl.read_device_status(ws)
    if rc != 0:
        raise SystemExit(f"device status {rc} ({word}) after warm-up")

    # forward: prep, logits GEMM, combine; backward: prep + per row chunk an
    # H_c transpose, per vocabulary slab a dZ GEMM and a dH/dW GEMM, and a dH
    # conversion when sliced; the capacity leaves headroom and a full trace is
    # treated as an error below.
    Cr, Sv, n_slabs = ckl.backward_plan(T, d, V, K, chunk)
    n_launch = 3 + 1 + -(-T // Cr) * (1 + 2 * n_slabs + (1 if n_slabs > 1 else 0))
    trace = ckl.Trace(capacity=args.steps * (n_launch + 4) + 16)
    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    if ws_n > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(uuid)
    time.sleep(0.1)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    t_begin = time.perf_counter()
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    t_end = time.perf_counter()
    clocks = sampler.stop(t_begin, t_end)
    # per-kernel times: the same steps again with an event pair around every
    # launch (the events keep each backward GEMM from starting while the one
    # ahead of it drains, so this pass is not the headline)
    if ws_n > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    for _ in range(args.steps):
        step(trace)
    torch.cuda.synchronize()
    if ws_n > 1:
        torch.distributed.barrier()
    ms_total = e0.elapsed_time(e1)
    ms_total = max_over_ranks(ms_total, ws_n, dev)
    ms_step = ms_total / args.steps
    tokens = T * ws_n
    value = tokens / (ms_step / 1e3)
    tflops = flops_per_token(c) * tokens / (ms_step / 1e3) / 1e12

    if trace.count >= trace.capacity:
        raise SystemExit("launch trace overflowed: per-kernel times would be incomplete")
    # per-kernel times from the library's own launch events
    per = {}
    for name, ms in trace.durations():
        a = per.setdefault(name, [0, 0.0])
        a[0] += 1
        a[1] += ms
    gpu_launches = trace.count
    peaks, peak_src = load_peaks()
    # algorithmic FLOPs per launch of each tensor-core kernel: its FLOPs per
    # step over its launches per step (the backward's blocking sets them)
    chunks = (T + chunk - 1) // chunk
    per_step = kernel_flops_per_step(T, d, V, (Cr, Sv, n_slabs))
    alg = {k: v / (per[k][0] / args.steps) for k, v in per_step.items()
           if k in per and v > 0 and per[k][0] == args.steps * backward_launches(
               T, V, (Cr, Sv, n_slabs)).get(k, 1)}
    dom = max(per, key=lambda k: per[k][1])
    dom_avg_ms = per[dom][1] / per[dom][0]
    roofline = None
    if dom in alg:
        achieved = alg[dom] / (dom_avg_ms / 1e3) / 1e12
        peak = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
        roofline = {"kernel": dom, "bound": "tensor", "achieved": round(achieved, 1),
                    "peak": peak, "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                    "peak_source": f"{peak_src} bf16_tflops_sustained",
                    "avg_launch_ms": round(dom_avg_ms, 4), "launches": per[dom][0],
                    "timing": "CUDA events around each launch, on the launching stream, in a "
                              "second pass of the same steps",
                    "traffic": profiled_traffic(dom, args.config),
                    "traffic_unit": "bytes per launch (ncu dram__bytes_read.sum + "
                                    "dram__bytes_write.sum)"}
    kernels = {k: {"launches": v[0], "total_ms": round(v[1], 3),
                   "share": round(v[1] / sum(x[1] for x in per.values()), 4)}
               for k, v in sorted(per.items())}
    rc, word = ckl.read_device_status(ws)
    if rc != 0:
        raise SystemExit(f"device status {rc} ({word}) after the timed steps")

    # ------------------------------------------------------------ single pass
    # ckl_forward_backward on the same inputs: each chunk's logits computed
    # once (6 d V FLOP per token executed), reported beside the headline.
    single = None
    if not args.no_single_pass:
        ws_sp = torch.empty(ckl.single_pass_workspace_bytes(T, d, V, K, chunk), dtype=torch.uint8,
                            device=dev)

        def sp_step(trace=None):
            ckl.forward_backward(H, W, idx, logp, mask, chunk=chunk, dW=dW, accumulate_dW=False,
                                 workspace=ws_sp, trace=trace, out_loss=loss, out_lse=lse,
                                 out_dH=dH)

        for _ in range(args.warmup):
            sp_step()
        torch.cuda.synchronize()
        rc, word = ckl.read_device_status(ws_sp)
        if rc != 0:
            raise SystemExit(f"device status {rc} ({word}) in the single pass")
        sp_trace = ckl.Trace(capacity=args.steps * (3 + 4 * chunks + 4) + 16)
        if ws_n > 1:
            torch.distributed.barrier()
        g0 = torch.cuda.Event(enable_timing=True)
        g1 = torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        for _ in range(args.steps):
            sp_step(sp_trace)
        g1.record(stream)
        torch.cuda.synchronize()
        if sp_trace.count >= sp_trace.capacity:
            raise SystemExit("single-pass launch trace overflowed")
        ms_sp = max_over_ranks(g0.elapsed_time(g1) / args.steps, ws_n, dev)
        sp_per = {}
        for name, ms in sp_trace.durations():
            a = sp_per.setdefault(name, [0, 0.0])
            a[0] += 1
            a[1] += ms
        sp_total = sum(x[1] for x in sp_per.values())
        single = {
            "value": round(tokens / (ms_sp / 1e3), 1), "unit": "tokens/s",
            "ms_per_step": round(ms_sp, 4),
            "executed_tflops": round(6.0 * d * V * tokens / (ms_sp / 1e3) / 1e12, 1),
            "tflops_8dV_convention": round(flops_per_token(c) * tokens / (ms_sp / 1e3) / 1e12, 1),
            "executed_flop_per_token": "6 d V (logits once, dH, dW)",
            "gpu_launches": sp_trace.count,
            "kernels": {k: {"launches": v[0], "total_ms": round(v[1], 3),
                            "share": round(v[1] / sp_total, 4)}
                        for k, v in sorted(sp_per.items())},
            "workspace_bytes": ws_sp.numel(),
        }
        rc, word = ckl.read_device_status(ws_sp)
        if rc != 0:
            raise SystemExit(f"device status {rc} ({word}) after the single-pass steps")
        del ws_sp

    # ------------------------------------------------------------ data parallel
    dp_line = None
    if args.dp_allreduce:
        import torch.distributed as dist
        from chunked_kl_loss_ckl_b200.dp import dp_forward_backward
        own_group = not dist.is_initialized()
        if own_group:  # one rank: the collectives sum one term
            import tempfile
            store = tempfile.mkdtemp()
            dist.init_process_group("nccl", init_method=f"file://{store}/s", rank=0,
                                    world_size=1, device_id=dev)

        def dp_step():
            dp_forward_backward(H, W, idx, logp, mask, chunk=chunk, workspace=ws, dW=dW)

        for _ in range(args.warmup):
            dp_step()
        torch.cuda.synchronize()
        dist.barrier()
        h0 = torch.cuda.Event(enable_timing=True)
        h1 = torch.cuda.Event(enable_timing=True)
        h0.record(stream)
        for _ in range(args.steps):
            dp_step()
        h1.record(stream)
        torch.cuda.synchronize()
        ms_dp = max_over_ranks(h0.elapsed_time(h1) / args.steps, ws_n, dev)
        dp_line = {"value": round(tokens / (ms_dp / 1e3), 1), "unit": "tokens/s",
                   "ms_per_step": round(ms_dp, 4), "ranks": ws_n,
                   "exchange": "all-reduce of (loss x N, N), then of dW per vocabulary slab "
                               "as the backward finishes it (NCCL)"}
        if own_group:
            dist.destroy_process_group()

    # ------------------------------------------------------------ end to end
    e2e = None
    if not args.no_e2e:
        pin = lambda a: torch.from_numpy(a).pin_memory()
        hH = pin(c["H"].view(np.int16))
        hidx = pin(c["idx"])
        hlogp = pin(c["logp"])
        hmask = None if c["mask"] is None else pin(c["mask"])
        hloss = torch.empty(1, dtype=torch.float32).pin_memory()
        bi = hH.numel() * 2 + hidx.numel() * 4 + hlogp.numel() * 4 + (0 if hmask is None else
                                                                        hmask.numel())

        # the public staging helper: batch i + 1 crosses PCIe on a side
        # stream while the loss of batch i runs (each batch is copied once,
        # inside the timed region)
        from chunked_kl_loss_ckl_b200.staging import Stager
        host = [hH, hidx, hlogp] + ([hmask] if hmask is not None else [])
        stager = Stager(host, dev, stream)

        def e2e_run(n):
            stager.put(host)
            for i in range(n):
                bufs = stager.get()
                if i + 1 < n:
                    stager.put(host)
                Hs, ids, lp = bufs[0].view(torch.bfloat16), bufs[1], bufs[2]
                ms = bufs[3] if hmask is not None else None
                ckl.forward(Hs, W, ids, lp, ms, chunk, workspace=ws, out_loss=loss, out_lse=lse)
                ckl.backward(Hs, W, ids, lp, ms, lse, chunk=chunk, dW=dW, accumulate_dW=False,
                             workspace=ws, out_dH=dH)
                stager.release()
                hloss.copy_(loss, non_blocking=True)

        e2e_run(max(1, args.warmup // 2))
        torch.cuda.synchronize()
        if ws_n > 1:
            torch.distributed.barrier()
        f0 = torch.cuda.Event(enable_timing=True)
        f1 = torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        stager.copy_stream.wait_stream(stream)  # no copy starts before f0
        e2e_run(args.steps)
        f1.record(stream)
        torch.cuda.synchronize()
        ms_e2e = max_over_ranks(f0.elapsed_time(f1) / args.steps, ws_n, dev)
        e2e = {"value": round(tokens / (ms_e2e / 1e3), 1), "unit": "tokens/s",
               "ms_per_step": round(ms_e2e, 4), "h2d_bytes_per_step": int(bi),
               "d2h_bytes_per_step": 4,
               "copied": "H, topk_idx, topk_logp, mask host->device (staged on a side stream, "
                         "batch i+1 during step i); loss device->host; W stays resident "
                         "(a model parameter)"}

    cpu = None
    if rank == 0 and ws_n == 1 and not args.no_cpu_baseline:
        tps, rows, secs, threads = cpu_oracle_sample(c, args.cpu_seconds)
        model, ncpu = cpu_description()
        cpu = {"value": round(tps, 3), "unit": "tokens/s", "cores": threads, "kind": "oracle",
               "cpu_model": model, "nproc": ncpu,
               "sample": f"fp64 oracle (numpy, chunked form) on the first {rows} tokens of the "
                         f"same workload, full V and d: loss, lse, dH, dW; {secs:.1f} s"}

    if ws_n > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": ws_n,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": workload_desc(c), "T": T, "d": d, "V": V, "K": K, "chunk": chunk,
                   "global_batch_tokens": tokens, "parallelism": f"dp{ws_n} (independent batches)",
                   "backward_blocking": {"rows": Cr, "vocab_slab": Sv, "slabs": n_slabs},
                   "l2": "inputs larger than L2 (W 788 MB, dZ buffer 263 MB vs 126 MB L2); "
                         "no flush"},
        "tflops": round(tflops, 1),
        "pct_peak_sustained": round(tflops / float(peaks.get("bf16_tflops_sustained", 1400.0)), 4),
        "pct_peak_burst": round(tflops / float(peaks.get("bf16_tflops", 1590.0)), 4),
        "peak_source": peak_src,
        "flop_convention": "8 d V per token (fwd logits, bwd recompute, dH, dW)",
        "roofline": roofline, "kernels": kernels, "cpu_baseline": cpu, "e2e": e2e,
        "single_pass": single, "dp_step": dp_line,
        "gpu_launches": gpu_launches, "clocks": clocks,
        "workspace_bytes": ws.numel(),
        "peak_mem_bytes": int(torch.cuda.max_memory_allocated(dev)),
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------- reference
def bench_reference(args):
    ws_n, rank, _ = dist_env()
    if rank != 0:
        return  # the oracle runs once, on rank 0
    from ckl_synth import make_config
    c = make_config(args.config, seed=args.seed)
    # rows per step: a bounded sample so warm-up + steps end in a few minutes
    probe_tps, _, _, threads = cpu_oracle_sample(c, 0.0, rows=16)
    rows = int(max(8, min(512, probe_tps * 150.0 / max(1, args.steps + args.warmup))))
    for _ in range(args.warmup):
        cpu_oracle_sample(c, 0.0, rows=rows)
    times = []
    for _ in range(args.steps):
        tps, _, dt, _ = cpu_oracle_sample(c, 0.0, rows=rows)
        times.append(dt)
    ms = 1e3 * statistics.median(times)
    value = rows / (ms / 1e3)
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "tokens/s",
        "n_gpus": ws_n, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 2),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": workload_desc(c), "T": c["T"], "d": c["d"], "V": c["V"],
                   "K": c["K"], "chunk": c["chunk"], "sample_rows_per_step": rows},
        "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": threads,
                         "kind": "oracle", "cpu_model": cpu_description()[0],
                         "nproc": cpu_description()[1],
                         "sample": f"fp64 oracle on {rows} tokens per step (full V, d)"},
        "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def memory_sweep(args):
    """Workspace and peak device memory of forward + backward vs T at the
    256K shape (d=4096, V=128256, K=100, chunk=4096, 1 % of each 32K
    sequence masked).  Inputs are seeded device tensors of the workload's
    shapes; memory does not depend on their values."""
    import torch
    import chunked_kl_loss_ckl_b200 as ckl
    d, V, K, chunk = 4096, 128256, 100, 4096
    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev).manual_seed(args.seed)
    W = (torch.randn(V, d, generator=g, device=dev) * 0.02).to(torch.bfloat16)
    rows = []
    for T in (8192, 16384, 32768, 65536, 131072, 262144):
        H = torch.randn(T, d, generator=g, device=dev).to(torch.bfloat16)
        idx = torch.randint(0, V, (T, K), generator=g, device=dev, dtype=torch.int32)
        logp = torch.log_softmax(2.0 * torch.randn(T, K, generator=g, device=dev), dim=1)
        mask = torch.ones(T, dtype=torch.uint8, device=dev)
        mask.view(-1, min(T, 32768))[:, -328:] = 0
        torch.cuda.synchronize()
        base = torch.cuda.memory_allocated(dev)
        torch.cuda.reset_peak_memory_stats(dev)
        ws = ckl.new_workspace(T, d, V, K, chunk, dev)
        loss, lse = ckl.forward(H, W, idx, logp, mask, chunk, workspace=ws)
        dH, dW = ckl.backward(H, W, idx, logp, mask, lse, chunk=chunk, workspace=ws)
        torch.cuda.synchronize()
        peak = torch.cuda.max_memory_allocated(dev) - base
        outputs = lse.numel() * 4 + 4 + dH.numel() * 2 + dW.numel() * 4
        rows.append({"T": T, "workspace_bytes": ws.numel(),
                     "peak_minus_inputs_bytes": int(peak),
                     "peak_minus_inputs_and_outputs_bytes": int(peak - outputs),
                     "loss": float(loss.item())})
        del H, idx, logp, mask, ws, loss, lse, dH, dW
        torch.cuda.empty_cache()
    Ts = np.array([r["T"] for r in rows], float)
    fit = {}
    for key in ("workspace_bytes", "peak_minus_inputs_and_outputs_bytes"):
        y = np.array([r[key] for r in rows], float)
        A = np.stack([np.ones_like(Ts), Ts], 1)
        (a, b), *_ = np.linalg.lstsq(A, y, rcond=None)
        resid = float(np.max(np.abs(A @ np.array([a, b]) - y) / y))
        fit[key] = {"a_bytes": a, "b_bytes_per_token": b, "max_rel_residual": resid}
    print(json.dumps({"memory_vs_T": rows, "linear_fit": fit,
                      "shape": {"d": d, "V": V, "K": K, "chunk": chunk}}), flush=True)


# ----------------------------------------------------------------- comparators
# The two non-fused ways of computing the same loss that the source pages
# measure beside the fused one ("Tối ưu hóa chi phí chưng cất tri thức ...",
# section "Hai thay đổi hệ thống"; their numbers in "LLMのための効率的な知識蒸留
# ...", section "ロングコンテキストへのスケーリング").  Plain PyTorch with autograd;
# used only by --compare and by the test that checks they agree with the
# library.

def _kl_rows_torch(Hc, W, idx, logp):
    """Per-row KL of the renormalised teacher top-K against the student's
    full-vocabulary softmax, for one block of rows (bf16 logits, fp32 math)."""
    import torch
    logq = torch.log_softmax((Hc @ W.T).float(), dim=1)
    logp_n = torch.log_softmax(logp, dim=1)
    g = logq.gather(1, idx.long())
    return (logp_n.exp() * (logp_n - g)).sum(1)


def dense_kl_torch(H, W, idx, logp, mask):
    """The textbook dense loss: the whole [T, V] logit grid at once."""
    m = mask.float()
    return (_kl_rows_torch(H, W, idx, logp) * m).sum() / m.sum().clamp(min=1.0)


def forward_chunked_kl_torch(H, W, idx, logp, mask, chunk):
    """The loss computed chunk by chunk; autograd still keeps every chunk's
    logits for the backward."""
    m = mask.float()
    total = 0.0
    for c0 in range(0, H.shape[0], chunk):
        c1 = min(H.shape[0], c0 + chunk)
        total = total + (_kl_rows_torch(H[c0:c1], W, idx[c0:c1], logp[c0:c1]) * m[c0:c1]).sum()
    return total / m.sum().clamp(min=1.0)


def compare(args):
    import torch
    import chunked_kl_loss_ckl_b200 as ckl
    d, V, K, chunk = 4096, 128256, 100, 2048
    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev).manual_seed(args.seed)
    W0 = (torch.randn(V, d, generator=g, device=dev) * 0.02).to(torch.bfloat16)
    out = []
    for T in (8192, 16384, 32768, 65536, 131072, 262144):
        H0 = torch.randn(T, d, generator=g, device=dev).to(torch.bfloat16)
        idx = torch.randint(0, V, (T, K), generator=g, device=dev, dtype=torch.int32)
        logp = torch.log_softmax(2.0 * torch.randn(T, K, generator=g, device=dev), dim=1)
        mask = torch.ones(T, dtype=torch.uint8, device=dev)
        row = {"T": T}
        for name in ("dense", "forward_chunked", "fused_library", "fused_single_pass"):
            if not name.startswith("fused") and T > 65536:
                row[name] = "not run (needs more than the 180 GB of one B200)"
                continue
            H = H0.detach().clone().requires_grad_(not name.startswith("fused"))
            W = W0.detach().clone().requires_grad_(not name.startswith("fused"))
            torch.cuda.synchronize()
            torch.cuda.empty_cache()
            base = torch.cuda.memory_allocated(dev)
            torch.cuda.reset_peak_memory_stats(dev)
            try:
                times = []
                for rep in range(3):
                    e0 = torch.cuda.Event(enable_timing=True)
                    e1 = torch.cuda.Event(enable_timing=True)
                    e0.record()
                    if name == "fused_library":
                        ws = ckl.new_workspace(T, d, V, K, chunk, dev)
                        loss, lse = ckl.forward(H, W, idx, logp, mask, chunk, workspace=ws)
                        dH, dW = ckl.backward(H, W, idx, logp, mask, lse, chunk=chunk,
                                              workspace=ws)
                        del ws, lse, dH, dW
                    elif name == "fused_single_pass":
                        loss, lse, dH, dW = ckl.forward_backward(H, W, idx, logp, mask,
                                                                 chunk=chunk)
                        del lse, dH, dW
                    else:
                        H.grad = None
                        W.grad = None
                        loss = (dense_kl_torch(H, W, idx, logp, mask) if name == "dense" else
                                forward_chunked_kl_torch(H, W, idx, logp, mask, chunk))
                        loss.backward()
                    e1.record()
                    torch.cuda.synchronize()
                    times.append(e0.elapsed_time(e1))
                peak = torch.cuda.max_memory_allocated(dev) - base
                # peak above the inputs: everything the method itself holds,
                # its outputs (lse, dH, dW or the two gradients) included
                row[name] = {"peak_gib_over_inputs": round(peak / 2 ** 30, 2),
                             "ms": round(float(np.median(times[1:])), 2),
                             "loss": float(loss.item())}
            except torch.OutOfMemoryError:
                row[name] = "out of memory"
            # `loss` keeps the autograd graph, and with it H, W and their
            # gradients, alive: drop it before the next method's baseline
            loss = None
            H.grad = None
            W.grad = None
            del H, W, loss
            torch.cuda.synchronize()
            torch.cuda.empty_cache()
        print(json.dumps(row), flush=True)
        out.append(row)
        del H0, idx, logp, mask
        torch.cuda.empty_cache()
    print(json.dumps({"compare": out, "shape": {"d": d, "V": V, "K": K, "chunk": chunk}}),
          flush=True)


def bench_f32(args):
    """Forward + backward of the fp32-input entry points (tf32 products) on the
    workload with H and W kept in fp32; TFLOP/s against the tf32 peak taken as
    the measured sustained bf16 peak x the nominal tf32 / bf16 ratio (1.1 / 2.25)."""
    import torch
    import chunked_kl_loss_ckl_b200 as ckl
    from ckl_synth import make_config
    dev = torch.device("cuda", 0)
    c = make_config(args.config, seed=args.seed, fp32=True)
    T, d, V, K, chunk = c["T"], c["d"], c["V"], c["K"], c["chunk"]
    H = torch.from_numpy(c["H"]).to(dev)
    W = torch.from_numpy(c["W"]).to(dev)
    idx = torch.from_numpy(c["idx"]).to(dev)
    logp = torch.from_numpy(c["logp"]).to(dev)
    mask = None if c["mask"] is None else torch.from_numpy(c["mask"]).to(dev)
    ws = torch.empty(ckl.lib.ckl_workspace_bytes_f32(T, d, V, K, chunk), dtype=torch.uint8,
                     device=dev)
    dW = torch.empty(V, d, dtype=torch.float32, device=dev)

    def step():
        loss, lse = ckl.forward_f32(H, W, idx, logp, mask, chunk, workspace=ws)
        ckl.backward_f32(H, W, idx, logp, mask, lse, chunk=chunk, dW=dW, workspace=ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    rc, word = ckl.read_device_status(ws)
    ms = e0.elapsed_time(e1) / args.steps
    peaks, src = load_peaks()
    tf32_peak = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])) \
        * 1.1 / 2.25
    tflops = flops_per_token(c) * T / (ms / 1e3) / 1e12
    print(json.dumps({"path": "fp32 inputs, tf32 tensor cores", "workload": workload_desc(c),
                      "value": round(T / (ms / 1e3), 1), "unit": "tokens/s", "ms_per_step": round(ms, 4),
                      "tflops": round(tflops, 1), "tf32_peak": round(tf32_peak, 1),
                      "frac": round(tflops / tf32_peak, 4),
                      "peak_source": f"{src} bf16_tflops_sustained x 1.1 / 2.25 (nominal tf32 / bf16)",
                      "status": rc}), flush=True)


def bench_topk(args):
    """The teacher top-K cache producer: one pass over [T, V] bf16 logits,
    HBM-bound; achieved GB/s = (T V 2 + T K 8) bytes / kernel time."""
    import torch
    import chunked_kl_loss_ckl_b200 as ckl
    T, V, K = 8192, 128256, 100
    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev).manual_seed(args.seed)
    logits = (2.0 * torch.randn(T, V, generator=g, device=dev)).to(torch.bfloat16)
    for _ in range(args.warmup):
        ckl.topk_cache(logits, K)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        idx, logp, st = ckl.topk_cache(logits, K)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    peaks, src = load_peaks()
    nbytes = T * V * 2 + T * K * 8
    gbs = nbytes / (ms / 1e3) / 1e9
    print(json.dumps({"kernel": "topk_cache", "T": T, "V": V, "K": K, "ms": round(ms, 4),
                      "rows_per_s": round(T / (ms / 1e3), 1), "achieved_gbs": round(gbs, 1),
                      "peak_gbs": peaks.get("hbm_gbs"), "frac": round(gbs / peaks.get("hbm_gbs"), 4),
                      "peak_source": src, "status": int(st.item())}), flush=True)


def main(argv=None):
    args = parse_args(argv)
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.memory_sweep:
        memory_sweep(args)
        return
    if args.compare:
        compare(args)
        return
    if args.topk:
        bench_topk(args)
        return
    if args.f32:
        bench_f32(args)
        return
    if args.impl == "reference":
        bench_reference(args)
    else:
        bench_ours(args)


if __name__ == "__main__":
    main()
