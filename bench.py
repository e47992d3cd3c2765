"""Throughput bench for the fused exact-attention library on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

One step is one pass of the hot path over one batch of synthetic inputs
already resident in device memory:
  * prefill: attn_fwd on the long-context GQA causal workload
    (B=1, Hq=32, Hkv=8, N=16384, D=128, bf16, scale 1/sqrt(128));
  * decode:  attn_decode_paged on the MLA absorbed paged-decode workload
    (64 sequences x 128 heads, latent 576/512, 64-token pages, lengths
    uniform on [1024, 8192]).
The headline metric is prefill TFLOP/s (4*Nq*Nk*D per head, halved for
causal); the decode KV-cache GB/s (bytes of the latent rows of valid tokens
over the time of the split + combine kernels) is reported in the "decode"
object of the same line.  Both are compared with the measured B200 peaks.

With N > 1 (torchrun, one process per GPU) every rank runs the same
independent workload (weak scaling, no collective on the data path); the
value is the sum of the ranks' work over the slowest rank's time.

--impl reference times the fp64 CPU oracle (the reference program of this
repository) on a bounded sample of the same workload.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from exact_attention_135_b200 import inputs  # noqa: E402

PREFILL_ID = 3
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(PEAKS_FALLBACK), "fallback"


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


class ClockSampler:
    """Samples SM clocks and throttle reasons with nvidia-smi during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


def prefill_setup(dev):
    cfg = inputs.PREFILL_CONFIGS[PREFILL_ID]
    q, k, v = inputs.prefill_config_inputs(cfg)
    host = {"q": q.pin_memory(), "k": k.pin_memory(), "v": v.pin_memory()}
    d = {n: t.to(dev) for n, t in host.items()}
    d["o"] = torch.empty((cfg.B, cfg.Nq, cfg.Hq, cfg.Dv), dtype=torch.bfloat16, device=dev)
    d["lse"] = torch.empty((cfg.B, cfg.Hq, cfg.Nq), dtype=torch.float32, device=dev)
    host["o"] = torch.empty(d["o"].shape, dtype=torch.bfloat16).pin_memory()
    host["lse"] = torch.empty(d["lse"].shape, dtype=torch.float32).pin_memory()
    return cfg, host, d


def run_gpu(args):
    import exact_attention_135_b200 as ea

    world, rank, local = dist_env()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    peaks, peaks_kind = load_peaks()

    cfg, host, d = prefill_setup(dev)
    stream = torch.cuda.current_stream(dev)

    def prefill():
        ea.fwd(d["q"], d["k"], d["v"], causal=cfg.causal, scale=cfg.scale, out=d["o"], lse=d["lse"])

    for _ in range(args.warmup):
        prefill()
    torch.cuda.synchronize(dev)
    if ea.read_device_status(dev.index) != 0:
        raise RuntimeError("device status error after warm-up")

    sampler = ClockSampler(dev.index)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    time.sleep(0.3)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    t_all0 = torch.cuda.Event(enable_timing=True)
    t_all1 = torch.cuda.Event(enable_timing=True)
    t_all0.record(stream)
    for i in range(args.steps):
        ev[i][0].record(stream)
        prefill()
        ev[i][1].record(stream)
    t_all1.record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    if world > 1:
        torch.distributed.barrier()
    launch_ms = [a.elapsed_time(b) for a, b in ev]
    total_ms = t_all0.elapsed_time(t_all1)
    if ea.read_device_status(dev.index) != 0:
        raise RuntimeError("device status error in timed region")

    # end to end through the public API, host buffers, copies inside the timed region
    e2e_ms = []
    for i in range(args.warmup + args.steps):
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for n in ("q", "k", "v"):
            d[n].copy_(host[n], non_blocking=True)
        prefill()
        host["o"].copy_(d["o"], non_blocking=True)
        host["lse"].copy_(d["lse"], non_blocking=True)
        b.record(stream)
        torch.cuda.synchronize(dev)
        if i >= args.warmup:
            e2e_ms.append(a.elapsed_time(b))
    h2d = sum(host[n].numel() * host[n].element_size() for n in ("q", "k", "v"))
    d2h = sum(host[n].numel() * host[n].element_size() for n in ("o", "lse"))

    flops = cfg.flops()
    step_ms = total_ms / args.steps
    e2e_step = sum(e2e_ms) / len(e2e_ms)
    if world > 1:
        t = torch.tensor([step_ms, e2e_step, statistics.mean(launch_ms)], device=dev)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        step_ms, e2e_step, avg_launch = t.tolist()
    else:
        avg_launch = statistics.mean(launch_ms)
    value = world * flops / (step_ms * 1e-3) / 1e12
    achieved = flops / (avg_launch * 1e-3) / 1e12
    peak = peaks["bf16_tflops"]
    line = {
        "metric": "attention TFLOP/s (prefill)",
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(step_ms, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic: i.i.d. N(0,1) bf16 from a seeded CPU generator",
        "config": {"workload": cfg.name, "B": cfg.B, "Hq": cfg.Hq, "Hkv": cfg.Hkv, "Nq": cfg.Nq, "Nk": cfg.Nk,
                   "D": cfg.D, "causal": cfg.causal, "scale": cfg.scale, "global_batch": cfg.B * world,
                   "seq_len": cfg.Nq, "parallelism": f"replicas x{world}",
                   "l2": "inputs larger than L2 (Q 134 MB + K/V 67 MB per step), no flush"},
        "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
                     "frac": round(achieved / peak, 4), "peak_kind": f"{peaks_kind} bf16 burst",
                     "traffic": None, "kernel": "attn_fwd_kernel<D=128,causal>"},
        "e2e": {"value": round(world * flops / (e2e_step * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": args.steps,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.cpu_rows)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def oracle_prefill_sample(cfg, rows_per_head: int, seed: int):
    """Time the fp64 oracle on `rows_per_head` random query rows of every head."""
    import numpy as np
    import oracle

    q, k, v = inputs.prefill_config_inputs(cfg)
    q64 = q.to(torch.float64).numpy()
    k64 = k.to(torch.float64).numpy()
    v64 = v.to(torch.float64).numpy()
    rng = np.random.default_rng(seed)
    rows = np.sort(rng.choice(cfg.Nq, size=rows_per_head, replace=False))
    t0 = time.perf_counter()
    oracle.attention(q64, k64, v64, cfg.causal, cfg.scale, q_rows=rows)
    dt = time.perf_counter() - t0
    # algorithmic FLOPs of the sampled rows under the workload's own count
    share = rows_per_head / cfg.Nq
    return cfg.flops() * share, dt, rows


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:
        return len(os.sched_getaffinity(0))


def cpu_baseline(rows_per_head: int):
    cfg = inputs.PREFILL_CONFIGS[PREFILL_ID]
    flops, dt, rows = oracle_prefill_sample(cfg, rows_per_head, seed=7)
    return {"value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{rows_per_head} random query rows of each of the {cfg.Hq} heads of {cfg.name} "
                      f"(fp64 NumPy oracle, full score rows materialised), {dt:.1f} s"}


def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return
    cfg = inputs.PREFILL_CONFIGS[PREFILL_ID]
    times, flops_s = [], 0.0
    for i in range(args.warmup + args.steps):
        flops, dt, _ = oracle_prefill_sample(cfg, args.cpu_rows, seed=100 + i)
        if i >= args.warmup:
            times.append(dt)
            flops_s = flops
    step_s = sum(times) / len(times)
    value = flops_s / step_s / 1e12
    line = {
        "impl": "reference",
        "metric": "attention TFLOP/s (prefill)",
        "value": round(value, 6),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(step_s * 1e3, 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic: i.i.d. N(0,1) bf16 from a seeded CPU generator",
        "config": {"workload": cfg.name, "B": cfg.B, "Hq": cfg.Hq, "Hkv": cfg.Hkv, "Nq": cfg.Nq, "Nk": cfg.Nk,
                   "D": cfg.D, "causal": cfg.causal},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
                         "sample": f"{args.cpu_rows} random query rows of each head per step"},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-rows", type=int, default=8, help="query rows per head in each oracle sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
