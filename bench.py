"""Throughput bench for the fused exact-attention library on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

One step is one pass of the hot path over one batch of synthetic inputs
already resident in device memory:
  * prefill: attn_fwd on the long-context GQA causal workload
    (B=1, Hq=32, Hkv=8, N=16384, D=128, bf16, scale 1/sqrt(128));
  * prefill_c4: attn_fwd on the MQA wide-head workload (B=4, Hq=16, Hkv=1,
    N=4096, D=256, non-causal, Q doubled for peaked rows);
  * prefill_c2 / prefill_c1: attn_fwd on the GPT-2-small-shaped causal
    workload (B=8, H=12, N=1024, D=64) and on the tiny one (B=1, H=2, N=128,
    D=64), both latency-bound at these sizes;
  * decode:  attn_decode_paged on the MLA absorbed paged-decode workload
    (64 sequences x 128 heads, latent 576/512, 64-token pages, lengths
    uniform on [1024, 8192]);
  * gqa:     attn_decode_paged_gqa on the GQA-path paged-decode workload
    (64 sequences x 32 query heads in 8 groups, D=128, separate K/V pages,
    the same length mix);
  * mtp:     attn_decode_paged_mtp, the MLA decode with two query tokens per
    sequence;
  * fp8:     attn_fwd_fp8, the prefill on E4M3 inputs (same shape);
  * bwd:     attn_bwd (gradients of the prefill) on the long-context workload.
The headline metric is prefill TFLOP/s (4*Nq*Nk*D per head, halved for
causal); the decode KV-cache GB/s (bytes of the K/V rows of valid tokens
over the time of the decode + combine kernels) is reported in the "decode"
and "gqa_decode" objects of the same line.  All are compared with the
measured B200 peaks.  Every part reports the mean, median and best of its
per-launch times, and the line ends with a compact "summary" object that
holds each part's headline figure and roofline fraction.

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

# DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) from one
# ncu capture of the same launch; see profiles/.  Set to None whenever the
# kernel changes until it is captured again.
NCU_TRAFFIC_BYTES = {
    "prefill": 364641536 + 105544448,   # attn_fwd_kernel<D=128, causal> (persistent), GQA N=16384 workload
    "prefill_c4": 151093504 + 101837824,   # attn_fwd_kernel<D=256> (persistent), MQA D=256 workload
    "prefill_c2": 37816320 + 63232,     # attn_fwd_kernel<D=64, causal> (persistent), GPT-2-small shape
    # decode_split_kernel, MLA decode workload (with one token per sequence the
    # token-major unit numbering is the identity, so its loads are unchanged)
    "decode": 349552640 + 15395840,
    "mtp": 363760000 + 26660000,        # decode_split_kernel, MLA decode workload with 2 query tokens per sequence
    "gqa": 1357133568 + 4723712,        # gqa_decode_kernel, GQA-path decode workload
    "bwd": 665277184 + 338907392,       # attn_bwd_dqt_kernel<causal>, GQA N=16384 workload (backward)
    "fp8": 100876800 + 89678080,        # attn_fwd_kernel<D=128, causal, fp8>, same shape in E4M3
}
# Timed regions longer than this run under the power cap: compare with the
# sustained peak rather than the burst one.
SUSTAINED_AFTER_S = 1.0


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(PEAKS_FALLBACK), "fallback"


def max_over_ranks(values, device=None):
    """Element-wise maximum of `values` over all ranks (identity with one rank).

    Every rank must call it with a list of the same length; works for any
    torch.distributed backend (NCCL with a CUDA device, gloo on the CPU).
    """
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return list(values)
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def whole_job_rate(world: int, work_per_rank: float, slowest_ms: float) -> float:
    """Work done by all ranks together per second, timed by the slowest rank."""
    return world * work_per_rank / (slowest_ms * 1e-3)


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


class Part:
    """One timed piece of the step: a callable on device-resident inputs plus
    its end-to-end variant (pinned host inputs copied in, result copied out)."""

    def __init__(self, name, run, h2d, d2h, launches):
        self.name, self.run, self.h2d, self.d2h, self.launches = name, run, h2d, d2h, launches

    def e2e(self):
        for dst, src in self.h2d:
            dst.copy_(src, non_blocking=True)
        self.run()
        for dst, src in self.d2h:
            dst.copy_(src, non_blocking=True)

    def bytes(self, pairs):
        return sum(a.numel() * a.element_size() for a, _ in pairs)


def prefill_part(ea, dev, cfg_id=PREFILL_ID, name="prefill"):
    cfg = inputs.PREFILL_CONFIGS[cfg_id]
    q, k, v = inputs.prefill_config_inputs(cfg)
    host = {"q": q.pin_memory(), "k": k.pin_memory(), "v": v.pin_memory()}
    d = {n: t.to(dev) for n, t in host.items()}
    d["o"] = torch.empty((cfg.B, cfg.Nq, cfg.Hq, cfg.Dv), dtype=torch.bfloat16, device=dev)
    d["lse"] = torch.empty((cfg.B, cfg.Hq, cfg.Nq), dtype=torch.float32, device=dev)
    host["o"] = torch.empty(d["o"].shape, dtype=torch.bfloat16).pin_memory()
    host["lse"] = torch.empty(d["lse"].shape, dtype=torch.float32).pin_memory()

    def run():
        ea.fwd(d["q"], d["k"], d["v"], causal=cfg.causal, scale=cfg.scale, out=d["o"], lse=d["lse"])

    p = Part(name, run, [(d[n], host[n]) for n in ("q", "k", "v")],
             [(host["o"], d["o"]), (host["lse"], d["lse"])], launches=1)
    p.cfg = cfg
    p.work = cfg.flops()
    return p


def decode_part(ea, dev):
    cfg = inputs.DECODE_CONFIG
    c = inputs.decode_config_inputs(cfg)
    host = {"q": c.q.pin_memory(), "kv": c.kv_pages.pin_memory(), "bt": c.block_table.pin_memory(),
            "sl": c.cache_seqlens.pin_memory()}
    d = {n: t.to(dev) for n, t in host.items()}
    d["o"] = torch.empty((cfg.B, 1, cfg.Hq, cfg.Dv), dtype=torch.bfloat16, device=dev)
    d["lse"] = torch.empty((cfg.B, cfg.Hq), dtype=torch.float32, device=dev)
    d["ws"] = torch.empty(ea.decode_workspace_size(cfg.B, cfg.Hq, cfg.Dv, dev), dtype=torch.uint8, device=dev)
    host["o"] = torch.empty(d["o"].shape, dtype=torch.bfloat16).pin_memory()
    host["lse"] = torch.empty(d["lse"].shape, dtype=torch.float32).pin_memory()

    def run():
        ea.decode_paged(d["q"], d["kv"], d["bt"], d["sl"], cfg.scale, dv=cfg.Dv, out=d["o"], lse=d["lse"],
                        workspace=d["ws"])

    p = Part("decode", run, [(d[n], host[n]) for n in ("q", "kv", "bt", "sl")],
             [(host["o"], d["o"]), (host["lse"], d["lse"])], launches=2)
    p.cfg = cfg
    p.kv_bytes = c.kv_valid_bytes(cfg.Dk)
    p.tokens = int(c.cache_seqlens.to(torch.int64).sum())
    p.flops = 2.0 * cfg.Hq * (cfg.Dk + cfg.Dv) * p.tokens
    p.ws_bytes = d["ws"].numel()
    return p


MTP_SQ = 2   # query tokens per sequence of the multi-token decode part


def mtp_part(ea, dev):
    cfg = inputs.DECODE_CONFIG
    gen = torch.Generator(device="cpu").manual_seed(int(cfg.seed))
    lens = torch.randint(cfg.min_len, cfg.max_len + 1, (cfg.B,), generator=gen, dtype=torch.int32)
    c = inputs.paged_decode_inputs(cfg.B, cfg.Hq, cfg.Dk, lens, cfg.page_size, cfg.seed + 200000, s_q=MTP_SQ)
    host = {"q": c.q.pin_memory(), "kv": c.kv_pages.pin_memory(), "bt": c.block_table.pin_memory(),
            "sl": c.cache_seqlens.pin_memory()}
    d = {n: t.to(dev) for n, t in host.items()}
    d["o"] = torch.empty((cfg.B, MTP_SQ, cfg.Hq, cfg.Dv), dtype=torch.bfloat16, device=dev)
    d["lse"] = torch.empty((cfg.B, MTP_SQ, cfg.Hq), dtype=torch.float32, device=dev)
    d["ws"] = torch.empty(ea.decode_mtp_workspace_size(cfg.B, MTP_SQ, cfg.Hq, cfg.Dv, dev), dtype=torch.uint8,
                          device=dev)
    host["o"] = torch.empty(d["o"].shape, dtype=torch.bfloat16).pin_memory()
    host["lse"] = torch.empty(d["lse"].shape, dtype=torch.float32).pin_memory()

    def run():
        ea.decode_paged_mtp(d["q"], d["kv"], d["bt"], d["sl"], cfg.scale, dv=cfg.Dv, out=d["o"], lse=d["lse"],
                            workspace=d["ws"])

    p = Part("mtp", run, [(d[n], host[n]) for n in ("q", "kv", "bt", "sl")],
             [(host["o"], d["o"]), (host["lse"], d["lse"])], launches=2)
    p.cfg = cfg
    p.kv_bytes = c.kv_valid_bytes(cfg.Dk)
    p.tokens = int(c.cache_seqlens.to(torch.int64).sum())
    # query token i of a sequence of length L attends to L - s_q + 1 + i positions
    p.pairs = MTP_SQ * p.tokens - cfg.B * MTP_SQ * (MTP_SQ - 1) // 2
    p.flops = 2.0 * cfg.Hq * (cfg.Dk + cfg.Dv) * p.pairs
    return p


def gqa_part(ea, dev):
    cfg = inputs.GQA_DECODE_CONFIG
    c = inputs.gqa_decode_config_inputs(cfg)
    host = {"q": c.q.pin_memory(), "kp": c.k_pages.pin_memory(), "vp": c.v_pages.pin_memory(),
            "bt": c.block_table.pin_memory(), "sl": c.cache_seqlens.pin_memory()}
    d = {n: t.to(dev) for n, t in host.items()}
    d["o"] = torch.empty((cfg.B, 1, cfg.Hq, cfg.D), dtype=torch.bfloat16, device=dev)
    d["lse"] = torch.empty((cfg.B, cfg.Hq), dtype=torch.float32, device=dev)
    d["ws"] = torch.empty(ea.decode_gqa_workspace_size(cfg.B, cfg.Hq, cfg.Hkv, cfg.D, dev), dtype=torch.uint8,
                          device=dev)
    host["o"] = torch.empty(d["o"].shape, dtype=torch.bfloat16).pin_memory()
    host["lse"] = torch.empty(d["lse"].shape, dtype=torch.float32).pin_memory()

    def run():
        ea.decode_paged_gqa(d["q"], d["kp"], d["vp"], d["bt"], d["sl"], cfg.scale, out=d["o"], lse=d["lse"],
                            workspace=d["ws"])

    p = Part("gqa", run, [(d[n], host[n]) for n in ("q", "kp", "vp", "bt", "sl")],
             [(host["o"], d["o"]), (host["lse"], d["lse"])], launches=2)
    p.cfg = cfg
    p.kv_bytes = c.kv_valid_bytes()
    p.tokens = int(c.cache_seqlens.to(torch.int64).sum())
    p.flops = 4.0 * cfg.Hq * cfg.D * p.tokens
    p.ws_bytes = d["ws"].numel()
    return p


def fp8_part(ea, dev):
    """attn_fwd_fp8 on the long-context GQA causal shape with E4M3 inputs
    (the same draws as the prefill workload, encoded per tensor)."""
    cfg = inputs.PREFILL_CONFIGS[PREFILL_ID]
    q8, k8, v8, ds = inputs.fp8_prefill_inputs(cfg.B, cfg.Hq, cfg.Hkv, cfg.Nq, cfg.Nk, cfg.D, cfg.seed, cfg.q_mult)
    host = {"q": q8.pin_memory(), "k": k8.pin_memory(), "v": v8.pin_memory()}
    d = {n: t.to(dev) for n, t in host.items()}
    d["o"] = torch.empty((cfg.B, cfg.Nq, cfg.Hq, cfg.D), dtype=torch.bfloat16, device=dev)
    d["lse"] = torch.empty((cfg.B, cfg.Hq, cfg.Nq), dtype=torch.float32, device=dev)
    host["o"] = torch.empty(d["o"].shape, dtype=torch.bfloat16).pin_memory()
    host["lse"] = torch.empty(d["lse"].shape, dtype=torch.float32).pin_memory()

    def run():
        ea.fwd_fp8(d["q"], d["k"], d["v"], *ds, causal=cfg.causal, scale=cfg.scale, out=d["o"], lse=d["lse"])

    p = Part("fp8", run, [(d[n], host[n]) for n in ("q", "k", "v")],
             [(host["o"], d["o"]), (host["lse"], d["lse"])], launches=1)
    p.cfg = cfg
    p.work = cfg.flops()
    return p


def bwd_part(ea, dev):
    """attn_bwd on the long-context GQA causal workload: O and LSE come from
    one forward pass at setup; dO ~ N(0,1) bf16 from its own seeded stream."""
    cfg = inputs.PREFILL_CONFIGS[PREFILL_ID]
    q, k, v, do = inputs.bwd_config_inputs(cfg)
    host = {"q": q.pin_memory(), "k": k.pin_memory(), "v": v.pin_memory(), "do": do.pin_memory()}
    d = {n: t.to(dev) for n, t in host.items()}
    d["o"], d["lse"] = ea.fwd(d["q"], d["k"], d["v"], causal=cfg.causal, scale=cfg.scale)
    host["o"] = d["o"].cpu().pin_memory()
    host["lse"] = d["lse"].cpu().pin_memory()
    for n, ref in (("dq", "q"), ("dk", "k"), ("dv", "v")):
        d[n] = torch.empty_like(d[ref])
        host[n] = torch.empty(d[n].shape, dtype=torch.bfloat16).pin_memory()
    d["ws"] = torch.empty(ea.bwd_workspace_size(cfg.B, cfg.Hq, cfg.Nq, cfg.D), dtype=torch.uint8, device=dev)

    def run():
        ea.bwd(d["q"], d["k"], d["v"], d["o"], d["lse"], d["do"], causal=cfg.causal, scale=cfg.scale,
               dq=d["dq"], dk=d["dk"], dv=d["dv"], workspace=d["ws"])

    p = Part("bwd", run, [(d[n], host[n]) for n in ("q", "k", "v", "o", "lse", "do")],
             [(host[n], d[n]) for n in ("dq", "dk", "dv")], launches=3)
    p.cfg = cfg
    # five products of the size of one forward product pair: 2.5 x the forward count
    p.work = 2.5 * cfg.flops()
    p.ws_bytes = d["ws"].numel()
    return p


def time_parts(parts, steps, stream):
    """Times `steps` steps; each step runs every part once.  Returns total ms
    and per-part lists of per-launch ms (CUDA events on the launching stream)."""
    ev = {p.name: [] for p in parts}
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    pairs = {p.name: [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                      for _ in range(steps)] for p in parts}
    t0.record(stream)
    for i in range(steps):
        for p in parts:
            a, b = pairs[p.name][i]
            a.record(stream)
            p.run()
            b.record(stream)
    t1.record(stream)
    torch.cuda.synchronize()
    for p in parts:
        ev[p.name] = [a.elapsed_time(b) for a, b in pairs[p.name]]
    return t0.elapsed_time(t1), ev


def time_e2e(parts, steps, warmup, dev, stream):
    out = {p.name: [] for p in parts}
    for p in parts:
        for i in range(warmup + steps):
            torch.cuda.synchronize(dev)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            p.e2e()
            b.record(stream)
            torch.cuda.synchronize(dev)
            if i >= warmup:
                out[p.name].append(a.elapsed_time(b))
    return out


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
    stream = torch.cuda.current_stream(dev)

    builders = [("prefill", lambda: prefill_part(ea, dev)),
                ("prefill_c4", lambda: prefill_part(ea, dev, 4, "prefill_c4")),
                ("prefill_c2", lambda: prefill_part(ea, dev, 2, "prefill_c2")),
                ("decode", lambda: decode_part(ea, dev)),
                ("prefill_c1", lambda: prefill_part(ea, dev, 1, "prefill_c1")),
                ("gqa", lambda: gqa_part(ea, dev)),
                ("mtp", lambda: mtp_part(ea, dev)),
                ("fp8", lambda: fp8_part(ea, dev)),
                ("bwd", lambda: bwd_part(ea, dev))]
    # The small workloads (1 and 2) fit in L2; in the step they run right after
    # parts that stream 200-400 MB, which evicts them between their launches.
    parts = [make() for name, make in builders if args.part in ("all", name)]

    for _ in range(args.warmup):
        for p in parts:
            p.run()
    torch.cuda.synchronize(dev)
    if ea.read_device_status(dev.index) != 0:
        raise RuntimeError("device status error after warm-up")

    sampler = ClockSampler(dev.index)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    time.sleep(0.3)
    total_ms, per = time_parts(parts, args.steps, stream)
    clocks = sampler.stop()
    if world > 1:
        torch.distributed.barrier()
    if ea.read_device_status(dev.index) != 0:
        raise RuntimeError("device status error in timed region")
    e2e = time_e2e(parts, args.e2e_steps, 3, dev, stream)

    # max over ranks of every timing (mean, median and best per launch, e2e mean)
    names = [p.name for p in parts]
    vec = [total_ms / args.steps]
    for n in names:
        vec += [statistics.mean(per[n]), statistics.median(per[n]), min(per[n]), statistics.mean(e2e[n])]
    vec = max_over_ranks(vec, device=dev)
    step_ms = vec[0]
    stat = {n: dict(zip(("mean", "median", "best", "e2e"), vec[1 + 4 * i:5 + 4 * i])) for i, n in enumerate(names)}
    by = {p.name: p for p in parts}

    sustained = step_ms * args.steps * 1e-3 > SUSTAINED_AFTER_S
    bf16_peak = peaks["bf16_tflops_sustained"] if sustained else peaks["bf16_tflops"]
    bf16_kind = f"{peaks_kind} bf16 {'sustained' if sustained else 'burst'}"

    def timing(n):
        t = stat[n]
        return {"ms_mean": round(t["mean"], 4), "ms_median": round(t["median"], 4), "ms_best": round(t["best"], 4)}

    def e2e_obj(p, work, unit, scale):
        return {"value": round(world * work / (stat[p.name]["e2e"] * 1e-3) / scale, 2), "unit": unit,
                "h2d_bytes_per_step": p.bytes(p.h2d), "d2h_bytes_per_step": p.bytes(p.d2h)}

    def tensor_obj(p, metric, kernel, peak, peak_kind, traffic=None):
        tf = p.work / (stat[p.name]["mean"] * 1e-3) / 1e12
        return {"metric": metric, "value": round(whole_job_rate(world, p.work, stat[p.name]["mean"]) / 1e12, 2),
                "unit": "TFLOP/s", **timing(p.name),
                "tflops_median": round(p.work / (stat[p.name]["median"] * 1e-3) / 1e12, 2),
                "config": {"workload": p.cfg.name, "causal": p.cfg.causal},
                "roofline": {"bound": "tensor", "achieved": round(tf, 2), "peak": round(peak, 1), "unit": "TFLOP/s",
                             "frac": round(tf / peak, 4), "peak_kind": peak_kind, "traffic": traffic,
                             "kernel": kernel, "frac_of_burst": round(tf / peaks["bf16_tflops"], 4)},
                "e2e": e2e_obj(p, p.work, "TFLOP/s", 1e12)}

    def hbm_obj(p, metric, kernel, traffic=None, extra=None):
        sec = stat[p.name]["mean"] * 1e-3
        gbs = p.kv_bytes / sec / 1e9
        o = {"metric": metric, "value": round(whole_job_rate(world, p.kv_bytes, stat[p.name]["mean"]) / 1e9, 1),
             "unit": "GB/s", **timing(p.name), "gbs_median": round(p.kv_bytes / (stat[p.name]["median"] * 1e-3) / 1e9, 1),
             "config": {"workload": p.cfg.name, "kv_bytes": p.kv_bytes, "tokens": p.tokens},
             "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                          "frac": round(gbs / peaks["hbm_gbs"], 4), "peak_kind": f"{peaks_kind} HBM copy",
                          "traffic": traffic, "kernel": kernel},
             "e2e": e2e_obj(p, p.kv_bytes, "GB/s", 1e9)}
        # against the nominal ~8 TB/s of HBM3e as well as the measured copy
        o["roofline"]["frac_of_nominal_8tbs"] = round(gbs / 8000.0, 4)
        if hasattr(p, "flops"):
            o["roofline"]["tflops"] = round(p.flops / sec / 1e12, 1)
            # combined roofline: the slower of moving the KV bytes at the HBM
            # peak and doing the FLOPs at this line's bf16 peak, over the time
            t_min = max(p.kv_bytes / (peaks["hbm_gbs"] * 1e9), p.flops / (bf16_peak * 1e12))
            o["roofline"]["frac_of_combined"] = round(t_min / sec, 4)
        if extra:
            o.update(extra)
        return o

    objs = {}
    if "prefill_c4" in by:
        objs["prefill_c4"] = tensor_obj(by["prefill_c4"], "attention TFLOP/s (prefill, MQA D=256)",
                                        "attn_fwd_kernel<D=256,non-causal>", bf16_peak, bf16_kind,
                                        NCU_TRAFFIC_BYTES.get("prefill_c4"))
    if "prefill_c2" in by:
        objs["prefill_c2"] = tensor_obj(by["prefill_c2"], "attention TFLOP/s (prefill, GPT-2-small shape)",
                                        "attn_fwd_kernel<D=64,causal>", bf16_peak, bf16_kind,
                                        NCU_TRAFFIC_BYTES.get("prefill_c2"))
    if "prefill_c1" in by:
        p = by["prefill_c1"]
        o = tensor_obj(p, "attention TFLOP/s (prefill, tiny)", "attn_fwd_kernel<D=64,non-causal>", bf16_peak,
                       bf16_kind)
        o["us_per_call"] = round(stat[p.name]["mean"] * 1e3, 2)
        objs["prefill_c1"] = o
    if "decode" in by:
        objs["decode"] = hbm_obj(by["decode"], "KV-cache GB/s (paged MLA decode)",
                                 "decode_split_kernel + decode_combine_kernel", NCU_TRAFFIC_BYTES.get("decode"),
                                 {"workspace_bytes": by["decode"].ws_bytes})
    if "gqa" in by:
        objs["gqa_decode"] = hbm_obj(by["gqa"], "KV-cache GB/s (GQA-path paged decode)",
                                     "gqa_decode_kernel + gqa_combine_kernel", NCU_TRAFFIC_BYTES.get("gqa"))
    if "mtp" in by:
        p = by["mtp"]
        extra = {"s_q": MTP_SQ, "query_tokens_per_s": round(world * p.cfg.B * MTP_SQ / (stat["mtp"]["mean"] * 1e-3), 1)}
        if "decode" in by:
            extra["time_vs_one_token"] = round(stat["mtp"]["mean"] / stat["decode"]["mean"], 3)
        objs["decode_mtp"] = hbm_obj(p, f"KV-cache GB/s (paged MLA decode, {MTP_SQ} query tokens per sequence)",
                                     "decode kernels over query units", NCU_TRAFFIC_BYTES.get("mtp"), extra)
    if "fp8" in by:
        # no measured fp8 peak: the measured bf16 peak times the nominal dense fp8/bf16 ratio (4.5 / 2.25)
        o = tensor_obj(by["fp8"], "attention TFLOP/s (FP8 E4M3 prefill)", "attn_fwd_kernel<D=128,causal,fp8>",
                       2.0 * bf16_peak, bf16_kind + " x 2 (nominal fp8/bf16 ratio)", NCU_TRAFFIC_BYTES.get("fp8"))
        o["roofline"]["frac_of_bf16_peak"] = o["roofline"].pop("frac_of_burst")
        objs["fp8"] = o
    if "bwd" in by:
        o = tensor_obj(by["bwd"], "attention backward TFLOP/s",
                       "bwd_prep_kernel + attn_bwd_dqt_kernel<causal> + bwd_dqt_kernel (timed together)",
                       bf16_peak, bf16_kind, NCU_TRAFFIC_BYTES.get("bwd"))
        o["config"]["flops"] = "2.5 x forward (five products)"
        objs["bwd"] = o

    line = {"n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_ms, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic: i.i.d. N(0,1) bf16 from a seeded CPU generator",
            "gpu_launches": args.steps * sum(p.launches for p in parts), "clocks": clocks}
    step_parts = "+".join(names)
    if "prefill" in by:
        p = by["prefill"]
        head = tensor_obj(p, "attention TFLOP/s (prefill)", "attn_fwd_kernel<D=128,causal>", bf16_peak, bf16_kind,
                          NCU_TRAFFIC_BYTES["prefill"])
        head["roofline"]["algorithmic_bytes"] = p.cfg.io_bytes()
        head["config"] = {"workload": p.cfg.name, "step": step_parts, "B": p.cfg.B, "Hq": p.cfg.Hq,
                          "Hkv": p.cfg.Hkv, "Nq": p.cfg.Nq, "Nk": p.cfg.Nk, "D": p.cfg.D, "causal": p.cfg.causal,
                          "global_batch": p.cfg.B * world, "seq_len": p.cfg.Nq, "parallelism": f"replicas x{world}",
                          "l2": "inputs larger than L2 (Q 134 MB + K/V 67 MB per step), no flush"}
    else:
        head = next(iter(objs.values()))
        head["config"]["step"] = step_parts
    line.update({k: head[k] for k in ("metric", "value", "unit", "config", "roofline", "e2e")})
    line.update({k: head[k] for k in ("ms_mean", "ms_median", "ms_best")})
    line.update(objs)
    if rank == 0 and world == 1 and not args.no_cpu_baseline and "prefill" in by:
        line["cpu_baseline"] = cpu_baseline(args.baseline_rows)
    # last key: one figure and one roofline fraction per part, short enough to
    # survive any truncation of the line's head
    summary = {}
    if "prefill" in by:
        summary["prefill_c3"] = [head["value"], head["roofline"]["frac"]]
    for k, o in objs.items():
        summary[k] = [o["value"], o["roofline"]["frac"]]
    if "decode_mtp" in objs and "time_vs_one_token" in objs["decode_mtp"]:
        summary["mtp_time_vs_one_token"] = objs["decode_mtp"]["time_vs_one_token"]
    summary["units"] = "prefill/fp8/bwd TFLOP/s, decodes GB/s; [value, roofline frac]"
    line["summary"] = summary
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


_ORACLE_INPUTS = {}


def oracle_prefill_sample(cfg, rows_per_head: int, seed: int):
    """Time the fp64 oracle on `rows_per_head` random query rows of every head.

    Returns (algorithmic FLOPs of the sampled rows, seconds, rows).  The inputs
    are drawn and upcast once per process, outside the timed region.
    """
    import numpy as np
    import oracle

    if cfg.name not in _ORACLE_INPUTS:
        q, k, v = inputs.prefill_config_inputs(cfg)
        _ORACLE_INPUTS[cfg.name] = tuple(t.to(torch.float64).numpy() for t in (q, k, v))
    q64, k64, v64 = _ORACLE_INPUTS[cfg.name]
    rng = np.random.default_rng(seed)
    rows = np.sort(rng.choice(cfg.Nq, size=rows_per_head, replace=False))
    t0 = time.perf_counter()
    oracle.attention(q64, k64, v64, cfg.causal, cfg.scale, q_rows=rows)
    dt = time.perf_counter() - t0
    # the sampled rows' share of the workload's FLOP count (4*Nq*Nk*D per head, halved when causal)
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
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-rows", type=int, default=64,
                    help="query rows per head in each step of --impl reference")
    ap.add_argument("--baseline-rows", type=int, default=768,
                    help="query rows per head in the cpu_baseline sample (about 10 s of CPU work)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--part", choices=["all", "prefill", "prefill_c4", "prefill_c2", "prefill_c1", "decode", "gqa",
                                       "mtp", "fp8", "bwd"], default="all",
                    help="time only one piece of the step (for profiling runs)")
    ap.add_argument("--e2e-steps", type=int, default=5, help="steps of the end-to-end (host buffer) timing")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
