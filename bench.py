"""Benchmark of the H-Spec block-parallel draft step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl hspec|reference]
                    [--C 128] [--K 16] [--sweep] [--draft-vocab V] [--no-cpu-baseline]
                    [--no-attention-configs] [--kernel step|attn|inject|ssd|verify|gemm]
                    [--workload NAME]

One step = one hspec_draft_step over a batch of C requests of the 4-layer M,A,M,A
drafter on Llama-3-8B shapes (SwiGLU 16384, shared 128256-token LM head), K block
positions each, context lengths uniform in [512, 16384], every attention layer
reading its own paged target KV cache in place.  Metric: drafted tokens/s
(C*K per step), with the step time in microseconds.  Inputs (~20 GB of weights
and KV) exceed the 126 MB L2, so no flush is needed between steps.

Multi-GPU: requests are independent, so each rank runs its own batch of C
requests (weak scaling, replicas only, no collective on the data path); the step
time is the max over ranks.

--impl reference times the CPU oracle on the same config and metric (rank 0 only).
--kernel times one kernel-level call on a named workload instead of the step.
The step line also carries, per concurrency point, the per-kernel-group times and
roofline fractions, and the paged attention timed alone on the Llama-3-8B C=32 and
Qwen-32B C=128 workloads (attention_configs: after a quarter of a second of its own
calls, so that it is timed at the SM clock it sustains alone, with that clock sampled).
"""
from __future__ import annotations

import argparse
from dataclasses import replace
import json
import re
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

METRIC = "drafted tokens/s (draft step, C*K tokens per step)"
UNIT = "tokens/s"


# --------------------------------------------------------------------- helpers

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 50 ms; the summary keeps the
    samples taken inside the timed region (window()), started early so that nvidia-smi
    is already sampling when the region begins."""
    FIELDS = ["index", "clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.lines = []
        self.t0 = self.t1 = None

    def start(self):
        try:
            uuid = str(torch.cuda.get_device_properties(self.dev).uuid)
            target = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={','.join(self.FIELDS)}", "--format=csv,noheader,nounits",
                 "-lms", "50", "-i", target], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.monotonic(), line.strip()))

    def window(self, t0, t1):
        self.t0, self.t1 = t0, t1

    def stop(self):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        inside = [ln for t, ln in self.lines if self.t0 is not None and self.t0 <= t <= self.t1 + 0.05]
        for ln in inside if inside else [ln for _, ln in self.lines]:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm), "in_timed_region": bool(inside)}


def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, world: int) -> float:
    """The slowest rank's value: every rank takes the same collective step (one
    all-reduce of one float64) on the process group's device (CUDA under NCCL, host
    memory under gloo)."""
    if world == 1:
        return v
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_workload(I, wl, rank: int):
    """Rank r's batch: the same shapes and context-length range, its own seed (the
    requests of different replicas are different requests)."""
    return I.Workload(wl.name, wl.shapes, wl.C, wl.K, wl.ctx_lo, wl.ctx_hi, seed=wl.seed + 1000 * rank)


def replica_throughput(tokens_per_rank: int, ms_per_rank: float, world: int):
    """Whole-job tokens/s of `world` replicas: all ranks' tokens over the slowest
    rank's step time (max over ranks)."""
    ms_max = max_over_ranks(ms_per_rank, world)
    return ms_max, tokens_per_rank * world / (ms_max / 1e3)


# ---------------------------------------------------------------- algorithmic work

def step_work(sh, C, K, ctx_lens):
    """Algorithmic bytes and flops of each kernel group for one launch."""
    d, H, P, N = sh.d, sh.H, sh.P, sh.N
    HP, HPN = H * P, H * P * N
    n_in = 2 * HP + 2 * N + H
    n_qkv = (sh.Hq + 2 * sh.Hkv) * sh.D
    M = C * K
    E = 2 if sh.dtype == "bf16" else 4
    ctx_sum = int(ctx_lens.sum())
    kv_bytes = ctx_sum * sh.Hkv * sh.D * 2 * E
    w = {}

    def gemm(name, m, n, k, extra_bytes=0):
        w[name] = {"flops": 2.0 * m * n * k, "bytes": float(n * k * E + m * k * E + extra_bytes)}

    gemm("in_proj", M, n_in, d, M * n_in * E)
    # the draft step as benchmarked stores h0 (the fused injection readout is opt-in)
    fused = False
    gemm("inject", C, HPN, d, M * (N + H) * E + M * HP * 8 if fused else C * HPN * 4)
    gemm("out_proj", M, d, HP, M * d * 8)
    gemm("qkv_proj", M, n_qkv, d, M * n_qkv * E)
    gemm("o_proj", M, d, sh.Hq * sh.D, M * d * 8)
    if sh.d_ff:
        gemm("mlp_gate_up", M, 2 * sh.d_ff, d, M * sh.d_ff * E)
        gemm("mlp_down", M, d, sh.d_ff, M * d * 8)
    if sh.vocab:
        gemm("lm_head_argmax", M, sh.draft_vocab or sh.vocab, d)
    w["attn_paged"] = {"flops": 4.0 * sh.Hq * sh.D * K * (ctx_sum + C * K),
                       "bytes": float(kv_bytes + 2 * M * sh.Hq * sh.D * E + 2 * M * sh.Hkv * sh.D * E)}
    if fused:  # zero-state scan: in-block terms and D x only
        w["ssd_scan"] = {"flops": float(C * H * K * K * (N + P)),
                         "bytes": float(M * (HP + 2 * N + H) * E + M * HP * 4)}
    else:
        w["ssd_scan"] = {"flops": float(C * H * (2 * K * P * N + K * K * (N + P))),
                         "bytes": float(C * HPN * 4 + M * (HP + 2 * N + H) * E + M * HP * 4)}
    return w


def step_roofline_ms(sh, C, K, ctx_lens, peaks):
    """Lower bound of one draft step: every kernel group at its own roofline (the
    slower of its algorithmic bytes at measured HBM bandwidth and its flops at the
    sustained bf16 peak), summed over the step's launches; the row kernels
    (RMSNorms, RoPE, embedding) as HBM traffic."""
    w = step_work(sh, C, K, ctx_lens)
    nM, nA = sh.layers.count("M"), sh.layers.count("A")
    nL = len(sh.layers)
    count = {"in_proj": nM, "inject": nM, "ssd_scan": nM, "out_proj": nM,
             "qkv_proj": nA, "attn_paged": nA, "o_proj": nA}
    if sh.d_ff:
        count.update(mlp_gate_up=nL, mlp_down=nL)
    if sh.vocab:
        count["lm_head_argmax"] = 1
    hbm, tf = peaks["hbm_gbs"] * 1e9, peaks["bf16_tflops_sustained"] * 1e12
    sec = sum(n * max(w[g]["bytes"] / hbm, w[g]["flops"] / tf) for g, n in count.items() if g in w)
    M, E = C * K, (2 if sh.dtype == "bf16" else 4)
    row_bytes = (nL * (2 if sh.d_ff else 1) + 1) * M * sh.d * (4 + E)          # RMSNorms
    row_bytes += nM * M * sh.H * sh.P * (4 + 2 * E)                          # gated RMSNorm
    row_bytes += nA * M * (sh.Hq + sh.Hkv) * sh.D * 2 * E                    # RoPE
    row_bytes += M * sh.d * (E + 4) if sh.vocab else 0                       # embedding
    return (sec + row_bytes / hbm) * 1e3


# DRAM bytes (read + write) per algorithmic byte of the paged-attention kernel, from
# one ncu capture (dram__bytes_read.sum + dram__bytes_write.sum) of the current
# attn_tc_kernel at Llama-3-8B shapes, C=32, ctx U[512,8192]: 664.1 MB (657.4 read, 6.8
# written) for 658.3 MB of algorithmic bytes as step_work counts them (K/V, q, output,
# block k/v).  The K/V tiles are loaded evict-first, so the pieces' partials stay in L2
# during the kernel and the merge reads them there.  The step's attention launch is too
# large to capture; its traffic is this ratio times its algorithmic bytes (traffic grows
# with the K/V read).  None whenever the kernel has changed since the last capture.
ATTN_TRAFFIC_PER_BYTE = 1.0089


def roofline_of(name, work, avg_ms, peaks, traffic=None, sustained=True):
    """hbm- or tensor-bound roofline fraction of one kernel group."""
    fl, by = work["flops"], work["bytes"]
    tf_peak = peaks["bf16_tflops_sustained"] if sustained else peaks["bf16_tflops"]
    t_tensor = fl / (tf_peak * 1e12)
    t_hbm = by / (peaks["hbm_gbs"] * 1e9)
    sec = avg_ms / 1e3
    if name in ("attn_paged", "ssd_scan") or t_hbm >= t_tensor:
        ach = by / sec / 1e9
        return {"bound": "hbm", "achieved": round(ach, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(ach / peaks["hbm_gbs"], 4), "traffic": traffic}
    ach = fl / sec / 1e12
    return {"bound": "tensor", "achieved": round(ach, 1), "peak": tf_peak, "unit": "TFLOP/s",
            "frac": round(ach / tf_peak, 4), "traffic": traffic}


def kernel_table(prof, work, steps, pass_ms, peaks, traffic_ratio=None):
    """Per kernel group of a profiled pass: average ms per launch, launches per step,
    share of the pass, and its roofline (traffic scaled from the attention capture)."""
    ratio = ATTN_TRAFFIC_PER_BYTE if traffic_ratio is None else traffic_ratio
    kernels = {}
    for name, (tot, cnt) in prof.items():
        avg = tot / max(cnt, 1)
        ent = {"avg_ms": round(avg, 4), "launches_per_step": cnt / steps,
               "share": round(tot / (pass_ms * steps), 4)}
        if name in work:
            traffic = None
            if name == "attn_paged" and ratio is not None:
                traffic = round(ratio * work[name]["bytes"])
            ent["roofline"] = roofline_of(name, work[name], avg, peaks, traffic=traffic)
        kernels[name] = ent
    return kernels


def compact_kernels(kernels):
    """{group: [ms per launch, launches per step, fraction of its roofline]} -- the
    per-kernel view of one sweep point."""
    return {k: [v["avg_ms"], v["launches_per_step"], v.get("roofline", {}).get("frac")] for k, v in kernels.items()}


def attention_configs(H, I, dev, peaks, warmup=3, warm_s=0.25, timed_s=0.2, local=0):
    """hspec_attn_paged_block alone on the two attention-heavy workloads: Llama-3-8B
    shapes at 32 requests (ctx U[512,8192]) and Qwen-32B shapes at 128 requests (ctx
    U[1024,32768]); CUDA events on the launching stream, K/V pools larger than L2.

    The kernel runs alone for warm_s seconds before it is timed: its time follows the
    SM clock, and the clock it is timed at is then the one it sustains by itself rather
    than the one the GEMM-heavy steps before it left under the power cap.  The timed
    calls span about timed_s seconds, and the SM clock sampled over them is reported."""
    out = {}
    for name in ("llama_c32", "qwen_c128"):
        wl = I.WORKLOADS[name]
        sh, C, K = wl.shapes, wl.C, wl.K
        clocks = ClockSampler(local)
        clocks.start()  # before the inputs are built: sampling by the time the calls are timed
        cfg = H.make_cfg(sh)
        inp = I.make_attn_inputs(sh, wl, K, wl.seed, dev, shuffle=wl.shuffle, slack=wl.slack)
        kv = H.kv_view(inp)
        ws = H.alloc_workspace(H.hspec_attn_workspace_size(cfg, C, K, kv.max_pages), dev)
        o = torch.empty_like(inp["q"])
        ctx = int(inp["ctx_lens"].sum())
        work = {"bytes": float(ctx * sh.Hkv * sh.D * 2 * 2 + 2 * C * K * (sh.Hq + sh.Hkv) * sh.D * 2),
                "flops": 4.0 * sh.Hq * sh.D * K * (ctx + C * K)}
        call = lambda: H.hspec_attn_paged_block(cfg, inp["q"], kv, inp["ctx_lens"], inp["k_blk"], inp["v_blk"], o, ws)
        for _ in range(warmup):
            call()
        torch.cuda.synchronize()
        if H.hspec_sync_status() != 0:
            raise RuntimeError(H.hspec_last_error())
        n_warm, tw = 0, time.monotonic()
        while True:
            for _ in range(8):
                call()
            torch.cuda.synchronize()
            n_warm += 8
            if time.monotonic() - tw >= warm_s:
                break
        per_call = (time.monotonic() - tw) / n_warm
        steps = int(min(2000, max(20, timed_s / max(per_call, 1e-6))))
        stream = torch.cuda.current_stream()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        t0 = time.monotonic()
        e0.record(stream)
        for _ in range(steps):
            call()
        e1.record(stream)
        torch.cuda.synchronize()
        clocks.window(t0, time.monotonic())
        clk = clocks.stop()
        if H.hspec_sync_status() != 0:
            raise RuntimeError(H.hspec_last_error())
        ms = e0.elapsed_time(e1) / steps
        roof = roofline_of("attn_paged", work, ms, peaks, sustained=False)
        out[name] = {"workload": wl.description, "us_per_call": round(ms * 1e3, 1),
                     "achieved_gbs": roof["achieved"], "frac_of_hbm": roof["frac"], "calls": steps,
                     "clocks": clk}
        del inp, kv, ws, o
        torch.cuda.empty_cache()
    return out


# ---------------------------------------------------------------------- our arm

class StepRunner:
    def __init__(self, H, I, wl, device, weights=None):
        self.H, self.wl, self.sh = H, wl, wl.shapes
        self.st = I.make_step_inputs(wl, device, weights=weights is None)
        if weights is not None:
            self.st["weights"] = weights
        C, K, sh = wl.C, wl.K, self.sh
        self.dr = H.Drafter(sh, self.st["weights"])
        self.max_pages = max(c["page_table"].shape[1] for c in self.st["kv"])
        self.ws = H.alloc_workspace(self.dr.workspace_size(C, K, self.max_pages), device)
        self.tokens_out = torch.empty(C, K, dtype=torch.int32, device=device)
        self.si = self.dr.step_in(C, K, self.st["h_last"], self.st["ctx_lens"], self.st["kv"],
                                  tokens=self.st["tokens"], x_in=self.st["x_in"])
        self.so = H.hspec_step_out(draft_tokens=self.tokens_out.data_ptr())

    def step(self):
        self.dr.step(self.si, self.so, self.ws)

    def check(self):
        s = self.H.hspec_sync_status()
        if s != 0:
            raise RuntimeError(f"draft step failed: {self.H.hspec_status_string(s)} ({self.H.hspec_last_error()})")

    def close(self):
        self.dr.close()


def time_steps(runner, steps, warmup, world, profile=False, clocks=None):
    H = runner.H
    for _ in range(warmup):
        runner.step()
    runner.check()
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if profile:
        H.hspec_profile_enable(True)
    n0 = H.hspec_launch_count()
    barrier(world)
    torch.cuda.synchronize()
    t0 = time.monotonic()
    e0.record(stream)
    for _ in range(steps):
        runner.step()
    e1.record(stream)
    torch.cuda.synchronize()
    if clocks is not None:
        clocks.window(t0, time.monotonic())
    barrier(world)
    launches = H.hspec_launch_count() - n0
    prof = H.hspec_profile_read() if profile else {}
    if profile:
        H.hspec_profile_enable(False)
    runner.check()
    return e0.elapsed_time(e1) / steps, launches, prof


def time_e2e(runner, steps):
    """Same step through the C-ABI with host inputs: every step copies h_last, block
    tokens, ctx_lens and the page tables from pinned host memory and reads the
    draft tokens back."""
    st = runner.st
    dev_in = [st["h_last"], st["tokens"], st["ctx_lens"]] + [c["page_table"] for c in st["kv"]]
    host_in = [t.to("cpu").pin_memory() for t in dev_in]
    host_out = torch.empty(runner.tokens_out.shape, dtype=torch.int32).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host_in)
    d2h = host_out.numel() * host_out.element_size()
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    e0.record(stream)
    for _ in range(steps):
        for d, h in zip(dev_in, host_in):
            d.copy_(h, non_blocking=True)
        runner.step()
        host_out.copy_(runner.tokens_out, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    wall = (time.perf_counter() - t0) / steps
    runner.check()
    return e0.elapsed_time(e1) / steps, wall * 1e3, h2d, d2h


def oracle_one_request(I, wl, runner=None, device="cpu", request=0):
    """Times the CPU oracle on one request of the workload (requests are
    independent, so C requests cost C times this)."""
    import oracle
    st = runner.st if runner is not None else I.make_step_inputs(wl, device)
    w = oracle.host_weights(st["weights"])
    rows = [request]
    kv = [oracle.host_sub_cache(c, rows) for c in st["kv"]]
    args = dict(tokens=st["tokens"].cpu()[rows] if st["tokens"] is not None else None,
                x_in=st["x_in"].cpu()[rows] if st["x_in"] is not None else None)
    h_last, lens = st["h_last"].cpu()[rows], st["ctx_lens"].cpu()[rows]
    t0 = time.perf_counter()
    oracle.draft_step(wl.shapes, w, kv, h_last, lens, **args)
    return time.perf_counter() - t0, int(lens[0]), oracle.threads()


def run_ours(args, rank, world, local):
    from hybrid_mamba_attention_b200 import hspec as H
    from hybrid_mamba_attention_b200 import inputs as I
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peaks = load_peaks()
    wl = replica_workload(I, I.full_workload(args.C, args.K, args.draft_vocab), rank)
    clocks = ClockSampler(local)
    clocks.start()  # before the inputs are built: sampling by the time the steps run
    runner = StepRunner(H, I, wl, dev)
    ms, launches, _ = time_steps(runner, args.steps, args.warmup, world, clocks=clocks)
    clk = clocks.stop()
    ms_max, value = replica_throughput(wl.C * wl.K, ms, world)
    # Per-kernel-group times: a second timed pass of the same steps with CUDA events
    # recorded around each group on the step's stream.  The events sit between the
    # kernels (so the next kernel no longer starts before the previous one ends), which
    # is why the headline steps above run without them.
    pms, _, prof = time_steps(runner, args.steps, args.warmup, world, profile=True)

    # roofline: per kernel group, from the events recorded on the step's stream
    work = step_work(wl.shapes, wl.C, wl.K, runner.st["ctx_lens"].cpu())
    kernels = kernel_table(prof, work, args.steps, pms, peaks)
    dominant = max(kernels, key=lambda k: kernels[k]["share"]) if kernels else None
    roof = dict(kernels[dominant]["roofline"]) if dominant and "roofline" in kernels[dominant] else None
    if roof:
        roof["kernel"] = dominant
        roof["peak_source"] = f"{peaks['source']} (MEASURED_PEAKS.json)" if peaks["source"] == "measured" else "fallback"
    attn_roof = kernels.get("attn_paged", {}).get("roofline")

    e2e_ms, e2e_wall_ms, h2d, d2h = time_e2e(runner, args.steps)
    e2e_ms, e2e_value = replica_throughput(wl.C * wl.K, e2e_ms, world)
    e2e = {"value": round(e2e_value, 1), "unit": UNIT, "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 4), "wall_ms_per_step": round(e2e_wall_ms, 4)}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        secs, ctx, cores = oracle_one_request(I, wl, runner)
        cpu = {"value": round(wl.K / secs, 3), "unit": UNIT, "cores": cores, "kind": "oracle",
               "sample": f"1 of {wl.C} requests (ctx {ctx}, K={wl.K}) through the full M,A,M,A step "
                         f"+ LM head; {secs:.2f} s; requests are independent so C requests take C times as long"}

    # concurrency sweep: draft-step latency and drafted tokens/s at C = 1 .. 128 (K = 16;
    # with --sweep also K = 8 and 32), each against the step's roofline.  The main
    # measurement above is the C = 128, K = 16 point.  Each other point runs on its own
    # batch with the weights shared and the headline batch's KV pools and workspace
    # released first: left resident, 17 GB of unrelated KV slowed the C = 1 step by 8-15%
    # (page-table reach), which no workload of that size sees.
    headline_lens = runner.st["ctx_lens"].cpu()
    weights = runner.st["weights"]
    runner.close()
    del runner
    torch.cuda.empty_cache()
    sweep = []
    for K in (I.FULL_SWEEP_K if args.sweep else (args.K,)):
        for C in I.FULL_SWEEP_C:
            if C == wl.C and K == wl.K:
                m2, lens2, k2 = ms_max, headline_lens, kernels
            else:
                w2 = I.full_workload(C, K, args.draft_vocab)
                r2 = StepRunner(H, I, w2, dev, weights=weights)
                n2 = max(5, args.steps // 2)
                m2, _, _ = time_steps(r2, n2, max(5, args.warmup), 1)
                p2, _, prof2 = time_steps(r2, n2, 1, 1, profile=True)
                lens2 = r2.st["ctx_lens"].cpu()
                k2 = kernel_table(prof2, step_work(wl.shapes, C, K, lens2), n2, p2, peaks)
                r2.close()
                del r2
                torch.cuda.empty_cache()
            roof_ms = step_roofline_ms(wl.shapes, C, K, lens2, peaks)
            sweep.append({"C": C, "K": K, "us_per_step": round(m2 * 1e3, 1),
                          "tokens_per_s": round(C * K / (m2 / 1e3), 1),
                          "roofline_us": round(roof_ms * 1e3, 1), "frac_of_roofline": round(roof_ms / m2, 4),
                          "kernels": compact_kernels(k2)})
    del weights
    torch.cuda.empty_cache()

    # the paged attention alone on the attention-heavy workloads (rank 0, one GPU)
    attn_cfg = attention_configs(H, I, dev, peaks, local=local) if (rank == 0 and not args.no_attention_configs) else None

    if rank == 0:
        line = {"metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": round(ms_max, 4), "us_per_step": round(ms_max * 1e3, 1),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic (seeded random-init weights and KV of the stated shapes)",
                "config": step_config(wl, world),
                "roofline": roof, "attention_roofline": attn_roof, "kernels": kernels,
                "kernels_pass_ms_per_step": round(pms, 4),
                "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches, "clocks": clk,
                "attention_configs": attn_cfg}
        if sweep is not None:
            line["sweep"] = sweep
        print(json.dumps(line), flush=True)


# ------------------------------------------------------------- kernel-level mode

def run_kernel(args, rank, world, local):
    """Times one C-ABI call (attn / inject / ssd) on a kernel-level workload, with
    CUDA events on the launching stream; inputs exceed L2 except the tiny workload."""
    from hybrid_mamba_attention_b200 import hspec as H
    from hybrid_mamba_attention_b200 import inputs as I
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peaks = load_peaks()
    m = re.fullmatch(r"full_C(\d+)_K(\d+)", args.workload)
    wl = I.full_workload(int(m.group(1)), int(m.group(2))) if m else I.WORKLOADS[args.workload]
    sh, C, K = wl.shapes, wl.C, wl.K
    cfg = H.make_cfg(sh)
    E = 2 if sh.dtype == "bf16" else 4
    if args.kernel == "attn":
        inp = I.make_attn_inputs(sh, wl, K, wl.seed, dev, shuffle=wl.shuffle, slack=wl.slack)
        kv = H.kv_view(inp)
        ws = H.alloc_workspace(H.hspec_attn_workspace_size(cfg, C, K, kv.max_pages), dev)
        out = torch.empty_like(inp["q"])
        call = lambda: H.hspec_attn_paged_block(cfg, inp["q"], kv, inp["ctx_lens"], inp["k_blk"], inp["v_blk"], out, ws)
        ctx = int(inp["ctx_lens"].sum())
        work = {"bytes": float(ctx * sh.Hkv * sh.D * 2 * E + 2 * C * K * sh.Hq * sh.D * E),
                "flops": 4.0 * sh.Hq * sh.D * K * (ctx + C * K)}
        name = "attn_paged"
    elif args.kernel == "gemm":
        # the tcgen05 GEMM alone in its tensor-bound regime: the injection GEMM of an
        # eighth of the heads (N = H/8 * P * N_state) for all C*K block rows (M = 2048 at
        # C=128, K=16), K = d; about 1.1 GB on the device
        sh8 = replace(sh, H=max(1, sh.H // 8))
        HPN, Mr = sh8.H * sh8.P * sh8.N, C * K
        inp = I.make_inject_inputs(sh8, Mr, wl.seed, dev)
        h0 = torch.empty(Mr, HPN, device=dev)
        gcfg = H.make_cfg(sh8)
        call = lambda: H.hspec_inject_state(gcfg, inp["W_inj"], inp["h_last"], h0)
        work = {"bytes": float(HPN * sh.d * E + Mr * HPN * 4 + Mr * sh.d * E), "flops": 2.0 * Mr * HPN * sh.d}
        name = "gemm_tc"
    elif args.kernel == "verify":
        # the target's logits for the K + 1 block positions of every request (synthetic)
        V = sh.vocab or 128256
        g = torch.Generator(device=dev).manual_seed(wl.seed)
        logits = torch.randn(C, K + 1, V, generator=g, device=dev).to(sh.torch_dtype)
        drafts = torch.randint(0, V, (C, K), generator=g, device=dev, dtype=torch.int32)
        vcfg = H.make_cfg(replace(sh, vocab=V))
        ws = H.alloc_workspace(H.hspec_verify_workspace_size(vcfg, C, K), dev)
        acc = torch.empty(C, dtype=torch.int32, device=dev)
        nxt = torch.empty(C, dtype=torch.int32, device=dev)
        call = lambda: H.hspec_verify_greedy(vcfg, logits, drafts, acc, nxt, ws)
        work = {"bytes": float(C * (K + 1) * V * E), "flops": 0.0}
        name = "verify_greedy"
    elif args.kernel == "inject":
        inp = I.make_inject_inputs(sh, C, wl.seed, dev)
        HPN = sh.H * sh.P * sh.N
        h0 = torch.empty(C, HPN, device=dev)
        call = lambda: H.hspec_inject_state(cfg, inp["W_inj"], inp["h_last"], h0)
        work = {"bytes": float(HPN * sh.d * E + C * HPN * 4 + C * sh.d * E), "flops": 2.0 * C * HPN * sh.d}
        name = "inject"
    else:
        inp = I.make_ssd_inputs(sh, C, K, wl.seed, dev)
        y = torch.empty(C, K, sh.H, sh.P, device=dev)
        call = lambda: H.hspec_ssd_block_scan(cfg, inp["x"], inp["dt"], inp["A"], inp["B"], inp["Cm"], inp["D"],
                                              inp["h0"], y)
        HPN = sh.H * sh.P * sh.N
        work = {"bytes": float(C * HPN * 4 + C * K * (sh.H * sh.P + 2 * sh.N) * E + C * K * sh.H * 4
                               + C * K * sh.H * sh.P * 4),
                "flops": float(C * sh.H * (2 * K * sh.P * sh.N + K * K * (sh.N + sh.P)))}
        name = "ssd_scan"
    for _ in range(args.warmup):
        call()
    if H.hspec_sync_status() != 0:
        raise RuntimeError(H.hspec_last_error())
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n0 = H.hspec_launch_count()
    clocks = ClockSampler(local)
    clocks.start()
    torch.cuda.synchronize()
    t0 = time.monotonic()
    e0.record(stream)
    for _ in range(args.steps):
        call()
    e1.record(stream)
    torch.cuda.synchronize()
    clocks.window(t0, time.monotonic())
    clk = clocks.stop()
    if H.hspec_sync_status() != 0:
        raise RuntimeError(H.hspec_last_error())
    ms = e0.elapsed_time(e1) / args.steps
    roof = roofline_of(name, work, ms, peaks, sustained=False)
    line = {"metric": f"{name} call time", "value": round(ms * 1e3, 2), "unit": "us", "higher_is_better": False,
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "dtype": sh.dtype,
            "config": {"workload": wl.description, "kernel": name, "C": C, "K": K},
            "roofline": roof, "gpu_launches": H.hspec_launch_count() - n0, "clocks": clk,
            "algorithmic_bytes": work["bytes"], "algorithmic_flops": work["flops"]}
    if rank == 0:
        print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- reference arm

def step_config(wl, world):
    """The `config` object of the draft-step line, the same for both arms."""
    return {"workload": f"full draft step {wl.name}: 4-layer M,A,M,A hybrid drafter, Llama-3-8B shapes, "
                        f"SwiGLU 16384, vocab 128256"
                        + (f" (draft head {wl.shapes.draft_vocab} rows)" if wl.shapes.draft_vocab else "")
                        + ", ctx U[512,16384], 16-token pages",
            "C": wl.C, "K": wl.K, "global_batch": wl.C * world, "parallelism": f"replicas x{world}",
            "l2": "inputs ~20 GB > 126 MB L2 (no flush needed)"}


def run_reference(args, rank, world):
    """The CPU oracle as the reference arm, on this arm's config and metric."""
    if rank != 0:
        return
    from hybrid_mamba_attention_b200 import inputs as I
    wl = I.full_workload(args.C, args.K, args.draft_vocab)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    st = I.make_step_inputs(wl, dev)

    class _R:
        pass

    r = _R()
    r.st = st
    import oracle  # noqa: F401
    for i in range(args.warmup):
        oracle_one_request(I, wl, r, request=i % wl.C)
    times = []
    for i in range(args.steps):
        secs, ctx, cores = oracle_one_request(I, wl, r, request=i % wl.C)
        times.append(secs)
    sec = sum(times) / len(times)
    value = wl.K / sec
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(sec * 1e3, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded random-init weights and KV of the stated shapes)",
            "config": step_config(wl, world),
            "cpu_baseline": {"value": round(value, 3), "unit": UNIT, "cores": oracle.threads(), "kind": "oracle",
                             "sample": f"one request of the {wl.C}-request batch per step (requests are "
                                       f"independent, so the batch takes C times as long)"},
            "e2e": {"value": round(value, 3), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["hspec", "reference"], default="hspec")
    ap.add_argument("--C", type=int, default=128)
    ap.add_argument("--K", type=int, default=16)
    ap.add_argument("--draft-vocab", type=int, default=0,
                    help="reduced draft head rows (0 = the full 128256-token head)")
    ap.add_argument("--sweep", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-attention-configs", action="store_true",
                    help="skip timing the paged attention alone on the Llama C=32 and Qwen C=128 workloads")
    ap.add_argument("--kernel", choices=["step", "attn", "inject", "ssd", "verify", "gemm"], default="step",
                    help="time one C-ABI call on --workload instead of the full draft step")
    ap.add_argument("--workload", default="llama_c32", help="kernel-level workload (tiny, llama_c1, llama_c32, qwen_c128, or full_C<C>_K<K>: one layer of the full step)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    rank, world, local = dist_setup(args.gpus)
    try:
        if args.impl == "reference":
            run_reference(args, rank, world)
        elif args.kernel != "step":
            run_kernel(args, rank, world, local)
        else:
            run_ours(args, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
