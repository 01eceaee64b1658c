"""Benchmark of the fused LoRA + SwiGLU MLP forward + backward on B200.

python bench.py [--gpus N] [--steps K] [--warmup W] [--impl b200|reference] [--workload NAME]

The default workload is the MLP on the Llama-3-8B shapes.  --workload
llama3_8b_qproj / llama3_8b_kproj instead times the single LoRA linear
projection (forward + backward) with the same JSON contract.

One step = forward + backward of the whole hot path over one batch of
synthetic tokens (all kernels: rank-r projections, gate/up GEMM with SwiGLU
epilogue, down GEMM, dH GEMM with SwiGLU-backward epilogue, dX GEMM, the
adapter-gradient reductions).  Inputs are resident in HBM when the timed
region starts; the frozen weights (352 MB on the default workload) are larger
than the 126 MB L2, so no L2 flush is needed between steps.

For N > 1 (torchrun) every rank runs an independent replica of the same
workload (the MLP has no exchange step on this path), the barrier-bracketed
device time is the max over ranks, and `value` is the total tokens of all
ranks over that time ("weak" scaling).

--impl reference times the fp64 CPU oracle on the host cores instead, on a
bounded token sample of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

from lora_fine_tuning_mlp_b200 import inputs as synth  # noqa: E402

METRIC = "fused LoRA-SwiGLU MLP fwd+bwd tokens/s and TFLOP/s vs bf16 dense peak"
LINEAR_METRIC = "fused LoRA linear fwd+bwd tokens/s and TFLOP/s vs bf16 dense peak"
CE_METRIC = "chunked cross-entropy fwd+bwd tokens/s and GB/s vs HBM bandwidth"
DEFAULT_WORKLOAD = "llama3_8b_mlp"
SUSTAINED_MS = 2000.0  # timed regions at least this long are held to the sustained (power-capped) peak


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            p = json.load(fh)
        return {"bf16_tflops": p.get("bf16_tflops", 1590.0),
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained", 1400.0),
                "hbm_gbs": p.get("hbm_gbs", 6650.0), "source": "measured"}
    return {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0, "source": "fallback"}


def csrc_sha256() -> str:
    """Hash of the translation unit the GEMM kernels are built from (lora_mlp.cu
    and every local file it includes, transitively), to tell whether a stored
    ncu figure still applies to the kernels the current sources compile to.
    Comments and blank space are left out, so that an edit to documentation
    alone keeps the figure."""
    import hashlib
    import re as _re
    csrc = os.path.join(ROOT, "lora_fine_tuning_mlp_b200", "csrc")
    inc = os.path.join(ROOT, "include")
    seen, todo = [], ["lora_mlp.cu"]
    while todo:
        f = todo.pop(0)
        if f in seen:
            continue
        path = next((os.path.join(dd, f) for dd in (csrc, inc) if os.path.exists(os.path.join(dd, f))), None)
        if path is None:
            continue
        seen.append(f)
        with open(path, "rb") as fh:
            text = fh.read()
        todo += [m.decode() for m in _re.findall(rb'#include\s+"([^"]+)"', text)]
    h = hashlib.sha256()
    for f in sorted(seen):
        path = next(os.path.join(dd, f) for dd in (csrc, inc) if os.path.exists(os.path.join(dd, f)))
        h.update(f.encode())
        with open(path, "rb") as fh:
            code = _re.sub(rb"/\*.*?\*/|//[^\n]*", b" ", fh.read(), flags=_re.S)
        h.update(b" ".join(code.split()))
    return h.hexdigest()


def ncu_traffic(workload: str, kernel: str):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, or
    None when there is none or the kernels changed since it was taken."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as fh:
            rec = json.load(fh)
    except (OSError, ValueError):
        return None
    if rec.get("csrc_sha256") != csrc_sha256():
        return None
    return rec.get(workload, {}).get(kernel, {}).get("dram_bytes")


def gemm_flops(cfg) -> dict:
    """Algorithmic flops of each tensor-core GEMM launch (2 per multiply-add)."""
    N, d, f, r = cfg.N, cfg.d, cfg.d_ff, cfg.r
    return {
        "F1_gate_up_swiglu": 2.0 * N * f * (2 * d + 2 * r),
        "F3_down": 2.0 * N * d * (f + r),
        "B1_dh_swiglu_bwd": 2.0 * N * f * (d + r),
        "B4_dX": 2.0 * N * d * (2 * f + 2 * r),
        "F0_lowrank_in": 2.0 * N * d * 2 * r,
        "F2_lowrank_mid": 2.0 * N * f * r,
        "B0_lowrank_out": 2.0 * N * d * r,
        "B0_dBd": 2.0 * N * d * r,
        "B2_dAd": 2.0 * N * f * r,
        "B3_lowrank_gu": 2.0 * 2 * N * f * r,
        "B3_dBgu": 2.0 * 2 * N * f * r,
        "B5_dA_in": 2.0 * N * d * 2 * r,
    }


# ----------------------------------------------------------------------------- clocks


class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(self.idx)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True, bufsize=1)
        except (OSError, ValueError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.monotonic(), line.strip()))

    def stop(self, window=None):
        """Median SM clock and the throttle reasons seen.  With `window` =
        (t0, t1) in time.monotonic() seconds, only the samples read while the
        timed region ran count (plus one sampling interval after it)."""
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        lines = self.lines
        if window is not None:
            inside = [(t, ln) for t, ln in lines if window[0] <= t <= window[1] + 0.15]
            if inside:
                lines = inside
        for _, ln in lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- CPU oracle timing


def weight_format_name(cfg) -> str:
    return "int4_b64" if cfg.int4 else ("fp8_e4m3_b64" if getattr(cfg, "fp8", False) else "bf16")


def oracle_inputs(cfg, block=False):
    c = synth.custom(min(cfg.N, 4096), cfg.d, cfg.d_ff, cfg.r, cfg.alpha, cfg.int4, seed_index=cfg.index,
                     fp8=cfg.fp8)
    return synth.make_block_inputs(c) if block else synth.make_inputs(c)


def oracle_step(p, x, dOut, alpha, gamma=None):
    """One fp64 oracle forward + backward (of the pre-norm block when gamma is given)."""
    import oracle
    from oracle import rmsnorm as orn

    if gamma is None:
        p["X"] = x
        oracle.backward(p, alpha, dOut, oracle.forward(p, alpha))
        return
    xn, rstd = orn.rmsnorm_forward(x, gamma, synth.RMS_EPS)
    p["X"] = xn
    b = oracle.backward(p, alpha, dOut, oracle.forward(p, alpha))
    orn.rmsnorm_backward(x, gamma, rstd, b["dX"])


def time_oracle(cfg, budget_s: float, inp=None, block=False, repeat=False):
    """Time the fp64 oracle forward+backward on a token sample of `cfg` sized
    to take about budget_s.  When the whole workload takes well under the
    budget and `repeat` is set, further passes over it are timed until most
    of the budget is spent.  Returns (tokens/s, sample tokens, seconds,
    passes)."""
    import oracle

    if inp is None:
        inp = oracle_inputs(cfg, block)
    p_full = oracle.weights_f64({k: v for k, v in inp.items() if k not in ("X", "dOut", "gamma")})
    gamma = oracle.bf16_to_f64(inp["gamma"]) if block else None

    def run(n):
        p = dict(p_full)
        x = oracle.bf16_to_f64(inp["X"][:n])
        dOut = oracle.bf16_to_f64(inp["dOut"][:n])
        t0 = time.perf_counter()
        oracle_step(p, x, dOut, cfg.alpha, gamma)
        return time.perf_counter() - t0

    t_probe = run(32)
    n = int(32 * budget_s / max(t_probe, 1e-3))
    n = max(32, min(n, inp["X"].shape[0]))
    n = n // 32 * 32
    dt = run(n)
    passes = 1
    while repeat and dt < 0.6 * budget_s and passes < 64:
        dt += run(n)
        passes += 1
    return n * passes / dt, n, dt, passes


def threads_used() -> int:
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        if info:
            return max(int(i.get("num_threads", 1)) for i in info)
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


# ----------------------------------------------------------------------------- arms


def reference_arm(args, cfg):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    per_step = max(2.0, min(20.0, 150.0 / max(1, args.steps + args.warmup)))
    import oracle

    block = getattr(args, "block", False)
    inp = oracle_inputs(cfg, block)
    _, n, _, _ = time_oracle(cfg, per_step, inp, block)
    p_full = oracle.weights_f64({k: v for k, v in inp.items() if k not in ("X", "dOut", "gamma")})
    gamma = oracle.bf16_to_f64(inp["gamma"]) if block else None
    times = []
    for i in range(args.warmup + args.steps):
        lo = (i * n) % inp["X"].shape[0]
        idx = np.arange(lo, lo + n) % inp["X"].shape[0]
        p = dict(p_full)
        x = oracle.bf16_to_f64(inp["X"][idx])
        dOut = oracle.bf16_to_f64(inp["dOut"][idx])
        t0 = time.perf_counter()
        oracle_step(p, x, dOut, cfg.alpha, gamma)
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            times.append(dt)
    total = sum(times)
    value = n * len(times) / total
    cores = threads_used()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * total / len(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_dict(cfg, getattr(args, "block", False)),
        "tflops": cfg.flops() * (n / cfg.N) * len(times) / total / 1e12,
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"{n} tokens of the {cfg.name} shapes per step (numpy fp64 oracle"
                                   + (", pre-norm block" if block else "") + ")"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_dict(cfg, block=False):
    if block:
        d = config_dict(cfg)
        d["workload"] = "llama3_8b_block" if cfg.name == "llama3_8b_mlp" else cfg.name + "_block"
        d["prenorm"] = f"RMSNorm (frozen gain), eps {synth.RMS_EPS}; out = MLP(RMSNorm(X))"
        return d
    w_mb = 3 * cfg.d * cfg.d_ff * (0.53125 if cfg.int4 else (1.0625 if cfg.fp8 else 2)) / 1e6
    x_mb, h_mb = 2 * cfg.N * cfg.d / 1e6, 2 * cfg.N * cfg.d_ff / 1e6
    sizes = "frozen weights %.0f MB, X %.0f MB, g/u/h %.0f MB each" % (w_mb, x_mb, h_mb)
    # a step reads the weights, X, dOut and writes/reads g, u, h, dg, du
    step_mb = w_mb + 2 * x_mb + 5 * h_mb
    l2 = ("no flush: a step's operands exceed the 126 MB L2 (%s)" % sizes if step_mb > 126.0 else
          "no flush; a step's operands fit in the 126 MB L2 (%s): a launch-bound parity case, not a "
          "throughput workload" % sizes)
    return {"workload": cfg.name, "N_tokens": cfg.N, "d": cfg.d, "d_ff": cfg.d_ff, "r": cfg.r, "alpha": cfg.alpha,
            "frozen_weights": weight_format_name(cfg), "l2": l2, "parallelism": "replicas"}


def b200_arm(args, cfg):
    import torch
    import torch.distributed as dist

    from lora_fine_tuning_mlp_b200 import _lib, api

    from lora_fine_tuning_mlp_b200 import replicas

    rank, local, world = replicas.world()
    if world > 1:
        torch.cuda.set_device(local)
        replicas.init("nccl", device=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())
    _lib.lib()

    block = args.block
    inp = synth.make_block_inputs(cfg) if block else synth.make_inputs(cfg)
    w = api.weights_from_host(inp, cfg.alpha, dev)
    X = api.to_device_bf16(inp["X"], dev)
    dOut = api.to_device_bf16(inp["dOut"], dev)
    gamma = api.to_device_bf16(inp["gamma"], dev) if block else None
    eps = synth.RMS_EPS
    N, d, f = cfg.N, cfg.d, cfg.d_ff
    out = torch.empty((N, d), dtype=torch.bfloat16, device=dev)
    dX = torch.empty((N, d), dtype=torch.bfloat16, device=dev)
    grads = {("d" + k): torch.empty_like(getattr(w, k)) for k in ("Ag", "Bg", "Au", "Bu", "Ad", "Bd")}
    wsf, wsb = api.Workspace(), api.Workspace()
    stream = torch.cuda.current_stream()

    def fwd(x=X):
        if block:
            return api.block_forward(x, w, gamma, eps, out=out, workspace=wsf)
        return api.forward(x, w, out=out, workspace=wsf)

    def bwd(saved, x=X, g_out=dOut):
        if block:
            return api.block_backward(x, w, gamma, saved, g_out, dX=dX, grads=grads, workspace=wsb)
        return api.backward(x, w, saved, g_out, dX=dX, grads=grads, workspace=wsb)

    def step(x=X, g_out=dOut):
        o, saved = fwd(x)
        bwd(saved, x, g_out)

    barrier = replicas.barrier

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    # ---- device-timed region: K steps, inputs resident in HBM.  No per-kernel
    # events here: an event between two launches would stop the next kernel
    # from starting under the previous one's tail (programmatic dependent
    # launch), so `value` is taken without them.
    sampler = ClockSampler(dev.index)
    launches0 = _lib.launch_count()
    barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    w0 = time.monotonic()
    t0.record(stream)
    for _ in range(args.steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize()
    w1 = time.monotonic()
    barrier()
    clocks = sampler.stop((w0, w1))
    launches = _lib.launch_count() - launches0
    ms_max = replicas.max_over_ranks(t0.elapsed_time(t1), device=dev)

    # ---- forward alone and backward alone (same protocol, device-timed)
    _, saved_fb = fwd()

    def timed_region(fn):
        barrier()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.steps):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        barrier()
        return replicas.max_over_ranks(a.elapsed_time(b), device=dev) / args.steps

    fwd_ms = timed_region(fwd)
    bwd_ms = timed_region(lambda: bwd(saved_fb))
    del saved_fb

    # ---- second timed region of the same work with the library's CUDA events
    # around every launch (on the stream each kernel runs on): the per-kernel
    # durations behind the roofline figures.
    _lib.timing_enable(True)
    _lib.timing_collect()
    barrier()
    torch.cuda.synchronize()
    for _ in range(args.steps):
        step()
    torch.cuda.synchronize()
    barrier()
    recs = _lib.timing_collect()
    _lib.timing_enable(False)

    # ---- end-to-end through the public API with host buffers: every step copies
    # its X and dOut from pinned host memory (overlapped with the previous
    # step's compute) and reads its six adapter gradients back to the host.
    Xh = [torch.from_numpy(inp["X"].view("int16")).view(torch.bfloat16).pin_memory() for _ in range(2)]
    dOh = [torch.from_numpy(inp["dOut"].view("int16")).view(torch.bfloat16).pin_memory() for _ in range(2)]
    trainer = api.HostBatchTrainer(w, N, dev, gamma=gamma, eps=eps)
    h2d, d2h = trainer.h2d_bytes(), trainer.d2h_bytes()

    def run_e2e(n):
        for i in range(n):
            nxt = (i + 1) % 2 if i + 1 < n else None
            trainer.step(Xh[i % 2], dOh[i % 2], None if nxt is None else Xh[nxt], None if nxt is None else dOh[nxt])

    run_e2e(3)
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    run_e2e(args.steps)
    trainer.finish()  # the last step's gradients are home before the clock stops
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ems = replicas.max_over_ranks(e0.elapsed_time(e1), device=dev)

    # ---- per-kernel breakdown and the dominant kernel's roofline
    per = {}
    for name, kms in recs:
        s = per.setdefault(name, [0.0, 0])
        s[0] += kms
        s[1] += 1
    peaks = load_peaks()
    fl = gemm_flops(cfg)
    dom = max(per.items(), key=lambda kv: kv[1][0])[0] if per else None
    roof = None
    if dom is not None and dom in fl:
        avg_ms = per[dom][0] / per[dom][1]
        achieved = fl[dom] / (avg_ms * 1e-3) / 1e12
        # The sustained (power-capped) peak applies once the timed region lasts
        # as long as the loop it was measured with (seconds); shorter regions
        # run at burst clocks and are held to the burst peak.
        long_run = ms_max >= SUSTAINED_MS
        peak = peaks["bf16_tflops_sustained"] if long_run else peaks["bf16_tflops"]
        roof = {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": ncu_traffic(cfg.name, dom),
                "peak_source": (f"{peaks['source']} bf16_tflops_sustained (timed region {ms_max / 1e3:.2f} s)"
                                if long_run else
                                f"{peaks['source']} bf16_tflops burst (timed region {ms_max / 1e3:.2f} s, "
                                f"shorter than the {SUSTAINED_MS / 1e3:.0f} s sustained loop)"),
                "flops_per_launch": fl[dom], "avg_launch_ms": avg_ms}

    barrier()
    if rank == 0:
        per_step_ms = ms_max / args.steps
        value = replicas.job_throughput(N, args.steps, ms_max, world)
        tflops = world * cfg.flops() * args.steps / (ms_max * 1e-3) / 1e12
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": per_step_ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": config_dict(cfg, args.block),
            "tflops": tflops, "frac_of_peak": {
                "measured_burst": tflops / world / peaks["bf16_tflops"],
                "measured_sustained": tflops / world / peaks["bf16_tflops_sustained"],
                "nominal_2250": tflops / world / 2250.0},
            "roofline": roof,
            "fwd_ms_per_step": fwd_ms, "bwd_ms_per_step": bwd_ms,
            "fwd_tflops_per_gpu": cfg.flops_fwd() / (fwd_ms * 1e-3) / 1e12,
            "bwd_tflops_per_gpu": cfg.flops_bwd() / (bwd_ms * 1e-3) / 1e12,
            "e2e": {"value": replicas.job_throughput(N, args.steps, ems, world), "unit": "tokens/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "what": "api.HostBatchTrainer: per step H2D of X and dOut from pinned host (overlapped with "
                            "the previous step's compute), forward+backward, D2H of the six adapter grads "
                            "(overlapped with the next step's compute)"},
            "gpu_launches": launches,
            "clocks": {"sm_mhz": clocks["sm_mhz"], "sm_max_mhz": clocks["sm_max_mhz"],
                       "reasons": clocks["reasons"], "samples": clocks["samples"]},
            "kernels_ms_per_step": {k: v[0] / args.steps for k, v in sorted(per.items(), key=lambda kv: -kv[1][0])},
            "kernels_note": "per-launch CUDA events, second timed region of the same length (events stop launch overlap)",
        }
        if world == 1 and not args.no_cpu_baseline:
            tps, n, dt, passes = time_oracle(cfg, args.cpu_budget, block=args.block, repeat=True)
            line["cpu_baseline"] = {"value": tps, "unit": "tokens/s", "cores": threads_used(), "kind": "oracle",
                                    "sample": f"{passes} pass(es) over {n} tokens of the {cfg.name} shapes, "
                                              f"numpy fp64 oracle, {dt:.1f} s"}
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.cuda.synchronize()
        dist.destroy_process_group()
    return 0


# ----------------------------------------------------------------------------- LoRA linear legs


def linear_flops(cfg) -> dict:
    N, di, do, r = cfg.N, cfg.d_in, cfg.d_out, cfg.r
    return {
        "L0_lowrank_in": 2.0 * N * di * r,
        "L1_linear_fwd": 2.0 * N * do * (di + r),
        "L2_lowrank_out_dB": 2.0 * 2 * N * do * r,
        "L3_linear_dX": 2.0 * N * di * (do + r),
        "L4_dA": 2.0 * N * di * r,
    }


def linear_config_dict(cfg):
    return {"workload": cfg.name, "N_tokens": cfg.N, "d_in": cfg.d_in, "d_out": cfg.d_out, "r": cfg.r,
            "alpha": cfg.alpha, "frozen_weights": weight_format_name(cfg),
            "l2": "flushed: a 256 MB buffer is written between timed steps",
            "parallelism": "replicas"}


def time_linear_oracle(cfg, budget_s: float, inp):
    from oracle import lora_linear as olin

    p_full = olin.weights_f64({k: v for k, v in inp.items() if k not in ("X", "dY")})

    def run(idx):
        p = dict(p_full)
        p["X"] = olin.bf16_to_f64(inp["X"][idx])
        dY = olin.bf16_to_f64(inp["dY"][idx])
        t0 = time.perf_counter()
        olin.backward(p, cfg.alpha, dY, olin.forward(p, cfg.alpha))
        return time.perf_counter() - t0

    rows = inp["X"].shape[0]
    t_probe = run(np.arange(64))
    n = max(64, min(rows, int(64 * budget_s / max(t_probe, 1e-3)) // 64 * 64))
    return n, run


def linear_reference_arm(args, cfg):
    if int(os.environ.get("RANK", "0")) != 0:
        return 0
    inp = synth.make_linear_inputs(cfg)
    per_step = max(1.0, min(10.0, 150.0 / max(1, args.steps + args.warmup)))
    n, run = time_linear_oracle(cfg, per_step, inp)
    times = []
    for i in range(args.warmup + args.steps):
        idx = (np.arange(n) + i * n) % cfg.N
        dt = run(idx)
        if i >= args.warmup:
            times.append(dt)
    total = sum(times)
    value = n * len(times) / total
    line = {
        "impl": "reference", "metric": LINEAR_METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * total / len(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": linear_config_dict(cfg),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads_used(), "kind": "oracle",
                         "sample": f"{n} tokens of the {cfg.name} shapes per step (numpy fp64 oracle)"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def linear_arm(args, cfg):
    """One step = LoRA linear forward + backward over N tokens.  The frozen
    projection (32 MB for q) fits in L2, so a 256 MB buffer is written
    between timed steps; the flush runs outside the per-step launches but
    inside the timed region, and its own time is measured and subtracted."""
    import torch
    import torch.distributed as dist

    from lora_fine_tuning_mlp_b200 import _lib, api, replicas

    rank, local, world = replicas.world()
    if world > 1:
        torch.cuda.set_device(local)
        replicas.init("nccl", device=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())
    _lib.lib()
    inp = synth.make_linear_inputs(cfg)
    w = api.linear_weights_from_host(inp, cfg.alpha, dev)
    X = api.to_device_bf16(inp["X"], dev)
    dY = api.to_device_bf16(inp["dY"], dev)
    N = cfg.N
    Y = torch.empty((N, cfg.d_out), dtype=torch.bfloat16, device=dev)
    dX = torch.empty((N, cfg.d_in), dtype=torch.bfloat16, device=dev)
    dA, dB = torch.empty_like(w.A), torch.empty_like(w.B)
    wsf, wsb = api.Workspace(), api.Workspace()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    barrier = replicas.barrier

    def step(x=X, g=dY):
        _, saved = api.linear_forward(x, w, Y=Y, workspace=wsf)
        api.linear_backward(x, w, saved, g, dX=dX, dA=dA, dB=dB, workspace=wsb)

    def timed(fn, n):
        barrier()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        barrier()
        return replicas.max_over_ranks(a.elapsed_time(b), device=dev)

    def flushed_step():
        flush.fill_(1)
        step()

    for _ in range(args.warmup):
        flushed_step()
    torch.cuda.synchronize()
    sampler = ClockSampler(dev.index)
    sampler.start()
    time.sleep(0.3)
    launches0 = _lib.launch_count()
    w0 = time.monotonic()
    ms_total = timed(flushed_step, args.steps)
    w1 = time.monotonic()
    launches = _lib.launch_count() - launches0
    clocks = sampler.stop((w0, w1))
    ms_flush = timed(lambda: flush.fill_(1), args.steps)
    ms_max = max(ms_total - ms_flush, 1e-6)

    _lib.timing_enable(True)
    _lib.timing_collect()
    timed(flushed_step, args.steps)
    recs = _lib.timing_collect()
    _lib.timing_enable(False)

    # end to end: pinned-host X and dY copied in, dA and dB copied out, every step
    Xh = torch.from_numpy(inp["X"].view("int16")).view(torch.bfloat16).pin_memory()
    dYh = torch.from_numpy(inp["dY"].view("int16")).view(torch.bfloat16).pin_memory()
    dAh = torch.empty(dA.shape, dtype=dA.dtype, pin_memory=True)
    dBh = torch.empty(dB.shape, dtype=dB.dtype, pin_memory=True)
    Xd, dYd = torch.empty_like(X), torch.empty_like(dY)

    def e2e_step():
        Xd.copy_(Xh, non_blocking=True)
        dYd.copy_(dYh, non_blocking=True)
        step(Xd, dYd)
        dAh.copy_(dA, non_blocking=True)
        dBh.copy_(dB, non_blocking=True)

    for _ in range(3):
        e2e_step()
    ems = timed(e2e_step, args.steps)
    h2d = (X.numel() + dY.numel()) * 2
    d2h = (dA.numel() + dB.numel()) * 2

    per = {}
    for name, kms in recs:
        s_ = per.setdefault(name, [0.0, 0])
        s_[0] += kms
        s_[1] += 1
    peaks = load_peaks()
    fl = linear_flops(cfg)
    dom = max(per.items(), key=lambda kv: kv[1][0])[0] if per else None
    roof = None
    if dom in fl:
        avg_ms = per[dom][0] / per[dom][1]
        achieved = fl[dom] / (avg_ms * 1e-3) / 1e12
        peak = peaks["bf16_tflops"]
        roof = {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": ncu_traffic(cfg.name, dom),
                "peak_source": f"{peaks['source']} bf16_tflops (burst: short steps between L2 flushes)",
                "flops_per_launch": fl[dom], "avg_launch_ms": avg_ms}
    barrier()
    if rank == 0:
        tflops = world * cfg.flops() * args.steps / (ms_max * 1e-3) / 1e12
        line = {
            "metric": LINEAR_METRIC, "value": replicas.job_throughput(N, args.steps, ms_max, world),
            "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_max / args.steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic", "config": linear_config_dict(cfg), "tflops": tflops,
            "frac_of_peak": {"measured_burst": tflops / world / peaks["bf16_tflops"]},
            "roofline": roof,
            "e2e": {"value": replicas.job_throughput(N, args.steps, ems, world), "unit": "tokens/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "what": "per step: H2D of X and dY from pinned host, forward+backward, D2H of dA and dB "
                            "(no L2 flush)"},
            "gpu_launches": launches,
            "clocks": {"sm_mhz": clocks["sm_mhz"], "sm_max_mhz": clocks["sm_max_mhz"],
                       "reasons": clocks["reasons"], "samples": clocks["samples"]},
            "kernels_ms_per_step": {k: v[0] / args.steps for k, v in sorted(per.items(), key=lambda kv: -kv[1][0])},
            "flush_ms_per_step": ms_flush / args.steps,
        }
        if world == 1 and not args.no_cpu_baseline:
            n, run = time_linear_oracle(cfg, args.cpu_budget, inp)
            dt = run(np.arange(n))
            line["cpu_baseline"] = {"value": n / dt, "unit": "tokens/s", "cores": threads_used(), "kind": "oracle",
                                    "sample": f"{n} tokens of the {cfg.name} shapes, numpy fp64 oracle, {dt:.1f} s"}
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.cuda.synchronize()
        dist.destroy_process_group()
    return 0


# ----------------------------------------------------------------------------- cross-entropy legs


def ce_config_dict(cfg):
    return {"workload": cfg.name, "N_tokens": cfg.N, "V": cfg.V, "logit_scale": cfg.logit_scale,
            "softcap": cfg.softcap, "ignore_index": synth.CE_IGNORE_INDEX, "ignore_frac": cfg.ignore_frac,
            "l2": "no flush: logits %.1f GB > 126 MB L2" % (2 * cfg.N * cfg.V / 1e9), "parallelism": "replicas"}


def time_ce_oracle(cfg, budget_s: float, inp):
    """Rows of the workload the fp64 oracle handles in about budget_s (forward
    + backward).  Returns (rows, run(idx) -> seconds)."""
    from oracle import cross_entropy as oce

    def run(idx):
        t0 = time.perf_counter()
        z = oce.bf16_to_f64(inp["logits"][idx])
        lab = inp["labels"][idx]
        _, lse = oce.forward(z, lab, cfg.logit_scale, cfg.softcap, synth.CE_IGNORE_INDEX)
        oce.backward(z, lab, lse, inp["dloss"][idx], cfg.logit_scale, cfg.softcap, synth.CE_IGNORE_INDEX)
        return time.perf_counter() - t0

    t_probe = run(np.arange(2))
    n = max(2, min(cfg.N, int(2 * budget_s / max(t_probe, 1e-3))))
    return n, run


def ce_reference_arm(args, cfg):
    if int(os.environ.get("RANK", "0")) != 0:
        return 0
    inp = synth.make_ce_inputs(cfg)
    per_step = max(1.0, min(10.0, 150.0 / max(1, args.steps + args.warmup)))
    n, run = time_ce_oracle(cfg, per_step, inp)
    times = []
    for i in range(args.warmup + args.steps):
        dt = run((np.arange(n) + i * n) % cfg.N)
        if i >= args.warmup:
            times.append(dt)
    total = sum(times)
    value = n * len(times) / total
    line = {
        "impl": "reference", "metric": CE_METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * total / len(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": ce_config_dict(cfg),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads_used(), "kind": "oracle",
                         "sample": f"{n} rows of the {cfg.name} logits per step (numpy fp64 oracle)"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def ce_arm(args, cfg):
    """One step = cross-entropy forward (chunk partials + row combine) and
    backward over N rows of V logits, the gradient written to its own buffer
    so that every step sees the same logits.  The logits (2 GB on the 256K
    workloads) are far larger than L2."""
    import torch
    import torch.distributed as dist

    from lora_fine_tuning_mlp_b200 import _lib, api, replicas

    rank, local, world = replicas.world()
    if world > 1:
        torch.cuda.set_device(local)
        replicas.init("nccl", device=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())
    _lib.lib()
    inp = synth.make_ce_inputs(cfg)
    N, V = cfg.N, cfg.V
    ld = (V + 7) // 8 * 8
    host = torch.zeros((N, ld), dtype=torch.int16)
    host[:, :V] = torch.from_numpy(inp["logits"].view(np.int16))
    zfull = host.view(torch.bfloat16).to(dev)
    z = zfull[:, :V]
    lab = torch.from_numpy(inp["labels"]).to(dev)
    dl = torch.from_numpy(inp["dloss"]).to(dev)
    dz = torch.empty_strided(z.size(), z.stride(), dtype=torch.bfloat16, device=dev)
    ws = api.Workspace()
    kw = dict(logit_scale=cfg.logit_scale, softcap=cfg.softcap, ignore_index=synth.CE_IGNORE_INDEX)
    stream = torch.cuda.current_stream()
    barrier = replicas.barrier

    def step(x=z):
        _, lse = api.ce_forward(x, lab, workspace=ws, **kw)
        api.ce_backward(x, lab, lse, dl, out=dz, **kw)

    def timed(fn, n):
        barrier()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        barrier()
        return replicas.max_over_ranks(a.elapsed_time(b), device=dev)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    sampler = ClockSampler(dev.index)
    sampler.start()
    time.sleep(0.3)
    launches0 = _lib.launch_count()
    w0 = time.monotonic()
    ms_max = timed(step, args.steps)
    w1 = time.monotonic()
    launches = _lib.launch_count() - launches0
    clocks = sampler.stop((w0, w1))

    _lib.timing_enable(True)
    _lib.timing_collect()
    timed(step, args.steps)
    recs = _lib.timing_collect()
    _lib.timing_enable(False)

    # end to end through the public API: the logits copied in from pinned host
    # memory and the per-row losses copied back, every step
    zh = host.view(torch.bfloat16).pin_memory()
    lossh = torch.empty((N,), dtype=torch.float32, pin_memory=True)
    zd = torch.empty_like(zfull)

    def e2e_step():
        zd.copy_(zh, non_blocking=True)
        loss, lse = api.ce_forward(zd[:, :V], lab, workspace=ws, **kw)
        api.ce_backward(zd[:, :V], lab, lse, dl, out=dz, **kw)
        lossh.copy_(loss, non_blocking=True)

    e2e_steps = max(3, min(args.steps, 20))
    for _ in range(2):
        e2e_step()
    ems = timed(e2e_step, e2e_steps)

    per = {}
    for name, kms in recs:
        s_ = per.setdefault(name, [0.0, 0])
        s_[0] += kms
        s_[1] += 1
    peaks = load_peaks()
    algo = {"CE_fwd_chunks": cfg.bytes_fwd(), "CE_bwd": cfg.bytes_bwd()}
    dom = max((k for k in per if k in algo), key=lambda k: per[k][0], default=None)
    roof = None
    if dom is not None:
        avg_ms = per[dom][0] / per[dom][1]
        achieved = algo[dom] / (avg_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "traffic": None,
                "peak_source": f"{peaks['source']} hbm_gbs (copy bandwidth)",
                "bytes_per_launch": algo[dom], "avg_launch_ms": avg_ms}
    barrier()
    if rank == 0:
        per_step = ms_max / args.steps
        line = {
            "metric": CE_METRIC, "value": replicas.job_throughput(N, args.steps, ms_max, world), "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": ce_config_dict(cfg),
            "gb_per_s": (cfg.bytes_fwd() + cfg.bytes_bwd()) / (per_step * 1e-3) / 1e9,
            "roofline": roof,
            "kernels_gb_per_s": {k: algo[k] / (v[0] / v[1] * 1e-3) / 1e9 for k, v in per.items() if k in algo},
            "e2e": {"value": replicas.job_throughput(N, e2e_steps, ems, world), "unit": "tokens/s",
                    "h2d_bytes_per_step": int(zfull.numel() * 2), "d2h_bytes_per_step": int(N * 4),
                    "what": "per step: H2D of the logits from pinned host, forward + backward, D2H of the per-row "
                            "losses"},
            "gpu_launches": launches,
            "clocks": {"sm_mhz": clocks["sm_mhz"], "sm_max_mhz": clocks["sm_max_mhz"],
                       "reasons": clocks["reasons"], "samples": clocks["samples"]},
            "kernels_ms_per_step": {k: v[0] / args.steps for k, v in sorted(per.items(), key=lambda kv: -kv[1][0])},
        }
        if world == 1 and not args.no_cpu_baseline:
            n, run = time_ce_oracle(cfg, args.cpu_budget, inp)
            dt = run(np.arange(n))
            line["cpu_baseline"] = {"value": n / dt, "unit": "tokens/s", "cores": threads_used(), "kind": "oracle",
                                    "sample": f"{n} rows of the {cfg.name} logits, numpy fp64 oracle, {dt:.1f} s"}
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.cuda.synchronize()
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="b200", choices=("b200", "reference"))
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    choices=sorted(synth.BY_NAME) + sorted(synth.LINEAR_BY_NAME) + sorted(synth.BLOCK_BY_NAME)
                    + sorted(synth.CE_BY_NAME))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.workload in synth.CE_BY_NAME:
        cfg = synth.CE_BY_NAME[args.workload]
        return ce_reference_arm(args, cfg) if args.impl == "reference" else ce_arm(args, cfg)
    if args.workload in synth.LINEAR_BY_NAME:
        cfg = synth.LINEAR_BY_NAME[args.workload]
        return linear_reference_arm(args, cfg) if args.impl == "reference" else linear_arm(args, cfg)
    block = args.workload in synth.BLOCK_BY_NAME
    cfg = synth.BLOCK_BY_NAME[args.workload] if block else synth.BY_NAME[args.workload]
    args.block = block
    if args.impl == "reference":
        return reference_arm(args, cfg)
    return b200_arm(args, cfg)


if __name__ == "__main__":
    sys.exit(main())
