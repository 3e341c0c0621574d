"""Benchmark of the LaCT fast-weight TTT layer forward on B200.

python bench.py [--gpus N] [--steps K] [--warmup W] [--workload IDX] [--impl ours|reference]

A step is one full layer forward (every chunk: apply, chunk gradient, rule,
renorm) over one batch of synthetic inputs already resident in HBM.  The
default workload is the 760M-shaped language-model layer at 32K context
(B=2, H=6, d=256, dh=512, chunk 2048, GD, bf16).  Inputs (q, k, v: 604 MB)
are larger than the 126 MB L2, so no flush is needed between steps.
With N > 1 (torchrun) every rank runs its own batch (independent problems,
no data-path collective: weak scaling); time is the max over ranks.

`--impl reference` times the fp64 CPU oracle on a bounded sample of the same
workload (one full-length (batch, head) sequence per step) on the host cores.
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

from lact_inputs import BF16, RULE_MUON, WORKLOADS, Workload, make_inputs  # noqa: E402

METRIC = "TTT-layer tokens/s (fwd) at 1 B200 and % of bf16 tensor-core peak"
UNIT = "tokens/s"
DEFAULT_WORKLOAD = 2


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p["hbm_gbs"], p["bf16_tflops"], p["bf16_tflops_sustained"], "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# ---------------------------------------------------------------- algorithmic work
def step_flops(w: Workload) -> float:
    """18 d dh FLOPs per key token per head (4 forward on k, 2 for W2^T v, 6 for
    the three gradients) + 6 d dh per query token (apply), plus Newton-Schulz."""
    per_head = 12.0 * w.d * w.dh * w.T + 6.0 * w.d * w.dh * w.Tq
    if w.rule == RULE_MUON:
        m, p = min(w.d, w.dh), max(w.d, w.dh)
        per_head += w.n_chunks * 3 * 5 * (4.0 * m * m * p + 2.0 * m ** 3)
    return per_head * w.B * w.H


def kernel_work(w: Workload):
    """Algorithmic work per kernel kind over one step: (bound, amount, unit).
    FLOPs count 2 per multiply-add; bytes count each tensor read or written once."""
    BH, d, dh, T, Tq = w.B * w.H, w.d, w.dh, w.T, w.Tq
    esz = 2 if w.dtype == BF16 else 4
    ns = 3 * 5 * w.n_chunks * BH if w.rule == RULE_MUON else 0   # NS matrix-iterations
    planes = 3 * BH * d * dh
    return {
        "fwd_query_umma": ("tensor", 4.0 * Tq * d * dh * BH, "FLOP"),
        "apply_out_umma": ("tensor", 2.0 * Tq * d * dh * BH, "FLOP"),
        "apply_fused_umma": ("tensor", 6.0 * Tq * d * dh * BH, "FLOP"),
        "fwd_key_umma": ("tensor", 6.0 * T * d * dh * BH, "FLOP"),
        "grad_umma": ("tensor", 6.0 * T * d * dh * BH, "FLOP"),
        "key_grad_umma": ("tensor", 12.0 * T * d * dh * BH, "FLOP"),
        "ns_gram_umma": ("tensor", 2.0 * d * d * dh * ns, "FLOP"),
        "ns_poly_umma": ("tensor", 2.0 * d ** 3 * ns, "FLOP"),
        "ns_update_umma": ("tensor", 2.0 * dh * d * d * ns, "FLOP"),
        "qk_prologue": ("hbm", 2.0 * (Tq + T) * d * esz * BH, "B"),
        "rule_renorm": ("hbm", w.n_chunks * planes * (4 + 4 + 4 + 2), "B"),
    }


# ---------------------------------------------------------------- clocks
_REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")


def _summary(sm, mx, reasons, source, power=None):
    if not sm:
        return None
    out = {"sm_mhz": statistics.median(sm), "sm_min_mhz": min(sm), "sm_max_mhz": max(mx),
           "reasons": sorted(reasons), "samples": len(sm), "source": source}
    if power:
        out["power_w_median"] = round(statistics.median(power), 1)
    return out


class NvmlClockSampler:
    """Reads the SM clock, the power draw and the clock-event reasons of this
    rank's GPU every `period_s` seconds on a background thread (NVML; reads
    only, changes no setting).  Found by PCI bus id, so a restricted
    CUDA_VISIBLE_DEVICES does not mislead it."""

    def __init__(self, device: int, period_s: float = 0.002):
        import threading
        import pynvml
        self.nv = pynvml
        pynvml.nvmlInit()
        pr = torch.cuda.get_device_properties(device)
        bus = f"{pr.pci_domain_id:08X}:{pr.pci_bus_id:02X}:{pr.pci_device_id:02X}.0"
        self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        self.mx = float(pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM))
        self.bits = {
            "hw_slowdown": pynvml.nvmlClocksEventReasonHwSlowdown,
            "hw_thermal_slowdown": pynvml.nvmlClocksEventReasonHwThermalSlowdown,
            "sw_thermal_slowdown": pynvml.nvmlClocksEventReasonSwThermalSlowdown,
            "sw_power_cap": pynvml.nvmlClocksEventReasonSwPowerCap,
        }
        self.sm, self.power, self.reasons = [], [], set()
        self.period = period_s
        self.stop_flag = threading.Event()
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()

    def _run(self):
        nv = self.nv
        while not self.stop_flag.is_set():
            try:
                self.sm.append(float(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)))
                self.power.append(nv.nvmlDeviceGetPowerUsage(self.h) / 1000.0)
                mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.reasons.update(n for n, b in self.bits.items() if mask & b)
            except Exception:
                pass
            self.stop_flag.wait(self.period)

    def stop(self):
        self.stop_flag.set()
        self.thread.join(timeout=5)
        try:
            self.nv.nvmlShutdown()
        except Exception:
            pass
        return _summary(self.sm, [self.mx], self.reasons, "nvml", self.power)


class SmiClockSampler:
    """nvidia-smi fallback (200 ms period) where NVML is not available."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            time.sleep(0.3)                     # its first row before the timed region
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = [r.split(",") for r in out.strip().splitlines() if r.strip()]
        sm, mx, reasons = [], [], set()
        for r in rows:
            try:
                sm.append(float(r[0]))
                mx.append(float(r[1]))
            except (ValueError, IndexError):
                continue
            for name, val in zip(_REASONS, r[4:8]):
                if val.strip().lower() == "active":
                    reasons.add(name)
        return _summary(sm, mx, reasons, "nvidia-smi")


def ClockSampler(device: int):
    try:
        return NvmlClockSampler(device)
    except Exception:
        return SmiClockSampler(device)



# ---------------------------------------------------------------- forward timing
def forward_timing(ct, w: Workload, dev, steps: int, warmup: int, seed: int, barrier, barrier_max, local: int):
    """Times `steps` layer forwards of workload `w` on inputs resident in HBM,
    then the same steps again under the library's launch profiler.  Returns
    the inputs, both pass times (max over ranks), the per-kernel profile and
    the clock record of the first pass."""
    inp_cpu = make_inputs(w, seed=seed)
    inp = {k: (None if v is None else v.to(dev)) for k, v in inp_cpu.items()}
    B, H = w.B, w.H
    out = torch.empty_like(inp["q"])
    w_out = (torch.empty((B * H, w.dh, w.d), device=dev), torch.empty((B * H, w.d, w.dh), device=dev),
             torch.empty((B * H, w.dh, w.d), device=dev))
    ws = torch.empty(ct.workspace_bytes(inp["q"], inp["k"], inp["w1"], w.chunk, w.order, w.rule),
                     device=dev, dtype=torch.uint8)
    stream = torch.cuda.current_stream(dev)

    def step():
        ct.ttt_fwd(inp["q"], inp["k"], inp["v"], inp["lr"], inp["beta"], inp["w1"], inp["w2"],
                   inp["w3"], w.chunk, w.order, w.rule, out=out, w_out=w_out, workspace=ws,
                   stream=stream)

    for _ in range(warmup):
        step()
    if ct.status(stream) != ct.LACT_OK:
        raise SystemExit("device status not OK after warm-up")

    # ---- timed region (device time, CUDA events on the launching stream).
    # The K steps run exactly as a caller runs them: no events between the
    # kernels, whose launches overlap (programmatic dependent launch).
    clocks = ClockSampler(local)
    barrier()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    clk = clocks.stop()
    ms_total = barrier_max(e0.elapsed_time(e1))
    if ct.status(stream) != ct.LACT_OK:
        raise SystemExit("device status not OK after the timed region")

    # ---- per-kernel pass: the same K steps again with a CUDA event pair around
    # every launch (the library's launch profiler).  The profiler runs every
    # launch alone on the caller's stream (no side-stream apply, no overlap of
    # consecutive launches), so this pass gives each kernel's own duration
    # (kernel shares, roofline) but not the headline time.
    ct.profile_enable(True)
    barrier()
    torch.cuda.synchronize(dev)
    p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    p0.record(stream)
    for _ in range(steps):
        step()
    p1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    ct.profile_enable(False)
    ms_profiled = barrier_max(p0.elapsed_time(p1))
    prof = ct.profile_read()
    if ct.status(stream) != ct.LACT_OK:
        raise SystemExit("device status not OK after the per-kernel pass")
    return {"inp_cpu": inp_cpu, "inp": inp, "w_out": w_out, "stream": stream, "ms_total": ms_total,
            "ms_profiled": ms_profiled, "prof": prof, "clocks": clk}


def roofline_entry(prof: dict, w: Workload, steps: int):
    """Roofline of the kernel with the largest summed duration in the
    per-kernel pass.  Every launch there runs alone, so a tensor-core kernel
    is measured against the burst bf16 peak; the sustained fraction is given
    beside it."""
    hbm, pk_burst, pk_sust, pk_src = peaks()
    work = kernel_work(w)
    name, (n_launch, ms_kind) = max(prof.items(), key=lambda kv: kv[1][1])
    if name not in work:
        return None
    bound, amount, _ = work[name]
    per_launch = amount * steps / n_launch
    dur_s = ms_kind / n_launch / 1e3
    if bound == "tensor":
        achieved = per_launch / dur_s / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": pk_burst, "unit": "TFLOP/s",
                "frac": achieved / pk_burst, "frac_of_sustained": achieved / pk_sust,
                "peak_source": f"{pk_src} burst bf16 (the kernel is timed alone)"}
    else:
        achieved = per_launch / dur_s / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                "frac": achieved / hbm, "peak_source": f"{pk_src} copy bandwidth"}
    roof.update({"kernel": name, "launches": n_launch, "avg_launch_us": 1e3 * ms_kind / n_launch,
                 "work_per_launch": per_launch, "timed": "alone (per-kernel pass)",
                 "traffic": traffic_for(name, w)})
    return roof


def config_entry(ct, idx: int, steps: int, warmup: int, dev, local: int) -> dict:
    """One line of the `configs` record: another workload of the same layer
    timed the same way on this GPU (inputs resident in HBM, larger than L2)."""
    w = WORKLOADS[idx]
    t = forward_timing(ct, w, dev, steps, warmup, 0, lambda: None, lambda x: x, local)
    _, pk_burst, pk_sust, _ = peaks()
    ms_step = t["ms_total"] / steps
    tflops = step_flops(w) / (ms_step / 1e3) / 1e12
    prof = t["prof"]
    total = sum(x[1] for x in prof.values())
    return {"workload": w.name, "steps": steps, "warmup": warmup, "ms_per_step": ms_step,
            "tokens_per_s": w.tokens / (ms_step / 1e3), "algorithmic_tflops": tflops,
            "frac_of_burst": tflops / pk_burst, "frac_of_sustained": tflops / pk_sust,
            "roofline": roofline_entry(prof, w, steps),
            "kernel_shares": {k: round(v[1] / total, 4) for k, v in sorted(prof.items(), key=lambda kv: -kv[1][1])},
            "clocks": t["clocks"]}

# ---------------------------------------------------------------- CPU oracle
def oracle_sample(w: Workload, inp: dict, budget_s: float, max_heads: int):
    """Runs the oracle on whole (batch, head) sequences until `budget_s`
    seconds have passed (at least one).  Returns (tokens, seconds, heads)."""
    import oracle
    heads = [(b, h) for b in range(w.B) for h in range(w.H)][:max_heads]
    tokens, t0, done = 0, time.perf_counter(), 0
    for b, h in heads:
        oracle.ttt_layer(inp["q"], inp["k"], inp["v"], inp["lr"], inp["beta"], inp["w1"],
                         inp["w2"], inp["w3"], w.chunk, w.order, w.rule, heads=[(b, h)])
        tokens += w.tokens // (w.B * w.H)
        done += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    return tokens, time.perf_counter() - t0, done


def blas_threads():
    import oracle
    return oracle.blas_threads()


# ---------------------------------------------------------------- helpers
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(x: float, device) -> float:
    """The maximum of x over all ranks (x itself on one rank); `device` is
    where the reduction tensor lives (cuda for NCCL, cpu for gloo)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(world: int, tokens_per_rank_step: int, steps: int, ms_max: float) -> float:
    """Whole-job throughput (tokens/s): every rank processes its own batch of
    tokens_per_rank_step per step; the job takes the slowest rank's time."""
    return world * tokens_per_rank_step * steps / (ms_max / 1e3)


def workload_config(w: Workload, n_gpus: int) -> dict:
    in_bytes = (w.B * w.H * (w.Tq + 2 * w.T) * w.d) * (2 if w.dtype == BF16 else 4)
    return {"workload": w.name, "B": w.B, "H": w.H, "T": w.T, "Tq": w.Tq, "d": w.d, "dh": w.dh,
            "chunk": w.chunk, "order": ["apply_then_update", "update_then_apply"][w.order],
            "rule": ["gd", "momentum", "muon"][w.rule], "tokens_per_step_per_gpu": w.tokens,
            "parallelism": f"replicas{n_gpus}" if n_gpus > 1 else "single",
            "l2": f"inputs larger than L2 ({in_bytes / 1e6:.0f} MB > 126 MB), no flush"}


def run_reference(args, w: Workload):
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    inp = make_inputs(w, seed=0)
    cores = blas_threads()
    per_step = []
    for i in range(args.warmup + args.steps):
        tok, sec, _ = oracle_sample(w, inp, budget_s=0.0, max_heads=1)
        if i >= args.warmup:
            per_step.append((tok, sec))
    tokens = sum(t for t, _ in per_step)
    secs = sum(s for _, s in per_step)
    value = tokens / secs
    sample = f"one (batch, head) sequence of {w.T} key tokens per step (of {w.B * w.H})"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * secs / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w, world),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", type=int, default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=15.0,
                    help="seconds of oracle work for the cpu_baseline sample")
    ap.add_argument("--pass", dest="which", default="fwd", choices=["fwd", "bwd", "swa"],
                    help="time the layer forward (default), its backward (lact_ttt_bwd) or the "
                         "block's sliding-window attention (lact_swa_fwd, window = the chunk)")
    ap.add_argument("--extra-steps", type=int, default=20,
                    help="timed steps of each other bf16 workload in the `configs` record "
                         "(1 GPU; 0 skips them)")
    ap.add_argument("--tokens", type=int, default=0,
                    help="run the workload at this sequence length instead (a scaled case "
                         "for profiling; named in config.workload)")
    args = ap.parse_args()
    w = WORKLOADS[args.workload]
    if args.tokens:
        T = args.tokens
        single = w.Tq != w.T
        w = w.scaled(name=f"{w.name}@T{T}", T=T, Tq=w.Tq if single else T,
                     chunk=T if single else min(w.chunk, T))
    if args.impl == "reference":
        return run_reference(args, w)
    if args.which == "bwd":
        return run_backward(args, w)
    if args.which == "swa":
        return run_swa(args, w)

    import chunk_test_b200 as ct

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    def barrier_max(x: float) -> float:
        return max_over_ranks(x, dev)

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    t = forward_timing(ct, w, dev, args.steps, args.warmup, rank, barrier, barrier_max, local)
    inp_cpu, ms_total, ms_profiled, prof, clk = t["inp_cpu"], t["ms_total"], t["ms_profiled"], t["prof"], t["clocks"]
    stream, w_out = t["stream"], t["w_out"]

    ms_step = ms_total / args.steps
    tok_step = w.tokens
    value = job_value(world, tok_step, args.steps, ms_total)
    hbm, pk_burst, pk_sust, pk_src = peaks()
    flops = step_flops(w)
    launches_per_step = ct.launch_count(t["inp"]["q"], t["inp"]["k"], t["inp"]["w1"], w.chunk, w.order, w.rule)
    roof = roofline_entry(prof, w, args.steps)
    kernels = {k: {"launches": v[0], "ms": round(v[1], 4),
                   "share": round(v[1] / sum(x[1] for x in prof.values()), 4)}
               for k, v in sorted(prof.items(), key=lambda kv: -kv[1][1])}
    del t

    # ---- end to end: host buffers in, results back, through the C ABI
    pin = {k: (None if v is None else v.pin_memory()) for k, v in inp_cpu.items()}
    hout = torch.empty_like(inp_cpu["q"]).pin_memory()
    hwo = tuple(torch.empty(t.shape, dtype=torch.float32).pin_memory() for t in w_out)
    hws = torch.empty(ct.host_workspace_bytes(pin["q"], pin["k"], pin["w1"], w.chunk, w.order,
                                              w.rule), device=dev, dtype=torch.uint8)

    def host_step():
        ct.ttt_fwd_host(pin["q"], pin["k"], pin["v"], pin["lr"], pin["beta"], pin["w1"], pin["w2"],
                        pin["w3"], w.chunk, w.order, w.rule, out=hout, w_out=hwo, workspace=hws,
                        stream=stream)

    for _ in range(args.warmup):
        host_step()
    barrier()
    torch.cuda.synchronize(dev)
    h0, h1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    h0.record(stream)
    for _ in range(args.steps):
        host_step()
    h1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    e2e_ms = barrier_max(h0.elapsed_time(h1))
    h2d = sum(t.numel() * t.element_size() for t in pin.values() if t is not None)
    d2h = hout.numel() * hout.element_size() + sum(t.numel() * 4 for t in hwo)

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if w.dtype == BF16 else "f32",
        "data": "synthetic (seeded normal q/k/v, softplus lr, random-init fast weights)",
        "config": workload_config(w, world),
        "tensor_peak_frac": {"algorithmic_tflops": flops / (ms_step / 1e3) / 1e12,
                             "frac_of_burst": flops / (ms_step / 1e3) / 1e12 / pk_burst,
                             "frac_of_sustained": flops / (ms_step / 1e3) / 1e12 / pk_sust,
                             "peak_source": pk_src},
        "roofline": roof,
        "kernels": kernels,
        "kernel_pass": {"ms_per_step": ms_profiled / args.steps,
                        "method": "the same K steps again, every launch alone on one stream "
                                  "with a CUDA event pair around it (kernel shares, roofline "
                                  "durations); this stops the side-stream apply and the overlap "
                                  "of consecutive launches, so the headline time is the first "
                                  "pass, without them"},
        "gpu_launches": launches_per_step * args.steps,
        "e2e": {"value": job_value(world, tok_step, args.steps, e2e_ms), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "clocks": clk,
    }
    if world == 1 and not args.tokens and args.extra_steps > 0:
        # the other bf16 workloads, timed the same way (1 GPU only)
        line["configs"] = [config_entry(ct, i, args.extra_steps, args.warmup, dev, local)
                           for i in (2, 3, 4, 5) if i != args.workload]
    if world == 1 and rank == 0:
        tok, sec, nh = oracle_sample(w, inp_cpu, args.cpu_budget, max_heads=w.B * w.H)
        line["cpu_baseline"] = {"value": tok / sec, "unit": UNIT, "cores": blas_threads(),
                                "kind": "oracle",
                                "sample": f"{nh} of {w.B * w.H} (batch, head) sequences, "
                                          f"{tok} tokens, {sec:.1f} s"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


# ---------------------------------------------------------------- backward
# fp32 FFMA peak of a B200: 148 SMs x 128 FP32 lanes x 2 FLOP x 1965 MHz.
FP32_FMA_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def bwd_flops(w: Workload) -> dict:
    """Algorithmic FLOPs of lact_ttt_bwd by where they run.  "layer": per key
    token per head 12 d dh to recompute the forward's updates (keys' forward
    6, gradient 6) and 30 d dh in the reverse loop (keys' forward again 6,
    (p, q, r) 6, the weight gradients 6, dk 8, dv 4); per query token per head
    16 d dh for the apply's backward (its forward 6, the weight gradients 6,
    dq 4).  "ns" (Muon only, fp32 on the CUDA cores): per chunk and matrix,
    with m = max(d, dh), n = min(d, dh), two passes of the five Newton-Schulz
    steps (4 m n^2 + 2 n^3 each: the Gram, its square, the update) and one
    pass of their vector-Jacobian product (6 m n^2 + 4 n^3 each)."""
    layer = w.B * w.H * w.d * w.dh * (42.0 * w.T + 16.0 * w.Tq)
    ns = 0.0
    if w.rule == RULE_MUON:
        m, n = max(w.d, w.dh), min(w.d, w.dh)
        ns = w.B * w.H * 3 * w.n_chunks * 5 * (14.0 * m * n * n + 8.0 * n ** 3)
    return {"layer": layer, "ns": ns}


def bwd_on_tc(w: Workload) -> bool:
    """Whether lact_ttt_bwd runs the layer's contractions on the tensor cores:
    bf16 GD and momentum problems; Muon ones run in fp32 on the CUDA cores."""
    return w.dtype == BF16 and w.rule != RULE_MUON


def run_backward(args, w: Workload):
    import chunk_test_b200 as ct
    from lact_inputs import make_output_grads
    world, rank, local = dist_env()
    if world > 1:
        raise SystemExit("--pass bwd runs on one GPU")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    inp_cpu = make_inputs(w, seed=0)
    dout_cpu, _ = make_output_grads(w, seed=0)
    inp = {k: (None if v is None else v.to(dev)) for k, v in inp_cpu.items()}
    dout = dout_cpu.to(dev)
    ws = torch.empty(ct.bwd_workspace_bytes(inp["q"], inp["k"], inp["w1"], w.chunk, w.order, w.rule),
                     device=dev, dtype=torch.uint8)
    stream = torch.cuda.current_stream(dev)

    def step():
        return ct.ttt_bwd(inp["q"], inp["k"], inp["v"], inp["lr"], inp["beta"], inp["w1"], inp["w2"],
                          inp["w3"], w.chunk, w.order, w.rule, dout, workspace=ws, stream=stream)

    for _ in range(args.warmup):
        step()
    if ct.status(stream) != ct.LACT_OK:
        raise SystemExit("device status not OK after warm-up")
    clocks = ClockSampler(local)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    ms_step = e0.elapsed_time(e1) / args.steps
    if ct.status(stream) != ct.LACT_OK:
        raise SystemExit("device status not OK after the timed region")
    # per-kernel pass (launch profiler on)
    ct.profile_enable(True)
    ct.profile_read()
    for _ in range(args.steps):
        step()
    torch.cuda.synchronize(dev)
    prof = ct.profile_read()
    ct.profile_enable(False)
    launches_per_step = sum(v[0] for v in prof.values()) // args.steps
    dom_name, (n_launch, ms_kind) = max(prof.items(), key=lambda kv: kv[1][1])
    fl = bwd_flops(w)
    roof = None
    _, pk_burst, pk_sust, pk_src = peaks()
    if dom_name in ("simt_gemm_f32", "bwd_gemm_umma"):
        # the layer's contractions run in bwd_gemm_umma on bf16 GD / momentum
        # workloads and in simt_gemm_f32 otherwise (fp32, and every Muon
        # workload); the Newton-Schulz ones in simt_gemm_f32
        if dom_name == "bwd_gemm_umma":
            flops = fl["layer"]
        else:
            flops = fl["ns"] + (0.0 if bwd_on_tc(w) else fl["layer"])
        achieved = flops * args.steps / (ms_kind / 1e3) / 1e12
        tensor = dom_name == "bwd_gemm_umma"
        peak = pk_burst if tensor else FP32_FMA_TFLOPS
        roof = {"bound": "tensor" if tensor else "alu", "achieved": achieved, "peak": peak,
                "unit": "TFLOP/s", "frac": achieved / peak, "kernel": dom_name, "launches": n_launch,
                "avg_launch_us": 1e3 * ms_kind / n_launch, "timed": "alone (per-kernel pass)",
                "traffic": None,
                "peak_source": f"{pk_src} burst bf16 (the kernel is timed alone)" if tensor else
                               "derived: 148 SMs x 128 FP32 lanes x 2 FLOP x 1965 MHz"}
        if tensor:
            roof["frac_of_sustained"] = achieved / pk_sust
    kernels = {k: {"launches": v[0], "ms": round(v[1], 4),
                   "share": round(v[1] / sum(x[1] for x in prof.values()), 4)}
               for k, v in sorted(prof.items(), key=lambda kv: -kv[1][1])}
    # end to end: inputs from pinned host memory, gradients back to it
    pin = {k: (None if v is None else v.pin_memory()) for k, v in inp_cpu.items()}
    pdout = dout_cpu.pin_memory()
    grads0 = step()
    hgrad = {k: (None if v is None else torch.empty(v.shape, dtype=v.dtype).pin_memory())
             for k, v in grads0.items()}

    def host_step():
        for k, v in pin.items():
            if v is not None:
                inp[k].copy_(v, non_blocking=True)
        dout.copy_(pdout, non_blocking=True)
        g = step()
        for k, v in g.items():
            if v is not None:
                hgrad[k].copy_(v, non_blocking=True)

    for _ in range(args.warmup):
        host_step()
    torch.cuda.synchronize(dev)
    h0, h1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    h0.record(stream)
    for _ in range(args.steps):
        host_step()
    h1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = h0.elapsed_time(h1) / args.steps
    h2d = sum(t.numel() * t.element_size() for t in pin.values() if t is not None) + \
        pdout.numel() * pdout.element_size()
    d2h = sum(t.numel() * t.element_size() for t in hgrad.values() if t is not None)
    tok, total = w.tokens, fl["layer"] + fl["ns"]
    line = {
        "metric": "TTT-layer backward tokens/s at 1 B200", "value": tok / (ms_step / 1e3),
        "unit": "tokens/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if bwd_on_tc(w) else "f32",
        "data": "synthetic (seeded normal q/k/v/dout, softplus lr, random-init fast weights)",
        "config": dict(workload_config(w, 1), **{"pass": "backward (lact_ttt_bwd)"}),
        "peak_frac": {"algorithmic_tflops": total / (ms_step / 1e3) / 1e12,
                      "frac_of_burst_bf16": total / (ms_step / 1e3) / 1e12 / pk_burst,
                      "frac_of_sustained_bf16": total / (ms_step / 1e3) / 1e12 / pk_sust,
                      "frac_of_fp32_fma": total / (ms_step / 1e3) / 1e12 / FP32_FMA_TFLOPS},
        "roofline": roof,
        "kernels": kernels,
        "gpu_launches": launches_per_step * args.steps,
        "e2e": {"value": tok / (e2e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "clocks": clk,
    }
    # the autograd oracle on whole (batch, head) sequences, until the budget
    from oracle import lact_oracle_bwd as ob
    heads, t0, done = [(b, h) for b in range(w.B) for h in range(w.H)], time.perf_counter(), 0
    while done < len(heads) and (done == 0 or time.perf_counter() - t0 < args.cpu_budget):
        b, h = heads[done]
        sl = {k: (None if v is None else v[b:b + 1, h:h + 1]) for k, v in inp_cpu.items()
              if k in ("q", "k", "v", "lr", "beta")}
        ob.ttt_layer_bwd(sl["q"], sl["k"], sl["v"], sl["lr"], sl["beta"], inp_cpu["w1"][h:h + 1],
                         inp_cpu["w2"][h:h + 1], inp_cpu["w3"][h:h + 1], w.chunk, w.order, w.rule,
                         dout_cpu[b:b + 1, h:h + 1])
        done += 1
    sec = time.perf_counter() - t0
    tok_done = done * (w.T if w.Tq == w.T else w.T + w.Tq)
    line["cpu_baseline"] = {"value": tok_done / sec, "unit": "tokens/s", "cores": torch.get_num_threads(),
                            "kind": "oracle",
                            "sample": f"autograd backward oracle on {done} of {len(heads)} "
                                      f"(batch, head) sequences, {tok_done} tokens, {sec:.1f} s"}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- window attention
def swa_flops(B: int, H: int, T: int, d: int, window: int) -> float:
    """Algorithmic FLOPs of sliding-window attention: 4 d per (query, key)
    pair in the window (q'.k and p v), min(t + 1, window) keys for token t."""
    pairs = sum(min(t + 1, window) for t in range(min(T, window))) + max(0, T - window) * window
    return 4.0 * d * B * H * pairs


def run_swa(args, w: Workload):
    import chunk_test_b200 as ct
    from lact_inputs import make_swa_inputs
    world, rank, local = dist_env()
    if world > 1:
        raise SystemExit("--pass swa runs on one GPU")
    window = w.chunk if w.Tq == w.T else 2048
    B, H, T, d = w.B, w.H, w.T, w.d
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    inp_cpu = make_swa_inputs(B, H, T, d, seed=0)
    inp = {k: v.to(dev) for k, v in inp_cpu.items()}
    out = torch.empty_like(inp["q"])
    ws = torch.empty(ct.swa_workspace_bytes(inp["q"], window), device=dev, dtype=torch.uint8)
    stream = torch.cuda.current_stream(dev)

    def step():
        ct.swa_fwd(inp["q"], inp["k"], inp["v"], inp["q_scale"], inp["q_offset"], inp["k_scale"],
                   inp["k_offset"], window, out=out, workspace=ws, stream=stream)

    for _ in range(args.warmup):
        step()
    clocks = ClockSampler(local)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    ms_step = e0.elapsed_time(e1) / args.steps
    if ct.status(stream) != ct.LACT_OK:
        raise SystemExit("device status not OK after the timed region")
    ct.profile_enable(True)
    ct.profile_read()
    for _ in range(args.steps):
        step()
    torch.cuda.synchronize(dev)
    prof = ct.profile_read()
    ct.profile_enable(False)
    hbm, pk_burst, pk_sust, pk_src = peaks()
    flops = swa_flops(B, H, T, d, window)
    kernels = {k: {"launches": v[0], "ms": round(v[1], 4),
                   "share": round(v[1] / sum(x[1] for x in prof.values()), 4)}
               for k, v in sorted(prof.items(), key=lambda kv: -kv[1][1])}
    dom, (n_launch, ms_kind) = max(prof.items(), key=lambda kv: kv[1][1])
    roof = None
    if dom in ("swa_gemm_umma", "swa_flash_umma"):
        achieved = flops * args.steps / (ms_kind / 1e3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": pk_burst, "unit": "TFLOP/s",
                "frac": achieved / pk_burst, "frac_of_sustained": achieved / pk_sust, "kernel": dom,
                "launches": n_launch, "avg_launch_us": 1e3 * ms_kind / n_launch,
                "timed": "alone (per-kernel pass)", "traffic": traffic_for(dom, w),
                "peak_source": f"{pk_src} burst bf16 (the kernel is timed alone)",
                "work": "algorithmic: 4 d FLOPs per (query, key) pair in the window"}
    elif dom == "swa_elem":
        Lw = window + 128
        bytes_step = B * H * T * (Lw * (4 + 4 + 2) + 3 * d * 2 * 2)
        achieved = bytes_step * args.steps / (ms_kind / 1e3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                "kernel": dom, "launches": n_launch, "avg_launch_us": 1e3 * ms_kind / n_launch,
                "timed": "alone (per-kernel pass)", "traffic": None,
                "peak_source": f"{pk_src} copy bandwidth",
                "work": "scores read twice (fp32) and probabilities written (bf16), plus the prologue"}
    # end to end from pinned host buffers
    pin = {k: v.pin_memory() for k, v in inp_cpu.items()}
    hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()

    def host_step():
        for k, v in pin.items():
            inp[k].copy_(v, non_blocking=True)
        step()
        hout.copy_(out, non_blocking=True)

    for _ in range(args.warmup):
        host_step()
    torch.cuda.synchronize(dev)
    h0, h1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    h0.record(stream)
    for _ in range(args.steps):
        host_step()
    h1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = h0.elapsed_time(h1) / args.steps
    tok = B * T
    line = {
        "metric": "LaCT sliding-window attention tokens/s at 1 B200", "value": tok / (ms_step / 1e3),
        "unit": "tokens/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic (seeded normal q/k/v, near-identity q/k scales and offsets)",
        "config": {"workload": f"swa-B{B}-H{H}-T{T}-d{d}-w{window}", "B": B, "H": H, "T": T, "d": d,
                   "window": window, "pass": "sliding-window attention (lact_swa_fwd)",
                   "l2": "inputs and scores larger than L2, no flush"},
        "peak_frac": {"algorithmic_tflops": flops / (ms_step / 1e3) / 1e12,
                      "frac_of_burst_bf16": flops / (ms_step / 1e3) / 1e12 / pk_burst,
                      "frac_of_sustained_bf16": flops / (ms_step / 1e3) / 1e12 / pk_sust},
        "roofline": roof, "kernels": kernels,
        "gpu_launches": sum(v[0] for v in prof.values()),
        "e2e": {"value": tok / (e2e_ms / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in pin.values()),
                "d2h_bytes_per_step": hout.numel() * hout.element_size()},
        "clocks": clk,
    }
    # the oracle on a bounded sample: one head's first query rows
    from oracle import swa_oracle as so
    t0, n_rows = time.perf_counter(), 0
    start = min(window, T - 1)      # rows with full windows (the steady state)
    step_rows = 256
    while start + n_rows < T and (n_rows == 0 or time.perf_counter() - t0 < args.cpu_budget):
        rows = list(range(start + n_rows, min(T, start + n_rows + step_rows)))
        so.swa_layer(inp_cpu["q"][:1, :1], inp_cpu["k"][:1, :1], inp_cpu["v"][:1, :1], inp_cpu["q_scale"][:1],
                     inp_cpu["q_offset"][:1], inp_cpu["k_scale"][:1], inp_cpu["k_offset"][:1], window,
                     rows=rows)
        n_rows += len(rows)
    sec = time.perf_counter() - t0
    # per (batch, head) query rows per second -> tokens/s of the whole B x H problem
    line["cpu_baseline"] = {"value": n_rows / sec / H, "unit": "tokens/s", "cores": blas_threads(),
                            "kind": "oracle",
                            "sample": f"{n_rows} query rows (full windows) of one (batch, head), "
                                      f"{sec:.1f} s, scaled to {H} heads per token"}
    print(json.dumps(line), flush=True)
    return 0


# The source files each timed kernel is built from: a traffic record holds
# only while their hash is the one it was taken with.
KERNEL_SOURCES = {
    "apply_fused_umma": ("apply_kernel.cuh", "umma_kernels.cuh", "sm100.cuh"),
    "key_grad_umma": ("key_grad_kernel.cuh", "apply_kernel.cuh", "umma_kernels.cuh", "sm100.cuh"),
    "fwd_key_umma": ("umma_kernels.cuh", "sm100.cuh"),
    "grad_umma": ("pair_kernels.cuh", "umma_kernels.cuh", "sm100.cuh"),
    "rule_renorm": ("elem_kernels.cuh", "sm100.cuh"),
    "qk_prologue": ("elem_kernels.cuh", "sm100.cuh"),
    "swa_flash_umma": ("swa_flash.cuh", "umma_kernels.cuh", "sm100.cuh"),
}


def traffic_for(kernel: str, w: Workload):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, if it
    was taken on this workload with the current sources of that kernel; else
    None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except Exception:
        return None
    r = rec.get(f"{kernel}@{w.name}")
    if not r or kernel not in KERNEL_SOURCES or r.get("source_hash") != source_hash(kernel):
        return None
    return r.get("bytes_per_launch")


def source_hash(kernel: str) -> str:
    import hashlib
    h = hashlib.sha256()
    d = os.path.join(ROOT, "chunk_test_b200", "csrc")
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(d, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


if __name__ == "__main__":
    sys.exit(main())
