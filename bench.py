"""Throughput of the top-1 MoE gate: routed tokens/s for one full step
(route + forward + backward + aux loss + lambda update) and its fraction of the
TF32/HBM roofline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--math tf32|ffma]
                    [--workload NAME] [--impl native|reference]

One JSON line on rank 0. N > 1 runs under torchrun as N independent replicas
(one per GPU, each with its own batch: the gate has no cross-GPU exchange),
timed on the device as the maximum over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
if HERE not in sys.path:
    sys.path.insert(0, HERE)

from bwd_route_b200 import workloads as wl  # noqa: E402

METRIC = "routed tokens/s (fwd+bwd+aux) at 1 B200; % of TF32/HBM roofline"
UNIT = "tokens/s"
# nominal dense TF32 / BF16 tensor throughput ratio (1.1 vs 2.25 PFLOP/s)
TF32_OVER_BF16 = 1.1 / 2.25
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
CPU_SAMPLE_TOKENS = 8192
REF_STEP_TOKENS = 512


def load_peaks():
    p = os.path.join(HERE, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def algorithmic(spec, grad: str = "token"):
    """Bytes and flops the method itself must move / compute for one step.
    grad = "mean_collapse": the gate's output is averaged over the horizon axis,
    so the forward writes ctx_mean [B, H] instead of routed [T, H], and the
    output gradient arrives as [B, H] (the gradient of that mean)."""
    T, E, H, B = spec.T, spec.E, spec.H, spec.B
    step_flops = 6 * H * H * T
    if grad == "mean_collapse":
        g_bytes = B * H * 4
        # per token: x read twice, d_x written (3 H floats); logits read twice and
        # d_logits written (3 E floats); expert index and permutation traffic
        step_bytes = T * (4 * (3 * H + 3 * E) + 16) + 2 * g_bytes + 2 * E * H * H * 4
        per_kernel_bytes = {
            # x and the expert indices read, ctx_mean written; W and bias
            "fwd": T * (4 * H + 4) + g_bytes + E * H * H * 4 + E * H * 4,
            # the whole backward call: x read, d_x written, perm read, grad_ctx_mean
            # read once; W read, dW and db written
            "bwd": T * (8 * H + 4) + g_bytes + 2 * E * H * H * 4 + E * H * 4,
        }
        return step_bytes, step_flops, per_kernel_bytes
    step_bytes = T * (4 * (5 * H + 3 * E) + 16) + 2 * E * H * H * 4
    per_kernel_bytes = {
        # x read, routed written, perm read; W and bias
        "fwd": T * (8 * H + 4) + E * H * H * 4 + E * H * 4,
        # the whole backward call: x and d_out read once, d_x written, perm read;
        # W read, dW and db written
        "bwd": T * (12 * H + 4) + 2 * E * H * H * 4 + E * H * 4,
    }
    return step_bytes, step_flops, per_kernel_bytes


L2_BYTES = 126 * 1024 * 1024
# FP32 SIMT peak of the FFMA path: 148 SMs x 128 FP32 lanes x 2 flop x 1.965 GHz (nominal)
FP32_SIMT_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def l2_note(spec, collapse: bool, flushed: bool) -> str:
    T, H, E, B = spec.T, spec.H, spec.E, spec.B
    act = T * H * 4
    if act * 2 > L2_BYTES:
        if collapse:
            return ("inputs larger than L2 (x, d_x: 2 x %.2f GB; the [B, H] mean and its gradient, %.0f MB each, "
                    "stay in L2)%s" % (act / 1e9, B * H * 4 / 1e6,
                                       ", L2 also flushed between steps" if flushed else ", no flush"))
        return "inputs larger than L2 (x, d_out, routed, d_x: 4 x %.2f GB)%s" % (
            act / 1e9, ", L2 also flushed between steps" if flushed else ", no flush")
    total = 4 * act + T * E * 8 + 2 * E * H * H * 4
    if flushed:
        return "inputs (%.1f MB) fit in L2; 256 MB written between steps to flush it" % (total / 1e6)
    return "inputs (%.1f MB) fit in L2 and stay there (back-to-back steps)" % (total / 1e6)


def simt_roofline(step_flops: float, ms_per_step: float) -> dict:
    """The FFMA path against its own ceiling, FP32 on the CUDA cores."""
    achieved = step_flops / (ms_per_step * 1e-3) / 1e12
    return {"bound": "alu", "achieved": achieved, "peak": FP32_SIMT_TFLOPS, "unit": "TFLOP/s",
            "frac": achieved / FP32_SIMT_TFLOPS, "peak_source": "148 SMs x 128 FP32 lanes x 2 x 1.965 GHz"}


def host_cpu() -> dict:
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    model = ln.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    try:
        avail = len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        avail = os.cpu_count()
    return {"cpu_model": model, "cores_available": avail}


TRAFFIC_RECORD = os.path.join(HERE, "profiles", "traffic_mid_b16384_e8_h256.md")

# The library kernels each timed call launches, per (call, fused TF32 backward).
CALL_KERNELS = {
    ("fwd", True): ["grouped_tf32_kernel (hmean_fwd_tf32_sum_kernel with the horizon mean)"],
    ("fwd", False): ["grouped_ffma_kernel"],
    ("bwd", True): ["grouped_tf32_kernel (d_x)", "wgrad_tf32_kernel", "wgrad_reduce_kernel"],
    ("bwd", False): ["grouped_ffma_kernel (d_x)", "wgrad_ffma_kernel", "wgrad_reduce_kernel"],
    ("bwd", "single_pass_256"): ["bwd_fused_pair_kernel", "wgrad_reduce_kernel"],
    ("bwd", "single_pass_128"): ["bwd_fused_single_kernel", "wgrad_reduce_kernel"],
}


def code_sha1(paths) -> str:
    """sha1 of the code of the given source files with comments and blank space
    removed, so that a change to a comment does not count as a kernel change."""
    import hashlib
    import re
    h = hashlib.sha1()
    for path in paths:
        with open(path) as fh:
            text = fh.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        h.update(" ".join(text.split()).encode())
    return h.hexdigest()


def scale_traffic(measured: int, fixed: int, scale: float) -> int:
    """DRAM bytes of a full launch from a capture of a smaller one: the part that
    moves with the tokens grows by the token ratio, the part that does not (W, the
    partial-sum slots, bias) is taken as its algorithmic size at both sizes."""
    return int(round(fixed + (measured - fixed) * scale))


def bwd_passes(math_name: str, grad: str, H: int, T: int) -> int:
    """Contraction passes of the library's default TF32 backward: one fused pass for
    the horizon-mean gradient at H = 256 and at H = 128 above 65,536 tokens, two
    (d_x; dW and db) otherwise."""
    if math_name != "tf32":
        return 2
    return 1 if ((grad == "mean_collapse" and H == 256) or (H == 128 and T > 65536)) else 2


def recorded_traffic(call: str, workload: str, math_name: str, grad: str = "token", H: int = 256,
                     T: int = 1048576):
    """DRAM bytes (read + write) of one launch of `call`, from the committed ncu
    record (counters taken on a smaller case of the same shape and scaled to the
    workload), or None when there is no record for this workload, gradient mode
    and math mode, when the recorded backward ran another number of passes than
    the default path, or when the kernel code changed since the counters were taken."""
    try:
        text = open(TRAFFIC_RECORD).read()
        data = json.loads(text.split("```json", 1)[1].split("```", 1)[0])
        for rec in data["records"]:
            if rec["workload"] != workload or rec["math"] != math_name or rec["grad"] != grad:
                continue
            if code_sha1([os.path.join(HERE, f) for f in rec["source_files"]]) != rec["code_sha1"]:
                return None
            if call == "bwd" and rec.get("bwd_passes") != bwd_passes(math_name, grad, H, T):
                return None
            v = rec["traffic_bytes_per_call"].get(call)
            return int(v) if v is not None else None
    except (OSError, IndexError, KeyError, ValueError, TypeError):
        return None
    return None


class ClockSampler:
    """Samples SM clock and clock-event reasons with NVML while the timed region runs."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting",
               0x10: "sync_boost", 0x1: "gpu_idle"}

    def __init__(self, index: int, period: float = 0.001):
        self.index, self.period = index, period
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._thr = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nvml = None

    def _run(self):
        n = self.nvml
        while not self._stop.is_set():
            try:
                self.samples.append(n.nvmlDeviceGetClockInfo(self.h, n.NVML_CLOCK_SM))
                r = n.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit and bit != 0x1:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nvml is not None:
            # the launching thread holds the interpreter lock between its library
            # calls; a short switch interval lets the sampler wake on time
            self._switch = sys.getswitchinterval()
            sys.setswitchinterval(2e-4)
            self._thr = threading.Thread(target=self._run, daemon=True)
            self._thr.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._thr:
            self._thr.join()
            sys.setswitchinterval(self._switch)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def max_over_ranks(value: float, device) -> float:
    """The maximum of a per-rank time over all ranks (one all-reduce; a no-op for
    a single process). Used for every multi-GPU time: the job is as slow as its
    slowest replica."""
    import torch
    import torch.distributed as dist
    if not dist.is_initialized() or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, tokens_per_rank: int, ms_per_step: float) -> float:
    """Whole-job routed tokens/s: every replica routes its own batch per step."""
    return world * tokens_per_rank / (ms_per_step * 1e-3)


def cpu_oracle_tokens_per_s(inp, n_tokens: int):
    """The CPU oracle, as it stands, on the first n_tokens tokens of the workload."""
    import oracle
    sample = wl.token_sample(inp, n_tokens)
    t0 = time.perf_counter()
    oracle.step(sample)
    dt = time.perf_counter() - t0
    return sample.spec.T / dt, dt, sample.spec.T


def _oracle_shard(shard):
    """One worker of the all-cores CPU baseline: the oracle, unchanged, on one
    token shard; returns its dW and db (the sums the shards share)."""
    import oracle
    out = oracle.step(shard)
    return out["dW"], out["db"]


def _shard(inp, lo: int, hi: int):
    """Tokens lo .. hi - 1 of a workload as a workload of their own (only these
    rows travel to a worker process)."""
    spec = wl.dataclasses.replace(inp.spec, name=inp.spec.name + f"_{lo}_{hi}", B=hi - lo, N_H=1)
    return wl.dataclasses.replace(inp, spec=spec, gate_logits=inp.gate_logits[lo:hi], x=inp.x[lo:hi],
                                  d_out=inp.d_out[lo:hi])


def cpu_oracle_all_cores(inp, tokens_per_core: int, cores: int):
    """The oracle, as it stands, on `cores` token shards in `cores` processes
    (spawned, so no process inherits a CUDA context), with dW and db of the
    shards added in shard order. Returns (tokens/s, seconds, tokens)."""
    import multiprocessing as mp
    n = min(inp.spec.T, tokens_per_core * cores)
    shards = [_shard(inp, n * k // cores, n * (k + 1) // cores) for k in range(cores)]
    with mp.get_context("spawn").Pool(cores) as pool:
        pool.map(_oracle_shard, [_shard(inp, 0, 64)] * cores)  # start-up and the oracle's build
        t0 = time.perf_counter()
        parts = pool.map(_oracle_shard, shards, chunksize=1)
        dW, db = parts[0]
        for pw, pb in parts[1:]:
            dW = dW + pw
            db = db + pb
        dt = time.perf_counter() - t0
    return n / dt, dt, n


def run_reference(args, spec):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    inp = wl.generate(spec)
    sample_tokens = min(REF_STEP_TOKENS, spec.T)
    for _ in range(args.warmup):
        cpu_oracle_tokens_per_s(inp, sample_tokens)
    times = []
    for _ in range(args.steps):
        _, dt, n = cpu_oracle_tokens_per_s(inp, sample_tokens)
        times.append(dt)
    per_step = sum(times) / len(times)
    value = sample_tokens / per_step
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_step * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": spec.name, "B": spec.B, "N_H": spec.N_H, "E": spec.E, "H": spec.H,
                   "tokens": spec.T, "math": "fp64 oracle"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": f"first {sample_tokens} tokens of {spec.name} per step (route, forward, "
                                   f"d_x, dW/db, aux) in plain single-threaded C, fp64 accumulation", **host_cpu()},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--math", choices=["tf32", "ffma"], default="tf32")
    ap.add_argument("--workload", default=wl.THROUGHPUT_WORKLOAD, choices=sorted(wl.WORKLOADS))
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--grad", choices=["token", "mean_collapse"], default="token",
                    help="the gate's output per token [T, H] with its gradient (default), or averaged over "
                         "the horizon axis: the forward writes ctx_mean [B, H] and its gradient is [B, H]")
    ap.add_argument("--graph", action="store_true",
                    help="time K replays of one step captured in a CUDA graph (the per-call times then come "
                         "from a separate un-captured loop); for launch-bound small workloads")
    ap.add_argument("--flush-l2", action="store_true",
                    help="write a 256 MB buffer between timed steps (outside each step's events)")
    args = ap.parse_args()
    spec = wl.WORKLOADS[args.workload]
    if args.impl == "reference":
        run_reference(args, spec)
        return
    args.warmup = max(args.warmup, 3)

    import torch
    import torch.distributed as dist

    from bwd_route_b200 import ops
    from bwd_route_b200.gate import MoETop1Gate

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)

    math_mode = ops.MOE_MATH_TF32 if args.math == "tf32" else ops.MOE_MATH_FFMA
    inp = wl.generate(spec)
    T, E, H = spec.T, spec.E, spec.H
    logits = torch.from_numpy(inp.gate_logits).to(dev)
    x = torch.from_numpy(inp.x).to(dev)
    collapse = args.grad == "mean_collapse"
    # the gradient of the horizon mean: one row per batch row (a seeded draw of its own)
    g_host = (np.random.default_rng(spec.seed + 7).standard_normal((spec.B, spec.H), dtype=np.float32)
              if collapse else inp.d_out)
    d_out = torch.from_numpy(g_host).to(dev)
    W = torch.from_numpy(inp.W).to(dev)
    bias = torch.from_numpy(inp.bias).to(dev)
    gate = MoETop1Gate(W, bias, spec.B, spec.N_H, math_mode, inp.lambda_floor, inp.lambda_max_extra,
                       inp.ent_target, inp.ent_ema)
    if args.graph:
        # a CUDA graph is captured on a stream other than the default one: run everything there
        torch.cuda.set_stream(torch.cuda.Stream(dev))
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        # the calls of one training step, with an event between consecutive calls
        if ev:
            ev[0].record(stream)
        gate.route(logits)
        if ev:
            ev[1].record(stream)
        if collapse:
            gate.forward_mean_collapse(x)
        else:
            gate.forward(x)
        if ev:
            ev[2].record(stream)
        if collapse:
            gate.backward_mean_collapse(x, d_out)
        else:
            gate.backward(x, d_out)
        if ev:
            ev[3].record(stream)
        gate.aux_and_update_lambda(logits)
        if ev:
            ev[4].record(stream)

    def barrier():
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    for _ in range(args.warmup):
        step()
    flags = ops.moe_top1_device_flags(gate.ws)
    if flags:
        raise RuntimeError(f"device flags set during warm-up: {flags:#x}")

    # timed region: K whole steps, events on the launching stream
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if args.flush_l2 else None
    per_call = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    graph = None
    if args.graph:
        # one step through the same public calls, captured once
        torch.cuda.synchronize(dev)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            step()
        graph.replay()
        torch.cuda.synchronize(dev)
    barrier()
    with ClockSampler(local) as clocks:
        start.record(stream)
        for k in range(args.steps):
            if flush is not None:
                flush.fill_(k & 0xFF)
            if graph is not None:
                per_call[k][0].record(stream)
                graph.replay()
                per_call[k][4].record(stream)
            else:
                step(per_call[k])
        end.record(stream)
        barrier()
    step_ms = sorted(per_call[k][0].elapsed_time(per_call[k][4]) for k in range(args.steps))
    if flush is not None:  # the flushes sit between the steps' own events
        ms = sum(step_ms)
    else:
        ms = start.elapsed_time(end)
    ms = max_over_ranks(ms, dev)
    ms_per_step = ms / args.steps
    pct = lambda f: step_ms[min(len(step_ms) - 1, int(f * len(step_ms)))]  # noqa: E731
    names = ["route", "fwd", "bwd", "aux+lambda"]
    if graph is not None:
        # per-call times from a separate un-captured loop
        per_call = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(min(args.steps, 20))]
        for ev in per_call:
            step(ev)
        torch.cuda.synchronize(dev)
    call_ms = {n: sum(ev[i].elapsed_time(ev[i + 1]) for ev in per_call) / len(per_call)
               for i, n in enumerate(names)}
    flags = ops.moe_top1_device_flags(gate.ws)

    # end to end through the public API: inputs from pinned host memory, loss back to the host
    h_logits = torch.from_numpy(inp.gate_logits).pin_memory()
    h_x = torch.from_numpy(inp.x).pin_memory()
    h_dout = torch.from_numpy(g_host).pin_memory()
    h_loss = torch.empty(2, dtype=torch.float32).pin_memory()
    e2e_steps = max(1, min(args.e2e_steps, args.steps))
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        logits.copy_(h_logits, non_blocking=True)
        x.copy_(h_x, non_blocking=True)
        d_out.copy_(h_dout, non_blocking=True)
        if collapse:
            gate.route(logits)
            gate.forward_mean_collapse(x)
            gate.backward_mean_collapse(x, d_out)
            gate.aux_and_update_lambda(logits)
        else:
            gate.step(logits, x, d_out)
        h_loss.copy_(gate.loss, non_blocking=True)
    e1.record(stream)
    barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, dev)

    if rank == 0:
        peaks, peak_kind = load_peaks()
        step_bytes, step_flops, kbytes = algorithmic(spec, args.grad)
        hbm = float(peaks["hbm_gbs"])
        tf32_sus = float(peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])) * TF32_OVER_BF16
        t_roof = max(step_bytes / (hbm * 1e9), step_flops / (tf32_sus * 1e12))
        value = job_throughput(world, T, ms_per_step)
        dominant = max(["fwd", "bwd"], key=lambda n: call_ms[n])
        fused = math_mode == ops.MOE_MATH_TF32
        achieved = kbytes[dominant] / (call_ms[dominant] * 1e-3) / 1e9
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "tf32" if fused else "f32", "data": "synthetic",
            "config": {"workload": spec.name + ("+mean_collapse" if collapse else ""), "B": spec.B,
                       "N_H": spec.N_H, "E": E, "H": H, "tokens": T, "grad": args.grad,
                       "math": args.math, "parallelism": "replicas only" if world > 1 else "single GPU",
                       "l2": l2_note(spec, collapse, flush is not None)},
            "roofline": {"bound": "hbm", "kernel": dominant, "launches_in_call": CALL_KERNELS[
                             (dominant, f"single_pass_{H}") if (fused and dominant == "bwd" and
                                                                bwd_passes(args.math, args.grad, H, T) == 1)
                             else (dominant, fused)],
                         "achieved": achieved, "peak": hbm, "unit": "GB/s",
                         "frac": achieved / hbm,
                         "traffic": recorded_traffic(dominant, spec.name, args.math, args.grad, H, T),
                         "algorithmic_bytes": kbytes[dominant], "peak_source": f"{peak_kind} hbm_gbs"},
            "step_roofline": {"bytes": step_bytes, "flops": step_flops, "t_roofline_ms": t_roof * 1e3,
                              "frac": t_roof * 1e3 / ms_per_step,
                              "peaks": {"hbm_gbs": hbm, "tf32_tflops": tf32_sus,
                                        "source": f"{peak_kind}; tf32 = bf16_tflops_sustained x 1.1/2.25"}},
            "per_call_ms": call_ms,
            **({"simt_roofline": simt_roofline(step_flops, ms_per_step)} if math_mode == ops.MOE_MATH_FFMA else {}),
            "step_ms_percentiles": {"p10": pct(0.1), "p50": pct(0.5), "p90": pct(0.9)},
            "timing": ("CUDA graph of one step, replayed" if graph is not None else "stream launches")
                      + ("; 256 MB written between steps, outside their events" if flush is not None else ""),
            "e2e": {"value": job_throughput(world, T, e2e_ms), "unit": UNIT, "ms_per_step": e2e_ms, "steps": e2e_steps,
                    "h2d_bytes_per_step": (T * (E + H) + g_host.shape[0] * H) * 4, "d2h_bytes_per_step": 8},
            "gpu_launches": args.steps * MoETop1Gate.launches_per_step(math_mode, H, T, E, collapse),
            "clocks": clocks.summary(),
            "device_flags": flags,
        }
        if world == 1 and not args.no_cpu_baseline:
            v, dt, n = cpu_oracle_tokens_per_s(inp, CPU_SAMPLE_TOKENS)
            line["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": 1, "kind": "oracle",
                                    "sample": f"first {n} tokens of {spec.name}: route, forward, d_x, dW/db and "
                                              f"aux in plain single-threaded C (fp64 accumulation), {dt:.1f} s",
                                    **host_cpu()}
            cores = host_cpu()["cores_available"] or 1
            if cores > 1:
                v, dt, n = cpu_oracle_all_cores(inp, CPU_SAMPLE_TOKENS, cores)
                line["cpu_baseline_all_cores"] = {
                    "value": v, "unit": UNIT, "cores": cores, "kind": "oracle",
                    "sample": f"first {n} tokens of {spec.name} in {cores} equal shards, one process per core, "
                              f"each running the unchanged single-threaded oracle (route, forward, d_x, dW/db, aux "
                              f"of its shard); dW and db of the shards added in shard order; {dt:.1f} s",
                    **host_cpu()}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
