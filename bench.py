"""Benchmark of the routed, weight-quantized MoE expert layer on B200.

Headline (one JSON line on rank 0): the decode W4A16 layer (T=32 tokens, H=7168, I=2048,
E=384 experts, top-8, INT4 group-32 weights with bf16 scales), one step = one full layer forward
(route, align, gate/up + SiLU*up, down + routing weight, combine) through the C ABI.
  value  = weight bytes of the experts the step touches / device time per step (GB/s)
  e2e    = the same with the step's input copied from pinned host memory and its output read back
           inside the timed region
  roofline = the dominant kernel (gate/up) against the measured HBM copy bandwidth
The same line carries the prefill W4A16 layer (T=8192, Zipf-skewed routing), the block-FP8 MoE
layer (T=4096, E=256) and the dense block-FP8 matmul sweep as secondary measurements.

--impl reference times the CPU oracle (oracle/, the one other consumer allowed here) on a bounded
sample of the same workload, on the host cores. Multi-GPU (--gpus N under torchrun): independent
replicas, one per rank, no collective on the data path ("replicas only"); value is the sum over
ranks of bytes / the slowest rank's time. --parallel ep|tp instead splits the one decode layer
over the ranks (expert- or tensor-parallel shares, then an all-reduce of the output over NCCL);
value is then the layer's weight bytes / the slowest rank's time (strong scaling).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "MoE layer TFLOP/s + weight GB/s vs roofline (decode T=32, prefill T=8192)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------------------------

def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(v: float, world: int) -> float:
    """Max of a per-rank value over all ranks (timings: the slowest rank sets the job's time)."""
    if world == 1:
        return v
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_value(units_per_rank: float, ms_per_rank: float, world: int) -> tuple[float, float]:
    """Whole-job throughput of `world` independent replicas: all ranks' units over the slowest
    rank's time. Returns (units per second, slowest ms)."""
    ms = max_over_ranks(ms_per_rank, world)
    return world * units_per_rank / (ms * 1e-3), ms


# ---------------------------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "200", "-i", str(self.dev)], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in getattr(self, "lines", []):
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        loaded = [v for v in sm if mx is None or v >= 0.5 * mx] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------------------------
# timing helpers
# ---------------------------------------------------------------------------------------------

def timed_steps(fn, steps, warmup, flush=None, world=1):
    """Device time per step (ms): CUDA events around each step on the current stream, L2 flushed
    between steps outside the events; barrier + synchronize on both sides."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for a, b in evs:
        if flush is not None:
            flush()
        a.record()
        fn()
        b.record()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in evs]


def src_sha(*names):
    h = hashlib.sha256()
    for n in names:
        h.update(open(os.path.join(ROOT, "quantized_mixture_experts_align_b200", "csrc", n), "rb").read())
    return h.hexdigest()[:16]


def traffic_for(key, sha):
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p)).get(key)
    if not d or d.get("src_sha") != sha:
        return None
    return d.get("bytes_per_launch")


# ---------------------------------------------------------------------------------------------
# workloads
# ---------------------------------------------------------------------------------------------

def touched_experts(moeq, d):
    ids, _ = moeq.moe_route_topk(d["logits"], d["k"])
    return int(torch.unique(ids).numel())


def expert_rows(moeq, d):
    """Routed rows per expert of a workload (its own routing, read once on the host, untimed)."""
    ids, _ = moeq.moe_route_topk(d["logits"], d["k"])
    return torch.bincount(ids.flatten().long(), minlength=d["E"]).cpu().numpy()


def skew_roof_ms(rows, expert_bytes, H, I, gbs, tflops):
    """Skew-aware roof of a routed layer: every active expert costs the slower of streaming its
    weights at the HBM rate and its own rows' FLOPs at the tensor peak, summed over experts."""
    t = 0.0
    for c in rows:
        if c > 0:
            t = t + max(expert_bytes / (gbs * 1e9), W.moe_flops(int(c), 1, H, I) / (tflops * 1e12))
    return t * 1e3


def measure_fp8_peak():
    """Dense E4M3 tensor-core throughput of this GPU in this run (torch._scaled_mm, 8192^3, f32
    scales of 1): best of 10 single launches (burst) and the mean over ~2 s back to back
    (sustained). None when the library call is unavailable."""
    try:
        n = 8192
        a = torch.randn(n, n, device="cuda").to(torch.float8_e4m3fn)
        b = torch.randn(n, n, device="cuda").to(torch.float8_e4m3fn).t()
        one = torch.ones((), device="cuda")
        f = lambda: torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
        for _ in range(3):
            f()
        torch.cuda.synchronize()
        best = float("inf")
        for _ in range(10):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(); f(); e1.record(); torch.cuda.synchronize()
            best = min(best, e0.elapsed_time(e1))
        reps = max(10, int(2000.0 / best))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            f()
        e1.record(); torch.cuda.synchronize()
        mean = e0.elapsed_time(e1) / reps
        fl = 2.0 * n * n * n
        del a, b
        torch.cuda.empty_cache()
        return {"burst": fl / (best * 1e-3) / 1e12, "sustained": fl / (mean * 1e-3) / 1e12,
                "how": "torch._scaled_mm 8192^3 e4m3 -> bf16 in this run (best of 10 / ~2 s back to back)"}
    except Exception as exc:  # noqa: BLE001 - any failure means: use the nominal ratio
        return {"error": f"{type(exc).__name__}: {exc}"[:200]}


def launch_overhead_w4a16(moeq, d, steps, warmup):
    """Launch overhead of the decode layer: host time to enqueue one eager forward (the C ABI
    call with its five launches) and one CUDA-graph replay of the same forward, and the device
    time per step of back-to-back eager calls and graph replays (no L2 flush: launch gaps show)."""
    out = torch.empty((d["T"], d["H"]), dtype=torch.bfloat16, device="cuda")
    ws = moeq.workspace(moeq.moe_w4a16_workspace_size(d["T"], d["H"], d["I"], d["E"], d["k"]), "cuda")

    def step():
        moeq.moe_w4a16_forward(d["x"], d["logits"], d["k"], d["w13q"], d["w13s"], d["w2q"], d["w2s"], out=out, ws=ws)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for _ in range(warmup):
            step()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    torch.cuda.synchronize()

    def back_to_back(fn):
        fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0 = time.perf_counter()
        e0.record()
        for _ in range(steps):
            fn()
        e1.record()
        host_us = (time.perf_counter() - t0) / steps * 1e6
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / steps, host_us

    moeq.moe_host_stats(reset=True)
    eager_ms, eager_host = back_to_back(step)
    lib = moeq.moe_host_stats(reset=True)
    graph_ms, graph_host = back_to_back(g.replay)
    del g
    lib_us = lib["host_us"] / max(lib["calls"], 1)
    return {"eager_ms_per_step": eager_ms, "graph_ms_per_step": graph_ms, "eager_host_submit_us": eager_host,
            "eager_library_host_us": lib_us, "eager_binding_host_us": eager_host - lib_us,
            "graph_host_submit_us": graph_host, "steps": steps,
            "how": "back-to-back steps on one stream, no L2 flush; host time = enqueue time per step; library = "
                   "the C entry point's own wall time (moe_host_stats), binding = the rest (Python + ctypes)"}


def run_w4a16(moeq, d, steps, warmup, flush, world, trace=False):
    out = torch.empty((d["T"], d["H"]), dtype=torch.bfloat16, device="cuda")
    ws = moeq.workspace(moeq.moe_w4a16_workspace_size(d["T"], d["H"], d["I"], d["E"], d["k"]), "cuda")

    def step():
        moeq.moe_w4a16_forward(d["x"], d["logits"], d["k"], d["w13q"], d["w13s"], d["w2q"], d["w2s"], out=out, ws=ws)

    if trace:
        for _ in range(warmup):
            step()
        torch.cuda.synchronize()
        moeq.moe_trace_read(reset=True)
        moeq.moe_trace_enable(True)
    ms = timed_steps(step, steps, 0 if trace else warmup, flush, world)
    stages = None
    if trace:
        moeq.moe_trace_enable(False)
        stages = moeq.moe_trace_read(reset=True)
    return ms, stages, out


def run_mxfp4(moeq, d, steps, warmup, flush, world):
    """The MXFP4 layer: scale factors prepacked once (outside the timed steps), then forwards."""
    out = torch.empty((d["T"], d["H"]), dtype=torch.bfloat16, device="cuda")
    ws = moeq.workspace(moeq.lib().moe_mxfp4_workspace_size(d["T"], d["H"], d["I"], d["E"], d["k"]), "cuda")
    if "w13f" not in d:
        d["w13f"] = moeq.moe_mxfp4_prepack_scales(d["w13s"])
        d["w2f"] = moeq.moe_mxfp4_prepack_scales(d["w2s"])

    def step():
        moeq.moe_mxfp4_forward(d["x"], d["logits"], d["k"], d["w13q"], d["w13f"], d["w2q"], d["w2f"], out=out, ws=ws)

    return timed_steps(step, steps, warmup, flush, world)


def run_fp8(moeq, d, steps, warmup, flush, world):
    """Timed steps untraced, then a traced pass of 3 steps for the per-kernel times."""
    out = torch.empty((d["T"], d["H"]), dtype=torch.bfloat16, device="cuda")
    ws = moeq.workspace(moeq.moe_w8a8_block_fp8_workspace_size(d["T"], d["H"], d["I"], d["E"], d["k"]), "cuda")

    def step():
        moeq.moe_w8a8_block_fp8_forward(d["x"], d["logits"], d["k"], d["w13"], d["w13s"], d["w2"], d["w2s"], out=out,
                                        ws=ws)

    ms = timed_steps(step, steps, warmup, flush, world)
    torch.cuda.synchronize()
    moeq.moe_trace_read(reset=True)
    moeq.moe_trace_enable(True)
    timed_steps(step, 3, 0, flush, world)
    moeq.moe_trace_enable(False)
    return ms, moeq.moe_trace_read(reset=True)


def e2e_w4a16(moeq, d, steps, warmup, world):
    """Same layer through the C ABI with the step's inputs in pinned host memory: H2D of x and
    the router logits, the forward, D2H of the output, all inside the timed region."""
    hx = d["x"].cpu().pin_memory()
    hl = d["logits"].cpu().pin_memory()
    hout = torch.empty((d["T"], d["H"]), dtype=torch.bfloat16).pin_memory()
    dx = torch.empty_like(d["x"])
    dl = torch.empty_like(d["logits"])
    out = torch.empty((d["T"], d["H"]), dtype=torch.bfloat16, device="cuda")
    ws = moeq.workspace(moeq.moe_w4a16_workspace_size(d["T"], d["H"], d["I"], d["E"], d["k"]), "cuda")

    def step():
        dx.copy_(hx, non_blocking=True)
        dl.copy_(hl, non_blocking=True)
        moeq.moe_w4a16_forward(dx, dl, d["k"], d["w13q"], d["w13s"], d["w2q"], d["w2s"], out=out, ws=ws)
        hout.copy_(out, non_blocking=True)

    ms = timed_steps(step, steps, warmup, None, world)
    h2d = hx.numel() * hx.element_size() + hl.numel() * hl.element_size()
    d2h = hout.numel() * hout.element_size()
    return ms, h2d, d2h


def oracle_sample_time(d, ntok):
    """Seconds the CPU oracle takes for `ntok` tokens of the workload (host copies excluded)."""
    import oracle
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from tests._util import host_moe_weights
    x = W.np_bits(d["x"])
    logits = W.np_bits(d["logits"])
    toks = np.arange(ntok, dtype=np.int32)
    ids, _ = oracle.route_topk(logits[:ntok], d["k"])
    hw = host_moe_weights(d, ids.ravel())
    t0 = time.perf_counter()
    if d["kind"] == "w4a16":
        oracle.moe_w4a16(x, logits, d["k"], hw["w13q"], hw["w13s"], hw["w2q"], hw["w2s"], tokens=toks)
    else:
        oracle.moe_fp8(x, logits, d["k"], hw["w13"], hw["w13s"], hw["w2"], hw["w2s"], tokens=toks)
    return time.perf_counter() - t0


def cpu_info():
    model = ""
    try:
        for ln in open("/proc/cpuinfo"):
            if ln.startswith("model name"):
                model = ln.split(":", 1)[1].strip()
                break
    except OSError:
        pass
    return model


# ---------------------------------------------------------------------------------------------
# arms
# ---------------------------------------------------------------------------------------------

def decode_config(E, n_active, step_bytes, world):
    """The `config` of the decode headline, shared by both arms so that their lines compare."""
    return {"workload": f"decode_w4a16 T=32 H=7168 I=2048 E={E} k=8 (INT4 group-32, bf16 scales)",
            "touched_experts": n_active, "weight_bytes_per_step": step_bytes,
            "l2": f"flushed between steps ({L2_FLUSH_BYTES >> 20} MB written then read: cold, clean L2), "
                  "outside the timed events",
            "parallelism": f"replicas x{world}"}


def reference_arm(args, rank, world):
    """The CPU oracle, as it stands, over whole decode steps (all 32 tokens of the batch, ~2 s each
    on 16 host cores), so `--steps K --warmup W` runs K + W full steps and the line's
    ms_per_step x steps is the time the timed steps took."""
    if rank != 0:
        return
    import oracle
    wl = W.WORKLOADS["decode_w4a16"]
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    d = W.make_moe(wl, device=dev)
    T = d["T"]
    n_active = int(np.unique(oracle.route_topk(W.np_bits(d["logits"]), d["k"])[0]).size)
    step_bytes = n_active * W.w4a16_expert_bytes(d["H"], d["I"])
    for _ in range(args.warmup):
        oracle_sample_time(d, T)
    times = [oracle_sample_time(d, T) for _ in range(args.steps)]
    step_s = statistics.mean(times)
    value = step_bytes / step_s / 1e9
    cores = oracle.threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": decode_config(d["E"], n_active, step_bytes, world),
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": f"whole decode steps ({T} tokens each), {args.steps} timed after {args.warmup} "
                                   f"warm-up, {sum(times):.1f} s timed; host CPU: {cpu_info()}"},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def parallel_arm(args, moeq, rank, world, peaks, peak_src, flush):
    """The decode W4A16 layer split over the ranks: expert-parallel (rank r holds experts
    [r E/N, (r+1) E/N)) or tensor-parallel (rank r holds intermediate features [r I/N, (r+1) I/N) of
    every expert). One step = this rank's share through the C ABI + the all-reduce (sum) of the
    [T, H] bf16 output over the process group. The job's time is the slowest rank's."""
    from quantized_mixture_experts_align_b200 import sharding as S
    d = W.make_moe(W.WORKLOADS["decode_w4a16"], device="cuda", E=args.experts)
    n_active = touched_experts(moeq, d)
    step_bytes = n_active * W.w4a16_expert_bytes(d["H"], d["I"])  # every touched expert read once, job-wide
    full = {n: d.pop(n) for n in ("w13q", "w13s", "w2q", "w2s")}
    out = torch.empty((d["T"], d["H"]), dtype=torch.bfloat16, device="cuda")
    if args.parallel == "ep":
        w, base, local = S.shard_experts(full, "w4a16", rank, world)
        ws = moeq.workspace(moeq.moe_w4a16_ep_workspace_size(d["T"], d["H"], d["I"], d["E"], d["k"], local), "cuda")
        fn = lambda: S.forward_ep("w4a16", d["x"], d["logits"], d["k"], w, base, out=out, ws=ws)
        shape = f"experts [{base}, {base + local}) of {d['E']} on rank {rank}"
    else:
        w = S.shard_intermediate(full, "w4a16", d["I"], rank, world)
        ws = moeq.workspace(moeq.moe_w4a16_workspace_size(d["T"], d["H"], d["I"] // world, d["E"], d["k"]), "cuda")
        fn = lambda: S.forward_tp("w4a16", d["x"], d["logits"], d["k"], w, out=out, ws=ws)
        shape = f"features [{rank * d['I'] // world}, {(rank + 1) * d['I'] // world}) of {d['I']} on rank {rank}"
    del full
    torch.cuda.empty_cache()
    with ClockSampler(torch.cuda.current_device()) as clk:
        ms = timed_steps(fn, args.steps, args.warmup, flush, world)
    ms_step = max_over_ranks(statistics.mean(ms), world)
    value = step_bytes / (ms_step * 1e-3) / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "strong",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"decode_w4a16 T=32 H=7168 I=2048 E={d['E']} k=8 (INT4 group-32, bf16 scales)",
                   "parallelism": f"{args.parallel}{world}", "rank0_share": shape,
                   "touched_experts": n_active, "weight_bytes_per_step": step_bytes,
                   "l2": f"flushed between steps ({L2_FLUSH_BYTES >> 20} MB written then read), outside the events",
                   "collective": "all-reduce (sum) of the bf16 [T, H] output, NCCL" if world > 1 else "none (one rank)"},
        "roofline": {"bound": "hbm", "achieved": value / world, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": value / world / peaks["hbm_gbs"], "traffic": None,
                     "note": "whole step per GPU (share + all-reduce), not one kernel; the kernel roofline is on the "
                             "default (replicas) line", "peak_source": f"{peak_src} hbm_gbs (copy)"},
        "e2e": None,
        "gpu_launches": 5 * args.steps,
        "clocks": clk.summary(),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


def only_arm(args, moeq, rank, world):
    """One workload alone, for profiler captures of a small case; prints a JSON line of timings."""
    name = args.only
    if name == "dense_fp8":
        wl = W.WORKLOADS[name]
        M = args.tokens or 4096
        dd = W.make_dense_fp8(wl, M, device="cuda")
        C = torch.empty((M, wl.N), dtype=torch.bfloat16, device="cuda")
        ms = timed_steps(lambda: moeq.w8a8_block_fp8_matmul(dd["A"], dd["As"], dd["B"], dd["Bs"], out=C),
                         args.steps, args.warmup, None, world)
        line = {"only": name, "M": M, "ms": statistics.mean(ms), "tflops": 2.0 * M * wl.N * wl.K / statistics.mean(ms) / 1e9}
    elif name == "dense_fp8_channel":
        wl = W.WORKLOADS[name]
        M = args.tokens or 4096
        dd = W.make_dense_fp8_channel(wl, M, device="cuda")
        C = torch.empty((M, wl.N), dtype=torch.bfloat16, device="cuda")
        ms = timed_steps(lambda: moeq.w8a8_channel_fp8_matmul(dd["A"], dd["As"], dd["B"], dd["Bs"], out=C),
                         args.steps, args.warmup, None, world)
        line = {"only": name, "M": M, "ms": statistics.mean(ms), "tflops": 2.0 * M * wl.N * wl.K / statistics.mean(ms) / 1e9}
    else:
        d = W.make_moe(W.WORKLOADS[name], device="cuda", T=args.tokens, E=args.experts)
        if d["kind"] == "w4a16":
            ms, st, _ = run_w4a16(moeq, d, args.steps, args.warmup, None, world, trace=True)
        else:
            ms, st = run_fp8(moeq, d, args.steps, args.warmup, None, world)
        fl = W.moe_flops(d["T"], d["k"], d["H"], d["I"])
        line = {"only": name, "T": d["T"], "E": d["E"], "ms": statistics.mean(ms),
                "tflops": fl / statistics.mean(ms) / 1e9,
                "stages_ms": {k: v[0] / max(v[1], 1) for k, v in st.items() if v[1]}}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="moeq", choices=["moeq", "reference"])
    ap.add_argument("--headline-only", action="store_true", help="skip the secondary workloads")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--experts", type=int, default=None,
                    help="override E of the workload (small cases for profiler captures)")
    ap.add_argument("--tokens", type=int, default=None, help="override T of the workload (with --only)")
    ap.add_argument("--parallel", choices=["replicas", "ep", "tp"], default="replicas",
                    help="replicas: one independent layer per rank (default); ep / tp: the decode layer split "
                         "over the ranks (expert- / tensor-parallel shares + an all-reduce)")
    ap.add_argument("--only", choices=["prefill_w4a16", "moe_fp8", "dense_fp8", "dense_fp8_channel"], default=None,
                    help="time one secondary workload alone (small cases for profiler captures)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    rank, world, local = dist_setup(args.gpus)
    if args.impl == "reference":
        reference_arm(args, rank, world)
        if world > 1:
            torch.distributed.destroy_process_group()
        return

    import quantized_mixture_experts_align_b200 as moeq
    moeq.lib()
    peaks, peak_src = load_peaks()
    if args.only:
        only_arm(args, moeq, rank, world)
        return
    flush_buf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")

    flush_words = flush_buf.view(torch.int32)

    def flush():
        # write a buffer larger than L2, then read it back: the timed step starts with a cold L2
        # holding only clean lines (a write alone leaves ~L2-size dirty lines whose write-back
        # would land inside the next timed step: ~9 us on a 176 MB weight stream)
        flush_buf.fill_(1)
        flush_words.max()

    if args.parallel != "replicas":
        parallel_arm(args, moeq, rank, world, peaks, peak_src, flush)
        return

    # ---- headline: decode W4A16 -----------------------------------------------------------
    d = W.make_moe(W.WORKLOADS["decode_w4a16"], device="cuda", E=args.experts)
    n_active = touched_experts(moeq, d)
    w13_bytes = W.w4a16_expert_bytes(d["H"], d["I"]) * 2 // 3
    step_bytes = n_active * W.w4a16_expert_bytes(d["H"], d["I"])
    flops = W.moe_flops(d["T"], d["k"], d["H"], d["I"])
    dev_index = torch.cuda.current_device()
    # the timed steps run untraced (the stage events between kernels would cost the programmatic
    # launch overlap); a second, traced pass of the same steps gives the per-kernel times
    with ClockSampler(dev_index) as clk:
        ms, _, _ = run_w4a16(moeq, d, args.steps, args.warmup, flush, world, trace=False)
    value, ms_step = job_value(step_bytes / 1e9, statistics.mean(ms), world)
    _, stages, _ = run_w4a16(moeq, d, args.steps, 3, flush, world, trace=True)
    gu_ms, gu_calls = stages["gate_up"]
    gu_avg = gu_ms / max(gu_calls, 1)
    gu_bytes = n_active * (d["H"] * 2 * d["I"] // 2 + d["H"] // 32 * 2 * d["I"] * 2)
    achieved = gu_bytes / (gu_avg * 1e-3) / 1e9
    sha = src_sha("w4a16_mma.cu", "common.cuh")
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "traffic": traffic_for("w4a16_gate_up_decode", sha),
                "kernel": "w4a16_grouped_mma_kernel<8,4,GATEUP> (gate/up + SiLU*up)",
                "algorithmic_bytes_per_launch": gu_bytes, "launch_ms": gu_avg,
                "peak_source": f"{peak_src} hbm_gbs (copy)"}
    del w13_bytes

    e2e_ms, h2d, d2h = e2e_w4a16(moeq, d, args.steps, args.warmup, world)
    e2e_value, e2e_step = job_value(step_bytes / 1e9, statistics.mean(e2e_ms), world)
    e2e = {"value": e2e_value, "unit": "GB/s", "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": d2h, "ms_per_step": e2e_step}
    launch = launch_overhead_w4a16(moeq, d, args.steps, args.warmup)

    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": decode_config(d["E"], n_active, step_bytes, world),
        "tflops": world * flops / (ms_step * 1e-3) / 1e12,
        "roofline": roofline,
        "stages_ms": {k: v[0] / max(v[1], 1) for k, v in stages.items() if v[1]},
        "stages_note": "per-kernel times from a separate traced pass (events between kernels)",
        "e2e": e2e,
        "launch_overhead": launch,
        "gpu_launches": 5 * args.steps,
    }

    # ---- secondary workloads -----------------------------------------------------------------
    # the prefill and block-FP8 layer summaries go last on the line, after the long `also` record
    closing = {}
    if not args.headline_only:
        also = {}
        fp8m = measure_fp8_peak()
        also["fp8_peak"] = fp8m
        dp = W.make_moe(W.WORKLOADS["prefill_w4a16"], device="cuda")
        pms, _, _ = run_w4a16(moeq, dp, max(3, args.steps // 4), 3, None, world, trace=False)
        phost = moeq.moe_host_stats(reset=True)  # the timed calls above (warm-up included)
        _, pst, _ = run_w4a16(moeq, dp, 3, 3, None, world, trace=True)
        pflops = W.moe_flops(dp["T"], dp["k"], dp["H"], dp["I"])
        pstep = max_over_ranks(statistics.mean(pms), world)
        prows = expert_rows(moeq, dp)
        pbytes = int((prows > 0).sum()) * W.w4a16_expert_bytes(dp["H"], dp["I"])
        # each prefill step is a ~7 ms run timed on its own (a few steps): the burst peak applies
        bf16_peak = peaks["bf16_tflops"]
        proof = skew_roof_ms(prows, W.w4a16_expert_bytes(dp["H"], dp["I"]), dp["H"], dp["I"], peaks["hbm_gbs"],
                             bf16_peak)
        ptf = pflops / (pstep * 1e-3) / 1e12
        # dominant kernel: the tcgen05 gate/up GEMM (stage gate_up; the expert blocks with at most
        # 8 routed rows run in the few_rows stage), algorithmic FLOPs of the real routed rows of
        # its blocks only (padding excluded)
        pgu_ms, pgu_calls = pst["gate_up"]
        pgu_avg = pgu_ms / max(pgu_calls, 1)
        tail = prows % 256
        few = int(tail[(tail > 0) & (tail <= 8)].sum())
        pgu_flops = 2.0 * (dp["T"] * dp["k"] - few) * 2 * dp["I"] * dp["H"]
        prefill = {
            "metric": "prefill W4A16 MoE layer TFLOP/s", "value": ptf, "unit": "TFLOP/s",
            "workload": "prefill_w4a16 T=8192 H=7168 I=2048 E=384 k=8, Zipf-biased routing (INT4 group-32)",
            "ms_per_step": pstep, "steps": len(pms), "frac_of_bf16_burst": ptf / bf16_peak,
            "roofline": {"bound": "tensor", "achieved": pgu_flops / (pgu_avg * 1e-3) / 1e12, "peak": bf16_peak,
                         "unit": "TFLOP/s", "frac": pgu_flops / (pgu_avg * 1e-3) / 1e12 / bf16_peak, "traffic": None,
                         "kernel": "w4a16_tc_kernel<GATEUP> (gate/up + SiLU*up, blocks of more than 8 rows)",
                         "algorithmic_flops_per_launch": pgu_flops, "launch_ms": pgu_avg,
                         "rows_in_few_row_blocks": few,
                         "peak_source": f"{peak_src} bf16_tflops (burst)"},
            "skew_aware_roof_ms": proof, "frac_of_skew_aware_roof": proof / pstep,
            "host": {"library_us_per_call": phost["host_us"] / max(phost["calls"], 1),
                     "tensor_maps_encoded": phost["tmap_encoded"], "tensor_maps_reused": phost["tmap_reused"]},
            "weight_gbs": pbytes / (pstep * 1e-3) / 1e9, "active_experts": int((prows > 0).sum()),
            "stages_ms": {k: v[0] / max(v[1], 1) for k, v in pst.items() if v[1]}}
        # MXFP4 weights (E2M1 codes, UE8M0 group-32 scales) on the same layer: decode (T = 32,
        # uniform routing) and prefill (T = 8192, Zipf routing) over one set of 384 experts
        dm = W.make_moe(W.WORKLOADS["decode_mxfp4"], device="cuda")
        mms = run_mxfp4(moeq, dm, max(3, args.steps // 2), 3, flush, world)
        mstep = max_over_ranks(statistics.mean(mms), world)
        mact = touched_experts(moeq, dm)
        # bytes the hot path reads: E2M1 codes + the prepacked bf16 group factors (as the INT4
        # format; the stored UE8M0 scales are 1 byte per group, 17/18 of this)
        mbytes = mact * W.w4a16_expert_bytes(dm["H"], dm["I"])
        also["decode_mxfp4"] = {
            "workload": "T=32 H=7168 I=2048 E=384 k=8, MXFP4 weights, bf16 activations", "ms_per_step": mstep,
            "weight_gbs": mbytes / (mstep * 1e-3) / 1e9,
            "hbm_frac": mbytes / (mstep * 1e-3) / 1e9 / peaks["hbm_gbs"], "touched_experts": mact,
            "weight_bytes_per_step": mbytes}
        wlp = W.WORKLOADS["prefill_mxfp4"]
        dpm = dict(dm)
        dpm.update(T=wlp.T, x=W.bf16_normal((wlp.T, dm["H"]), W.generator(wlp.wid, 0, device="cuda"), "cuda"),
                   logits=W.router_logits(wlp, wlp.T, dm["E"], "cuda"))
        qms = run_mxfp4(moeq, dpm, max(3, args.steps // 4), 3, None, world)
        qstep = max_over_ranks(statistics.mean(qms), world)
        also["prefill_mxfp4"] = {
            "workload": "T=8192 H=7168 I=2048 E=384 k=8, Zipf-biased routing, MXFP4 weights", "ms_per_step": qstep,
            "tflops": pflops / (qstep * 1e-3) / 1e12,
            "frac_of_bf16_burst": pflops / (qstep * 1e-3) / 1e12 / bf16_peak}
        del dm, dpm
        torch.cuda.empty_cache()
        # NVFP4 weights (E2M1 codes, E4M3 group-16 scales, f32 tensor scales) on the same layer
        dn = W.make_moe(W.WORKLOADS["decode_nvfp4"], device="cuda")
        dn["w13f"] = moeq.moe_nvfp4_prepack_scales(dn["w13s"])
        dn["w2f"] = moeq.moe_nvfp4_prepack_scales(dn["w2s"])
        nout = torch.empty((dn["T"], dn["H"]), dtype=torch.bfloat16, device="cuda")
        nws = moeq.workspace(moeq.lib().moe_nvfp4_workspace_size(dn["T"], dn["H"], dn["I"], dn["E"], dn["k"]), "cuda")
        nstep_fn = lambda: moeq.moe_nvfp4_forward(dn["x"], dn["logits"], dn["k"], dn["w13q"], dn["w13f"], dn["g13"],
                                                  dn["w2q"], dn["w2f"], dn["g2"], out=nout, ws=nws)
        nms = timed_steps(nstep_fn, max(3, args.steps // 2), 3, flush, world)
        nstep = max_over_ranks(statistics.mean(nms), world)
        nact = touched_experts(moeq, dn)
        # bytes the hot path reads: codes + the prepacked bf16 group-16 factors
        H_, I_ = dn["H"], dn["I"]
        nexp = (2 * I_ * H_ + H_ * I_) // 2 + (2 * I_ * H_ + H_ * I_) // 16 * 2
        also["decode_nvfp4"] = {
            "workload": "T=32 H=7168 I=2048 E=384 k=8, NVFP4 weights, bf16 activations", "ms_per_step": nstep,
            "weight_gbs": nact * nexp / (nstep * 1e-3) / 1e9,
            "hbm_frac": nact * nexp / (nstep * 1e-3) / 1e9 / peaks["hbm_gbs"], "touched_experts": nact,
            "weight_bytes_per_step": nact * nexp}
        # NVFP4 prefill: the same experts, the prefill tokens and Zipf routing
        pout = torch.empty((wlp.T, dn["H"]), dtype=torch.bfloat16, device="cuda")
        pws = moeq.workspace(moeq.lib().moe_nvfp4_workspace_size(wlp.T, dn["H"], dn["I"], dn["E"], dn["k"]), "cuda")
        px = W.bf16_normal((wlp.T, dn["H"]), W.generator(wlp.wid, 0, device="cuda"), "cuda")
        plg = W.router_logits(wlp, wlp.T, dn["E"], "cuda")
        pfn = lambda: moeq.moe_nvfp4_forward(px, plg, dn["k"], dn["w13q"], dn["w13f"], dn["g13"], dn["w2q"], dn["w2f"],
                                             dn["g2"], out=pout, ws=pws)
        pnms = timed_steps(pfn, max(3, args.steps // 4), 3, None, world)
        pnstep = max_over_ranks(statistics.mean(pnms), world)
        also["prefill_nvfp4"] = {
            "workload": "T=8192 H=7168 I=2048 E=384 k=8, Zipf-biased routing, NVFP4 weights", "ms_per_step": pnstep,
            "tflops": pflops / (pnstep * 1e-3) / 1e12,
            "frac_of_bf16_burst": pflops / (pnstep * 1e-3) / 1e12 / bf16_peak}
        del dn, nout, nws, pout, pws, px, plg
        torch.cuda.empty_cache()
        # grouped W4A16 GEMM, contiguous layout: the prefill routing's rows per expert, each
        # expert padded to 128 rows (m_indices -1), its W13 (N = 2I = 4096, K = H = 7168)
        pad = [int(c) + (-int(c)) % 128 for c in prows]
        m_idx = torch.cat([torch.cat([torch.full((int(c),), e, dtype=torch.int32),
                                      torch.full((p - int(c),), -1, dtype=torch.int32)])
                           for e, (c, p) in enumerate(zip(prows, pad)) if p]).cuda()
        gA = W.bf16_normal((m_idx.numel(), dp["H"]), W.generator(90, 0, device="cuda"), "cuda")
        gC = torch.empty((m_idx.numel(), 2 * dp["I"]), dtype=torch.bfloat16, device="cuda")
        gws = moeq.workspace(moeq.lib().moe_w4a16_grouped_contiguous_workspace_size(
            m_idx.numel(), dp["H"], 2 * dp["I"], dp["E"]), "cuda")
        gms = timed_steps(lambda: moeq.moe_w4a16_grouped_contiguous(gA, dp["w13q"], dp["w13s"], m_idx, out=gC, ws=gws),
                          max(3, args.steps // 4), 3, None, world)
        gstep = max_over_ranks(statistics.mean(gms), world)
        gfl = 2.0 * int(prows.sum()) * 2 * dp["I"] * dp["H"]
        also["grouped_w4a16_contiguous"] = {
            "workload": f"prefill routing rows per expert padded to 128 ({m_idx.numel()} rows), N=4096 K=7168, E=384",
            "ms_per_step": gstep, "tflops": gfl / (gstep * 1e-3) / 1e12,
            "frac_of_bf16_burst": gfl / (gstep * 1e-3) / 1e12 / bf16_peak}
        del gA, gC, gws, m_idx, dp
        torch.cuda.empty_cache()
        # masked layout: the decode routing's rows per expert in budgets of 16 rows, expected_m 1
        dd8 = W.make_moe(W.WORKLOADS["decode_w4a16"], device="cuda")
        drows = expert_rows(moeq, dd8)
        max_m = 16
        masked = torch.as_tensor(np.minimum(drows, max_m).astype(np.int32)).cuda()
        mA = W.bf16_normal((dd8["E"] * max_m, dd8["H"]), W.generator(91, 0, device="cuda"), "cuda")
        mC = torch.empty((dd8["E"] * max_m, 2 * dd8["I"]), dtype=torch.bfloat16, device="cuda")
        mws = moeq.workspace(moeq.lib().moe_w4a16_grouped_masked_workspace_size(
            dd8["E"], max_m, dd8["H"], 2 * dd8["I"], 1), "cuda")
        mms = timed_steps(lambda: moeq.moe_w4a16_grouped_masked(mA, dd8["w13q"], dd8["w13s"], masked, 1, out=mC, ws=mws),
                          args.steps, 3, flush, world)
        mstep = max_over_ranks(statistics.mean(mms), world)
        mbytes = int((drows > 0).sum()) * (W.w4a16_expert_bytes(dd8["H"], dd8["I"]) * 2 // 3)
        also["grouped_w4a16_masked"] = {
            "workload": f"decode routing rows per expert in budgets of {max_m} rows, N=4096 K=7168, E=384, expected_m 1",
            "ms_per_step": mstep, "weight_gbs": mbytes / (mstep * 1e-3) / 1e9,
            "hbm_frac": mbytes / (mstep * 1e-3) / 1e9 / peaks["hbm_gbs"], "active_experts": int((drows > 0).sum())}
        del mA, mC, mws, dd8
        torch.cuda.empty_cache()
        df = W.make_moe(W.WORKLOADS["moe_fp8"], device="cuda")
        fms, fst = run_fp8(moeq, df, max(3, args.steps // 4), 3, None, world)
        fflops = W.moe_flops(df["T"], df["k"], df["H"], df["I"])
        fstep = max_over_ranks(statistics.mean(fms), world)
        # a ~3 ms step timed on its own (a few steps): the burst peak applies
        if "burst" in fp8m:
            fp8_peak, fp8_src = fp8m["burst"], "measured in this run: " + fp8m["how"] + " (burst)"
        else:
            fp8_peak = 2.0 * peaks["bf16_tflops"]
            fp8_src = f"2 x {peak_src} bf16 burst (nominal fp8/bf16 ratio; fp8 measurement failed)"
        frows = expert_rows(moeq, df)
        fbytes = int((frows > 0).sum()) * W.fp8_expert_bytes(df["H"], df["I"])
        froof = skew_roof_ms(frows, W.fp8_expert_bytes(df["H"], df["I"]), df["H"], df["I"], peaks["hbm_gbs"], fp8_peak)
        fgu_ms, fgu_calls = fst["gate_up"]
        fgu_avg = fgu_ms / max(fgu_calls, 1)
        fgu_flops = 2.0 * df["T"] * df["k"] * 2 * df["I"] * df["H"]
        moe_fp8 = {
            "metric": "block-FP8 MoE layer TFLOP/s", "value": fflops / (fstep * 1e-3) / 1e12, "unit": "TFLOP/s",
            "workload": "moe_fp8 T=4096 H=7168 I=2048 E=256 k=8, block-FP8 [128,128], Zipf-biased routing",
            "ms_per_step": fstep, "tflops": fflops / (fstep * 1e-3) / 1e12,
            "frac_of_fp8_burst": fflops / (fstep * 1e-3) / 1e12 / fp8_peak,
            "roofline": {"bound": "tensor", "achieved": fgu_flops / (fgu_avg * 1e-3) / 1e12, "peak": fp8_peak,
                         "unit": "TFLOP/s", "frac": fgu_flops / (fgu_avg * 1e-3) / 1e12 / fp8_peak, "traffic": None,
                         "kernel": "block-FP8 grouped gate/up (+ SiLU*up + E4M3 requantization)",
                         "algorithmic_flops_per_launch": fgu_flops, "launch_ms": fgu_avg},
            "peak_tflops": fp8_peak, "peak_source": fp8_src,
            "weight_gbs": fbytes / (fstep * 1e-3) / 1e9, "hbm_frac": fbytes / (fstep * 1e-3) / 1e9 / peaks["hbm_gbs"],
            "active_experts": int((frows > 0).sum()),
            "skew_aware_roof_ms": froof, "frac_of_skew_aware_roof": froof / fstep,
            "stages_ms": {k: v[0] / max(v[1], 1) for k, v in fst.items() if v[1]}}
        del df
        torch.cuda.empty_cache()
        sweep = {}
        fp8_burst = fp8m.get("burst", 2.0 * peaks["bf16_tflops"])
        wl = W.WORKLOADS["dense_fp8"]
        for M in wl.M_list:
            dd = W.make_dense_fp8(wl, M, device="cuda")
            C = torch.empty((M, wl.N), dtype=torch.bfloat16, device="cuda")
            fn = lambda: moeq.w8a8_block_fp8_matmul(dd["A"], dd["As"], dd["B"], dd["Bs"], out=C)
            dms = statistics.mean(timed_steps(fn, max(3, args.steps // 4), 3, flush, world))
            byts = wl.N * wl.K + dd["Bs"].numel() * 4 + M * wl.K + M * (wl.K // 128) * 4 + 2 * M * wl.N
            fl = 2.0 * M * wl.N * wl.K
            sweep[M] = {"ms": dms, "tflops": fl / (dms * 1e-3) / 1e12, "gbs": byts / (dms * 1e-3) / 1e9,
                        "hbm_frac": byts / (dms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                        "fp8_frac": fl / (dms * 1e-3) / 1e12 / fp8_burst}
            del dd, C
        also["dense_fp8_sweep"] = {"workload": "A [M,7168] x B [24576,7168] block-FP8, C bf16", "by_M": sweep,
                                   "fp8_peak_tflops": fp8_burst,
                                   "fp8_peak_source": ("measured in this run (burst): " + fp8m["how"]) if "burst" in fp8m
                                   else f"2 x {peak_src} bf16 burst (nominal ratio)"}
        # channelwise FP8 (per-token x per-channel scales) at the page's N = K = 4096 example, plus
        # the block sweep's 24576 x 7168 weights at 4096 rows for comparison
        cwl = W.WORKLOADS["dense_fp8_channel"]
        csweep = {}
        for (M, Nc, Kc) in [(M, cwl.N, cwl.K) for M in cwl.M_list] + [(4096, 24576, 7168)]:
            dd = W.make_dense_fp8_channel(cwl, M, device="cuda", N=Nc, K=Kc)
            C = torch.empty((M, Nc), dtype=torch.bfloat16, device="cuda")
            fn = lambda: moeq.w8a8_channel_fp8_matmul(dd["A"], dd["As"], dd["B"], dd["Bs"], out=C)
            dms = statistics.mean(timed_steps(fn, max(3, args.steps // 4), 3, flush, world))
            byts = Nc * Kc + Nc * 4 + M * Kc + M * 4 + 2 * M * Nc
            fl = 2.0 * M * Nc * Kc
            csweep[f"M={M} N={Nc} K={Kc}"] = {
                "ms": dms, "tflops": fl / (dms * 1e-3) / 1e12, "gbs": byts / (dms * 1e-3) / 1e9,
                "hbm_frac": byts / (dms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                "fp8_frac": fl / (dms * 1e-3) / 1e12 / fp8_burst,
                "roof_frac": max(byts / (peaks["hbm_gbs"] * 1e9), fl / (fp8_burst * 1e12)) / (dms * 1e-3)}
            del dd, C
        also["dense_fp8_channel_sweep"] = {
            "workload": "A [M,K] e4m3 x As [M] per token, B [N,K] e4m3 x Bs [N] per channel, C bf16",
            "by_shape": csweep, "fp8_peak_tflops": fp8_burst,
            "roof": "max(bytes / measured HBM, flops / FP8 burst peak) / time"}
        line["also"] = also
        closing = {"prefill": prefill, "moe_fp8": moe_fp8}

    line["clocks"] = clk.summary()

    # ---- CPU baseline: the oracle as it stands, bounded sample, rank 0 only --------------------
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        # whole decode steps (all T tokens), repeated until about 10 s of CPU work
        times = []
        while sum(times) < 10.0 and len(times) < 20:
            times.append(oracle_sample_time(d, d["T"]))
        full_s = statistics.mean(times)
        line["cpu_baseline"] = {"value": step_bytes / full_s / 1e9, "unit": "GB/s", "cores": oracle.threads(),
                                "kind": "oracle",
                                "sample": f"{len(times)} full decode steps ({d['T']} tokens each, {sum(times):.1f} s "
                                          f"total); host CPU: {cpu_info()}"}
    line.update(closing)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
