"""Benchmark of the MoE FFN layer on B200 (one JSON line on stdout).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]

A step is one moe_layer call (router, top-K, permutation, expert GEMMs, shared
expert, combine) over one batch of the workload, inputs resident in HBM.  The
default workload is the largest one that fits one GPU: the skewed layer
(T=8192, H=7168, E=256, K=8, I=2048, SiLU, bf16, one ungated shared expert of
intermediate 2048, Zipf(1.1) router bias; 22.5 GB of expert weights).  Under
torchrun (N > 1) every rank runs an independent replica of the layer on its own
GPU (the layer does not shard); the time is the max over ranks and `value`
counts the tokens of all ranks.  `--gpus N` with N > 1 outside torchrun starts
the N ranks itself (torch.distributed.run on 127.0.0.1).

--impl reference times the f64 CPU oracle on the host cores instead (rank 0
only), on bounded token samples of the same workload.

--op backward times the backward of the combine and of act*up (one launch of
each per step, f32) on the workload's T, K, H, I instead of the forward layer.
"""
from __future__ import annotations

import argparse
import hashlib
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

import workloads  # noqa: E402

METRIC = "MoE layer tokens/s at 1 B200; % of BF16 tensor peak (prefill) / HBM BW (decode)"
UNIT = "tokens/s"
DEFAULT_CONFIG = "skewed_zipf_t8192"
NROT = 8  # token batches a layer bench rotates over
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
NOMINAL = {"hbm_gbs": 8000.0, "bf16_tflops": 2250.0}  # B200 data-sheet HBM3e bandwidth and dense bf16 rate


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


# ------------------------------------------------------------------ algorithmic work per kernel launch
def algorithmic(spec, counts):
    """Bytes (and flops) each kernel of one step must move at minimum, from the actual routing.

    Weights are counted once per touched expert; activations read once and outputs written once."""
    T, H, E, I, K, Is = spec.T, spec.H, spec.E, spec.I, spec.K, spec.shared_I
    P = T * K
    touched = int(np.count_nonzero(counts))
    # stored bytes per weight of the gate/up and of the down projections
    wb = {"f32": 4, "bf16": 2, "q8_0": 1 + 2.0 / 32, "q4_k": 144 / 256, "q4_k_q6_k": 144 / 256}[spec.w_dtype]
    wbd = 210 / 256 if spec.w_dtype == "q4_k_q6_k" else wb
    ab = 4 if spec.act_dtype == "f32" else 2
    rb = 4 if spec.router_dtype == "f32" else 2
    tc = spec.act_dtype == "bf16" and spec.w_dtype == "bf16" and T > 64
    hb = 2 if tc else 4
    k = {}
    k["expert_gate_up_gemm"] = k["stream_gate_up"] = dict(
        bytes=touched * 2 * I * H * wb + P * H * ab + P * I * hb, flops=2.0 * P * 2 * I * H)
    k["expert_down_gemm"] = k["stream_down"] = dict(
        bytes=touched * H * I * wbd + P * I * hb + P * H * 4 + P * 4, flops=2.0 * P * H * I)
    k["router_gemm"] = k["router_logits"] = dict(bytes=E * H * rb + T * H * ab + T * E * 4, flops=2.0 * T * E * H)
    k["router_topk"] = dict(bytes=T * E * 4 * (2 if spec.router_bias else 1) + P * 8, flops=0)
    k["permute"] = dict(bytes=P * 4 * 3 + (2 * E + 1) * 4, flops=0)
    k["gather_rows"] = dict(bytes=P * H * ab * 2 + P * 4, flops=0)
    k["combine"] = dict(bytes=P * H * 4 + (T * H * 4 if Is else 0) + T * H * ab, flops=0)
    if Is:
        k["shared_gate_up_gemm"] = dict(bytes=2 * Is * H * wb + T * H * ab + T * Is * hb, flops=2.0 * T * 2 * Is * H)
        k["shared_down_gemm"] = dict(bytes=Is * H * wbd + T * Is * hb + T * H * 4, flops=2.0 * T * H * Is)
    layer = dict(bytes=touched * (2 * wb + wbd) * I * H + E * H * rb + ((2 * wb + wbd) * Is * H if Is else 0)
                 + 2 * T * H * ab,
                 flops=2.0 * (T * E * H + P * 3 * H * I + T * 3 * H * Is))
    # fused launches: the sum of the steps they replace
    k["route_permute_gather"] = dict(bytes=sum(k[n]["bytes"] for n in ("router_topk", "permute", "gather_rows")),
                                     flops=0)
    k["decode_layer"] = dict(layer)  # the whole layer in one launch
    return k, layer, touched


def kernel_roofline(alg, avg_ms, peaks, peak_src):
    """One kernel's achieved rate (its algorithmic work per step over its time per step, `avg_ms`) against its
    roofline: TFLOP/s when its arithmetic intensity is above the
    ridge of the measured peaks, else GB/s.  `frac` divides by the sustained bf16 rate (a kernel timed inside a
    long loop of steps) or the measured copy bandwidth; `frac_burst` by the burst bf16 rate; `frac_nominal` by
    the data-sheet figure (2.25 PFLOP/s dense bf16, 8 TB/s)."""
    avg_s = avg_ms / 1e3
    tensor_bound = alg["flops"] / max(alg["bytes"], 1) > 1e3 * peaks["bf16_tflops"] / peaks["hbm_gbs"]
    if tensor_bound:
        achieved, peak, unit = alg["flops"] / avg_s / 1e12, peaks["bf16_tflops_sustained"], "TFLOP/s"
        extra = {"frac_burst": achieved / peaks["bf16_tflops"], "peak_burst": peaks["bf16_tflops"],
                 "frac_nominal": achieved / NOMINAL["bf16_tflops"]}
    else:
        achieved, peak, unit = alg["bytes"] / avg_s / 1e9, peaks["hbm_gbs"], "GB/s"
        extra = {"frac_nominal": achieved / NOMINAL["hbm_gbs"]}
    return dict({"bound": "tensor" if tensor_bound else "hbm", "achieved": achieved, "peak": peak, "unit": unit,
                 "frac": achieved / peak}, **extra, avg_us=1e3 * avg_ms,
                algorithmic_bytes_per_launch=alg["bytes"], algorithmic_flops_per_launch=alg["flops"],
                peak_source=f"{peak_src} ({'bf16_tflops_sustained' if tensor_bound else 'hbm_gbs'})")


def expert_load(counts_list):
    """Rows per expert over the step's token batches: touched experts, the largest and the smallest
    nonzero load (mean over batches), and batch 0's sorted loads in full."""
    touched = [int(np.count_nonzero(c)) for c in counts_list]
    mx = [int(c.max()) for c in counts_list]
    mn = [int(c[c > 0].min()) if np.any(c > 0) else 0 for c in counts_list]
    c0 = np.sort(counts_list[0])[::-1]
    return {"touched_mean": float(np.mean(touched)), "max_rows_mean": float(np.mean(mx)),
            "min_nonzero_rows_mean": float(np.mean(mn)), "max_rows": max(mx), "min_nonzero_rows": min(mn),
            "batch0_rows_desc": [int(v) for v in c0[c0 > 0]]}


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


# ------------------------------------------------------------------ clocks during the timed region
class ClockSampler:
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, index: int, period_s: float = 0.02):
        self.index, self.period = index, period_s
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.nv = None

    def _sample(self):
        nv = self.nv
        self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
        try:
            r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except Exception:
            r = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
        for bit, name in self.REASONS.items():
            if r & bit:
                self.reasons.add(name)

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            self._stop.wait(self.period)

    def start(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()

    def stop(self):
        if self.ok and self._t:
            self._stop.set()
            self._t.join()
            self._sample()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["nvml unavailable"]}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples)}


# ------------------------------------------------------------------ traffic from a committed ncu capture
def _traffic(kernel: str, workload: str):
    """Per-launch DRAM bytes of `kernel` from profiles/traffic.json, if taken on the current source."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    rec = d.get(f"{kernel}@{workload}")
    if not rec:
        return None
    for name, sha in rec["sources"].items():  # every source the kernel is built from, unchanged
        src = os.path.join(ROOT, "mixture_experts_ffn_07_b200", "csrc", name)
        if not os.path.exists(src) or hashlib.sha256(open(src, "rb").read()).hexdigest()[:16] != sha:
            return None
    return rec["bytes_per_launch"]


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def per_call_ms(call, stream, n: int = 50, warmup: int = 10, flush=None) -> float:
    """Median over n single calls of their CUDA-event time on `stream`; with `flush` (a device buffer
    larger than L2) each call follows a write of the whole buffer, so it starts from a cold L2."""
    import torch
    for _ in range(warmup):
        call()
    ts = []
    for i in range(n):
        if flush is not None:
            flush.fill_(i & 0xFF)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        call()
        b.record(stream)
        b.synchronize()
        ts.append(a.elapsed_time(b))
    return float(statistics.median(ts))


def max_over_ranks(dist, x: float, device) -> float:
    """The largest of every rank's x (a device time in ms): the job's time.  Every
    rank must call it at the same point."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, tokens_per_step: int, steps: int, ms: float) -> float:
    """Whole-job tokens/s: every replica runs `steps` layers of `tokens_per_step`
    tokens; the job takes the slowest rank's `ms`."""
    return world * tokens_per_step * steps / (ms / 1e3)


# ------------------------------------------------------------------ CPU oracle timing
def time_oracle(spec, wl, budget_s: float, max_tokens=None):
    """Oracle on host cores over a bounded token sample sized to ~budget_s seconds. Returns (tokens/s, info)."""
    import oracle
    L = oracle.from_workload(wl)
    cores = oracle.threads()
    n0 = max(1, min(spec.T, cores))
    t0 = time.perf_counter()
    oracle.layer(L, tokens=np.arange(n0))
    dt = time.perf_counter() - t0
    n = int(min(spec.T if max_tokens is None else max_tokens, max(n0, n0 * budget_s / max(dt, 1e-6))))
    if n > n0:
        tok = np.linspace(0, spec.T - 1, n).round().astype(np.int64)
        t0 = time.perf_counter()
        oracle.layer(L, tokens=tok)
        dt = time.perf_counter() - t0
    else:
        n = n0
    return n / dt, dict(cores=cores, sample=f"{n} of {spec.T} tokens, full layer in f64 ({dt:.2f} s)", tokens=n,
                        seconds=dt)


def time_oracle_1thread(spec, wl, budget_s: float):
    """The same oracle on one host thread, over a small token sample (about budget_s seconds)."""
    import oracle
    n_all = oracle.threads()
    oracle.set_threads(1)
    try:
        v, info = time_oracle(spec, wl, budget_s=budget_s, max_tokens=max(1, min(spec.T, 64)))
    finally:
        oracle.set_threads(n_all)
    return v, info


def run_reference(args, spec):
    ws, rank, _ = _dist()
    if rank != 0:
        return 0
    wl = workloads.make(spec)
    import oracle
    L = oracle.from_workload(wl)
    cores = oracle.threads()
    per_step = max(1, min(spec.T, cores))
    rng = np.random.default_rng(0)
    for _ in range(args.warmup):
        oracle.layer(L, tokens=rng.integers(0, spec.T, per_step))
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.layer(L, tokens=rng.integers(0, spec.T, per_step))
    dt = time.perf_counter() - t0
    value = per_step * args.steps / dt
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": spec.name, "T": spec.T, "H": spec.H, "E": spec.E, "I": spec.I, "top_k": spec.K,
                       "shared_I": spec.shared_I, "step_sample_tokens": per_step},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "cpu_model": cpu_model(), "kind": "oracle",
                             "sample": f"{per_step} random tokens of {spec.T} per step, full layer in f64"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ our arm
def run_ours(args, spec):
    import torch
    ws_n, rank, local = _dist()
    torch.cuda.set_device(local)
    dist = None
    if ws_n > 1:
        import datetime

        import torch.distributed as dist
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))

    import mixture_experts_ffn_07_b200 as moe
    from mixture_experts_ffn_07_b200 import host

    moe.set_pair_gemm(bool(args.pair_gemm))
    moe.set_decode_stream(bool(args.decode_stream))
    wl = workloads.make(spec)
    desc, w, x = host.upload(wl)
    T, H = spec.T, spec.H
    out = torch.empty((T, H), dtype=x.dtype, device="cuda")
    wsb = torch.empty(moe.workspace_bytes(desc), dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    # Steps rotate over NROT seeded token batches, so consecutive steps route to different experts (a step
    # that re-ran the same batch would find part of its experts' weights still in L2).
    xs = [x] + [host.to_device(workloads.token_batch(spec, i), spec.act_dtype) for i in range(1, NROT)]
    # routing once per batch (outside timing) for the touched-expert counts of the algorithmic bytes (mean)
    algs, loads = [], []
    for xb in xs:
        _, ids, _, _ = host.run_route(desc, w, xb)
        loads.append(np.bincount(ids.cpu().numpy().reshape(-1), minlength=spec.E))
        algs.append(algorithmic(spec, loads[-1]))
    kern_alg = {n: {q: float(np.mean([a[0][n][q] for a in algs])) for q in ("bytes", "flops")} for n in algs[0][0]}
    layer_alg = {q: float(np.mean([a[1][q] for a in algs])) for q in ("bytes", "flops")}
    touched = float(np.mean([a[2] for a in algs]))

    for i in range(max(args.warmup, 3)):
        moe.layer(desc, xs[i % NROT], w, out, wsb)
    torch.cuda.synchronize()
    assert moe.last_device_status() == moe.MOE_OK

    clocks = ClockSampler(torch.cuda.current_device())
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    n_launch0 = moe.launch_count()
    ev0.record(stream)
    for i in range(args.steps):
        moe.layer(desc, xs[i % NROT], w, out, wsb)
    ev1.record(stream)
    torch.cuda.synchronize()
    n_launch = moe.launch_count() - n_launch0
    clocks.stop()
    if dist:
        dist.barrier()
    ms = ev0.elapsed_time(ev1)
    status = moe.last_device_status()

    # per-kernel durations: the same steps again with an event pair around every launch
    # (events between kernels serialise them, so this pass is not the timed one)
    moe.trace_enable(True)
    for i in range(min(args.steps, 400)):
        moe.layer(desc, xs[i % NROT], w, out, wsb)
    torch.cuda.synchronize()
    moe.trace_enable(False)
    trace = moe.trace_read()
    ms = max_over_ranks(dist, ms, "cuda")
    ms_step = ms / args.steps
    value = job_throughput(ws_n, T, args.steps, ms)

    # per-kernel durations (CUDA events around each launch on the launching stream)
    per = {}
    for name, t in trace:
        per.setdefault(name, []).append(t)
    kernels = {n: {"launches": len(v), "avg_ms": sum(v) / len(v), "total_ms": sum(v)} for n, v in per.items()}
    tot = sum(k["total_ms"] for k in kernels.values()) or 1.0
    for k in kernels.values():
        k["share"] = k["total_ms"] / tot
    # a step's time per kernel: a compute-bound expert GEMM runs as two launches (full 256-row tiles on CTA pairs,
    # then each group's remaining rows, traced as "<name>_tail"), which together do that GEMM's work
    traced_steps = min(args.steps, 400)
    step_ms = {}
    for n, k in kernels.items():
        base = n[: -len("_tail")] if n.endswith("_tail") else n
        step_ms[base] = step_ms.get(base, 0.0) + k["total_ms"] / traced_steps
    dom = max(step_ms, key=step_ms.get) if step_ms else None

    peaks, peak_src = _peaks()
    roofline = None
    if dom:
        roofline = kernel_roofline(kern_alg.get(dom, {"bytes": 0, "flops": 0}), step_ms[dom], peaks, peak_src)
        roofline.update(traffic=_traffic(dom, spec.name), kernel=dom,
                        launches_per_step=sum(k["launches"] for n, k in kernels.items()
                                              if n in (dom, dom + "_tail")) / traced_steps)
        # every GEMM of the step against the same peaks (the expert GEMMs carry the layer's arithmetic)
        roofline["gemms"] = {n: kernel_roofline(kern_alg[n], step_ms[n], peaks, peak_src)
                             for n in step_ms if n.endswith("_gemm") and n in kern_alg}
    layer_s = ms_step / 1e3
    layer_roof = {"bytes": layer_alg["bytes"], "flops": layer_alg["flops"],
                  "GB/s": layer_alg["bytes"] / layer_s / 1e9, "TFLOP/s": layer_alg["flops"] / layer_s / 1e12,
                  "hbm_frac": layer_alg["bytes"] / layer_s / 1e9 / peaks["hbm_gbs"],
                  "tensor_frac": layer_alg["flops"] / layer_s / 1e12 / peaks["bf16_tflops_sustained"],
                  "touched_experts": touched, "expert_load": expert_load(loads)}

    # end to end through the public host-buffer call (moe_layer_host): every step copies its x from pinned host
    # memory, runs the layer and copies its out back.  Two streams, each with its own device buffers, workspace
    # and pinned output, take alternate steps, so one step's copies overlap the other's compute -- how a server
    # keeps the GPU busy while it moves the next batch.
    xhs = [xb.cpu().pin_memory() for xb in xs]
    xh = xhs[0]
    e2e_sets = []
    for _ in range(2):
        e2e_sets.append(dict(oh=torch.empty_like(xh).pin_memory(), xd=torch.empty_like(x), od=torch.empty_like(x),
                             ws=torch.empty(moe.workspace_bytes(desc), dtype=torch.uint8, device="cuda"),
                             stream=torch.cuda.Stream()))

    def e2e_step(i):
        b = e2e_sets[i % 2]
        moe.layer_host(desc, xhs[i % NROT], w, b["oh"], b["xd"], b["od"], b["ws"], stream=b["stream"])

    for i in range(max(args.warmup, 3)):
        e2e_step(i)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for b in e2e_sets:
        b["stream"].wait_event(e0)
    for i in range(args.steps):
        e2e_step(i)
    for b in e2e_sets:
        done = torch.cuda.Event()
        done.record(b["stream"])
        stream.wait_event(done)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    e2e_ms = max_over_ranks(dist, e2e_ms, "cuda")
    io_bytes = T * H * x.element_size()

    # single calls on one token batch: median of 50 after 10 warm-up calls, each after a 512 MB scratch write
    # (cold L2), and back to back (warm: whatever of the step's data L2 still holds)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device="cuda")
    one = lambda: moe.layer(desc, xs[0], w, out, wsb)  # noqa: E731
    cold_ms = per_call_ms(one, stream, flush=flush)
    warm_ms = per_call_ms(one, stream)
    del flush
    single = {"calls": 50, "warmup": 10, "flush_bytes": 512 << 20, "cold_median_ms": cold_ms,
              "warm_median_ms": warm_ms, "cold_tokens_per_s": T / cold_ms * 1e3, "warm_tokens_per_s": T / warm_ms * 1e3,
              "cold_hbm_frac": algs[0][1]["bytes"] / (cold_ms / 1e3) / 1e9 / peaks["hbm_gbs"]}

    cpu = None
    if rank == 0 and ws_n == 1 and not args.no_cpu_baseline:
        v, info = time_oracle(spec, wl, budget_s=args.cpu_budget)
        v1, info1 = time_oracle_1thread(spec, wl, budget_s=min(3.0, args.cpu_budget))
        cpu = {"value": v, "unit": UNIT, "cores": info["cores"], "cpu_model": cpu_model(), "kind": "oracle",
               "sample": info["sample"], "value_1thread": v1, "sample_1thread": info1["sample"]}
        if info["tokens"] < spec.T:  # tokens/s of the sample; the full layer's time is extrapolated from it
            cpu["extrapolation"] = {"full_layer_s": spec.T / v, "from_tokens": info["tokens"], "of_tokens": spec.T}

    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws_n, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": spec.act_dtype if spec.w_dtype in ("f32", "bf16") else f"{spec.w_dtype}x{spec.act_dtype}",
            "data": "synthetic",
            "config": {"workload": spec.name, "T": spec.T, "H": spec.H, "E": spec.E, "I": spec.I, "top_k": spec.K,
                       "act": spec.act, "shared_I": spec.shared_I, "parallelism": f"replicas{ws_n}",
                       "pair_gemm": bool(args.pair_gemm), "decode_stream": bool(args.decode_stream),
                       "l2": f"no flush: inputs larger than L2; x rotates over {NROT} token batches, so consecutive "
                             "steps route to different experts"},
            "e2e": {"value": job_throughput(ws_n, T, args.steps, e2e_ms), "unit": UNIT, "h2d_bytes_per_step": io_bytes,
                    "d2h_bytes_per_step": io_bytes, "call": "moe_layer_host", "streams": 2},
            "roofline": roofline, "layer_roofline": layer_roof, "cpu_baseline": cpu, "gpu_launches": n_launch,
            "single_call": single, "clocks": clocks.summary(), "device_status": moe.status_string(status),
            "kernels": {n: {"launches": k["launches"], "avg_us": 1e3 * k["avg_ms"], "share": round(k["share"], 4)}
                        for n, k in sorted(kernels.items(), key=lambda kv: -kv[1]["total_ms"])}}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    return 0


# ------------------------------------------------------------------ backward of combine and act * up
BWD_METRIC = "MoE backward (combine + act*up) tokens/s at 1 B200; % of HBM BW"


def backward_bytes(T, K, H, I):
    """Algorithmic bytes of one launch of each backward kernel: every input read once, every output written once."""
    P = T * K
    return {"combine_backward": 4 * (T * H + 2 * P * H + 2 * P), "act_up_backward": 4 * P * I * 5}


def _backward_host_inputs(spec, seed=11):
    T, K, H, I = spec.T, spec.K, spec.H, spec.I
    P = T * K
    rng = np.random.default_rng(seed)
    return {"y": rng.standard_normal((T, K, H), np.float32), "w": rng.random((T, K), np.float32),
            "d_out": rng.standard_normal((T, H), np.float32),
            "gate_up": (3 * rng.standard_normal((P, 2 * I))).astype(np.float32),
            "d_h": rng.standard_normal((P, I), np.float32)}


def _time_oracle_backward(spec, hin, budget_s):
    import oracle
    reps, t0 = 0, time.perf_counter()
    while True:
        oracle.combine_backward(hin["y"], hin["w"], hin["d_out"])
        oracle.act_up_backward(spec.act, hin["gate_up"], hin["d_h"])
        reps += 1
        dt = time.perf_counter() - t0
        if dt >= budget_s or reps >= 1000:
            break
    return spec.T * reps / dt, dict(cores=oracle.threads(), sample=f"all {spec.T} tokens x {reps} passes, f64")


def run_backward(args, spec):
    """--op backward: one step = moe_combine_backward + moe_act_up_backward over one batch of the workload's slots."""
    T, K, H, I = spec.T, spec.K, spec.H, spec.I
    P = T * K
    ws_n, rank, local = _dist()
    hin = _backward_host_inputs(spec)
    if args.impl == "reference":
        if rank != 0:
            return 0
        v, info = _time_oracle_backward(spec, hin, budget_s=min(args.cpu_budget, 5.0))
        print(json.dumps({"impl": "reference", "metric": BWD_METRIC, "value": v, "unit": UNIT, "n_gpus": ws_n,
                          "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * T / v,
                          "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                          "data": "synthetic", "config": {"workload": spec.name + "/backward", "T": T, "K": K,
                                                          "H": H, "I": I, "act": spec.act},
                          "cpu_baseline": {"value": v, "unit": UNIT, "cores": info["cores"], "kind": "oracle",
                                           "sample": info["sample"]},
                          "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}),
              flush=True)
        return 0
    import torch
    torch.cuda.set_device(local)
    import mixture_experts_ffn_07_b200 as moe
    dev = {k: torch.from_numpy(v).cuda() for k, v in hin.items()}
    alg = backward_bytes(T, K, H, I)
    set_bytes = sum(alg.values())
    nsets = max(1, min(8, -(-400_000_000 // set_bytes)))  # rotate buffer sets: > 3x L2 between reuses
    sets = []
    for i in range(nsets):
        d = dev if i == 0 else {k: v.clone() for k, v in dev.items()}
        d = dict(d, d_y=torch.empty((T, K, H), device="cuda"), d_w=torch.empty((T, K), device="cuda"),
                 d_gu=torch.empty((P, 2 * I), device="cuda"))
        sets.append(d)
    stream = torch.cuda.current_stream()

    def step(i):
        b = sets[i % nsets]
        moe.combine_backward(b["y"], b["w"], b["d_out"], b["d_y"], b["d_w"])
        moe.act_up_backward(spec.act, b["gate_up"], b["d_h"], b["d_gu"])

    for i in range(max(args.warmup, 3)):
        step(i)
    torch.cuda.synchronize()
    clocks = ClockSampler(torch.cuda.current_device())
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    clocks.start()
    n0 = moe.launch_count()
    ev0.record(stream)
    for i in range(args.steps):
        step(i)
    ev1.record(stream)
    torch.cuda.synchronize()
    n_launch = moe.launch_count() - n0
    clocks.stop()
    ms = ev0.elapsed_time(ev1)
    # per-kernel durations: each kernel alone, back to back over the rotating sets, between one event pair
    # (an event pair around every launch would add the launch gap to these ~10 us kernels)
    one = {"combine_backward": lambda b: moe.combine_backward(b["y"], b["w"], b["d_out"], b["d_y"], b["d_w"]),
           "act_up_backward": lambda b: moe.act_up_backward(spec.act, b["gate_up"], b["d_h"], b["d_gu"])}
    kernels = {}
    for name, fn in one.items():
        for i in range(3):
            fn(sets[i % nsets])
        k0, k1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        k0.record(stream)
        for i in range(args.steps):
            fn(sets[i % nsets])
        k1.record(stream)
        torch.cuda.synchronize()
        t = k0.elapsed_time(k1)
        kernels[name] = {"launches": args.steps, "avg_ms": t / args.steps, "total_ms": t}
    tot = sum(k["total_ms"] for k in kernels.values()) or 1.0
    dom = max(kernels, key=lambda n: kernels[n]["total_ms"])
    peaks, peak_src = _peaks()
    ach = {n: alg[n] / (kernels[n]["avg_ms"] / 1e3) / 1e9 for n in kernels}
    roofline = {"bound": "hbm", "achieved": ach[dom], "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": ach[dom] / peaks["hbm_gbs"], "traffic": _traffic(dom, spec.name + "/backward"), "kernel": dom,
                "algorithmic_bytes_per_launch": alg[dom], "peak_source": f"{peak_src} (hbm_gbs)",
                "per_kernel_frac": {n: ach[n] / peaks["hbm_gbs"] for n in kernels}}
    # end to end: inputs from pinned host memory, both kernels, outputs back, every step
    pin = {k: torch.from_numpy(v).pin_memory() for k, v in hin.items()}
    outs = {"d_y": torch.empty((T, K, H)).pin_memory(), "d_w": torch.empty((T, K)).pin_memory(),
            "d_gu": torch.empty((P, 2 * I)).pin_memory()}
    b = sets[0]

    def e2e_step():
        for k in hin:
            b[k].copy_(pin[k], non_blocking=True)
        moe.combine_backward(b["y"], b["w"], b["d_out"], b["d_y"], b["d_w"])
        moe.act_up_backward(spec.act, b["gate_up"], b["d_h"], b["d_gu"])
        for k in outs:
            outs[k].copy_(b[k], non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    e_steps = max(1, min(args.steps, 50))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    cpu = None
    if rank == 0 and ws_n == 1 and not args.no_cpu_baseline:
        v, info = _time_oracle_backward(spec, hin, budget_s=min(args.cpu_budget, 5.0))
        cpu = {"value": v, "unit": UNIT, "cores": info["cores"], "kind": "oracle", "sample": info["sample"]}
    line = {"metric": BWD_METRIC, "value": job_throughput(1, T, args.steps, ms), "unit": UNIT, "n_gpus": ws_n,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": spec.name + "/backward", "T": T, "K": K, "H": H, "I": I, "act": spec.act,
                       "l2": f"no flush: {nsets} rotating input sets of {set_bytes / 1e6:.0f} MB"},
            "e2e": {"value": job_throughput(1, T, e_steps, e2e_ms), "unit": UNIT,
                    "h2d_bytes_per_step": int(sum(v.nbytes for v in hin.values())),
                    "d2h_bytes_per_step": int(4 * (P * H + P + 2 * P * I))},
            "roofline": roofline, "cpu_baseline": cpu, "gpu_launches": n_launch, "clocks": clocks.summary(),
            "device_status": moe.status_string(moe.last_device_status()),
            "kernels": {n: {"launches": k["launches"], "avg_us": 1e3 * k["avg_ms"],
                            "share": round(k["total_ms"] / tot, 4), "timing": "alone, back to back"}
                        for n, k in kernels.items()}}
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ where the two paths cross
CROSS_T = (1, 2, 4, 8, 16, 32, 48, 64, 96, 128, 192, 256)
CROSS_SHAPES = {  # bf16 layers: the prefill and routed+shared shapes, and the Q8_0-decode shape with bf16 weights
    "prefill_bf16": workloads.Spec(T=max(CROSS_T), H=2048, E=64, I=1024, K=8, name="cross_prefill_bf16"),
    "routed_shared_bf16": workloads.Spec(T=max(CROSS_T), H=2048, E=256, I=512, K=8, shared_I=512, shared_gated=True,
                                         name="cross_routed_shared_bf16"),
    "decode_shape_bf16": workloads.Spec(T=max(CROSS_T), H=2048, E=128, I=768, K=8, name="cross_decode_shape_bf16"),
}


def run_crossover(args):
    """--op crossover: one bf16 layer call per step on the weight-streaming path (the fused decode kernel up to
    64 tokens, the step-by-step streaming launches beyond) and on the tensor-core path, for each batch size in
    CROSS_T, over 8 rotating token batches (weights of every shape exceed L2).  Prints the table as one JSON line;
    the fastest path per size is where moe_layer's default threshold should sit."""
    import dataclasses

    import torch
    import mixture_experts_ffn_07_b200 as moe
    from mixture_experts_ffn_07_b200 import host
    ws_n, rank, local = _dist()
    if rank != 0:
        return 0
    torch.cuda.set_device(local)
    stream = torch.cuda.current_stream()
    table = {}
    for shape, spec in CROSS_SHAPES.items():
        wl = workloads.make(spec)
        desc0, w, x0 = host.upload(wl)
        xs = [x0] + [host.to_device(workloads.token_batch(spec, i), "bf16") for i in range(1, NROT)]
        rows = {}
        for T in CROSS_T:
            desc = dataclasses.replace(desc0, T=T)
            res = {}
            for path, thr in (("streaming", 10 ** 9), ("tensor", 1)):
                moe.set_tensor_min_tokens(thr)
                try:
                    out = torch.empty((T, spec.H), dtype=torch.bfloat16, device="cuda")
                    wsb = torch.empty(moe.workspace_bytes(desc), dtype=torch.uint8, device="cuda")
                    xb = [xx[:T] for xx in xs]
                    for i in range(max(args.warmup, 3)):
                        moe.layer(desc, xb[i % NROT], w, out, wsb)
                    n = max(10, min(args.steps, 200))
                    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    torch.cuda.synchronize()
                    a.record(stream)
                    for i in range(n):
                        moe.layer(desc, xb[i % NROT], w, out, wsb)
                    b.record(stream)
                    torch.cuda.synchronize()
                    res[path] = 1e3 * a.elapsed_time(b) / n
                finally:
                    moe.set_tensor_min_tokens(65)
            assert moe.last_device_status() == moe.MOE_OK
            res["faster"] = min(("streaming", "tensor"), key=lambda k: res[k])
            rows[T] = res
        table[shape] = rows
        del w, xs
        torch.cuda.empty_cache()
    print(json.dumps({"op": "crossover", "unit": "us per layer call", "tokens": list(CROSS_T), "table": table}),
          flush=True)
    return 0


def spawn_ranks(n: int) -> int:
    """Runs this command again as n ranks on this node (torch.distributed.run, rendezvous on 127.0.0.1)
    and returns its exit status."""
    import socket
    with socket.socket() as so:
        so.bind(("127.0.0.1", 0))
        port = so.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__), *sys.argv[1:]]
    return subprocess.call(cmd)


def dist_selftest(args) -> int:
    """The multi-rank plumbing without a GPU: each rank reports a time that depends on its rank, the job
    takes the largest, and rank 0 prints the line the GPU bench would print for it."""
    import datetime

    import torch.distributed as dist
    ws, rank, _ = _dist()
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        ms = max_over_ranks(dist, 10.0 + rank, "cpu")
        if rank == 0:
            print(json.dumps({"selftest": True, "n_gpus": ws, "ms": ms,
                              "value": job_throughput(ws, 1, args.steps, ms)}), flush=True)
        dist.barrier()
    finally:
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", default=DEFAULT_CONFIG, choices=workloads.CONFIG_ORDER)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=10.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--op", default="layer", choices=["layer", "backward", "crossover"],
                    help="backward: the combine and act*up backward kernels on the workload's slots; "
                         "crossover: both paths of bf16 layers over batch sizes 8..256")
    ap.add_argument("--pair-gemm", type=int, default=1, choices=[0, 1],
                    help="0: compute-bound expert GEMMs on single CTAs only (moe_set_pair_gemm), for comparison")
    ap.add_argument("--decode-stream", type=int, default=1, choices=[0, 1],
                    help="0: the decode kernel's gate/up and down as two phases for every format "
                         "(moe_set_decode_stream), for comparison")
    ap.add_argument("--dist-selftest", action="store_true",
                    help="ranks only: gloo process group, max over ranks of a rank-dependent time, no GPU work")
    args = ap.parse_args()
    ws = int(os.environ.get("WORLD_SIZE", "0"))
    if args.gpus > 1 and ws == 0:
        return spawn_ranks(args.gpus)
    if ws and ws != args.gpus:
        print(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={ws}", file=sys.stderr)
        return 2
    if args.dist_selftest:
        return dist_selftest(args)
    spec = workloads.CONFIGS[args.config]
    if args.op == "crossover":
        return run_crossover(args)
    if args.op == "backward":
        return run_backward(args, spec)
    if args.impl == "reference":
        return run_reference(args, spec)
    return run_ours(args, spec)


if __name__ == "__main__":
    sys.exit(main())
