"""Benchmark of the B200 MoE block (gpt-oss MoE feed-forward layer).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one moe_forward over the workload's token batch (RMSNorm, router,
top-k + softmax, grouping, gate/up GEMM + SwiGLU, down GEMM + weighted
combine, bf16 output) with every input already resident in HBM.  Prints ONE
JSON line.  Under torchrun (N > 1) every rank runs an independent replica on
its own GPU (the block does not shard; there is no collective on the data
path); the time is the max over ranks and the value counts every rank's
tokens.

Workloads (seeded synthetic inputs, ``moe_inputs``): decode20b (default),
prefill20b, decode120b, stack20b (24 layers), tiny.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from moe_inputs import CONFIGS, make_config_inputs, make_tokens  # noqa: E402

L2_BYTES = 126 * 2 ** 20
# kernels of one moe_forward: route, group + permute, gate/up GEMM, down GEMM, combine; batches over
# 64 tokens add the pass plan before the gate/up GEMM, and over 2048 pairs the grouping and the
# tokens' encoding are two kernels
def kernels_per_layer(T: int, k: int = 4, d: int = 2880, F: int = 2880) -> int:
    """The library's launches per layer step of moe_forward: route + group (one launch for
    decode-sized batches), the pass plan (above 64 tokens), the token encoder (above 2048
    pairs), the two GEMMs (one launch for decode-sized batches with d_model == d_ff) and the
    combine."""
    if T <= 64 and d <= 3072:
        return 3 if d == F else 4
    n = 5 if T <= 64 else 6
    return n + 1 if T * k > 2048 else n
METRIC = "MoE-layer tokens/s (decode & prefill) and % of HBM / bf16 tensor roofline"
DESCRIPTIONS = {
    "tiny": "tiny MoE layer: T=16, d_model=d_ff=128, E=8, top-4",
    "decode20b": "gpt-oss-20b-shaped MoE layer, decode: T=32, d_model=d_ff=2880, E=32, top-4",
    "prefill20b": "gpt-oss-20b-shaped MoE layer, prefill: T=8192, d_model=d_ff=2880, E=32, top-4",
    "decode120b": "gpt-oss-120b-shaped MoE layer, decode: T=64, d_model=d_ff=2880, E=128, top-4",
    "stack20b": "24 gpt-oss-20b-shaped MoE blocks, T=2048, E=32, top-4, Zipf(1.1)-skewed routing",
}
KERNEL_SOURCES = ["sparse_moe_rmsnorm_b200/csrc/expert_gemm.cu", "sparse_moe_rmsnorm_b200/csrc/ptx.cuh",
                  "sparse_moe_rmsnorm_b200/csrc/kernels.cuh", "sparse_moe_rmsnorm_b200/csrc/route_group.cu"]


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for p in KERNEL_SOURCES:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            pk = json.load(f)
        return {"hbm_gbs": pk["hbm_gbs"], "bf16_tflops": pk["bf16_tflops"],
                "bf16_tflops_sustained": pk.get("bf16_tflops_sustained", pk["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def committed_traffic(key: str):
    """DRAM bytes per launch from the committed ncu summary, if the kernel is unchanged since."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        tab = json.load(f)
    ent = tab.get(key)
    if not ent or ent.get("kernel_src_sha") != kernel_source_hash():
        return None
    return ent.get("dram_bytes_per_launch")


class ClockSampler:
    """SM clocks and clock-event (throttle) reasons sampled while running (read only).

    NVML is polled from a thread every millisecond, so that even a timed region
    of a few milliseconds gets samples; nvidia-smi (every 200 ms) is the fallback
    when NVML is unavailable."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.samples = []          # (sm_mhz, sm_max_mhz, [reason names])
        self.proc = None
        self.thread = None
        self.nvml = None
        self.handle = None

    def _nvml_handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        props = torch.cuda.get_device_properties(self.gpu)
        try:
            bus = "%08X:%02X:%02X.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
            return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.gpu)

    def _sample(self):
        nv, h = self.nvml, self.handle
        try:
            sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
            r = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
            self.samples.append((float(sm), float(self.max_mhz),
                                 [n for n, attr in self.REASONS if getattr(nv, attr, 0) and (r & getattr(nv, attr))]))
        except Exception:
            pass

    def _poll(self):
        while not self.stop.is_set():
            self._sample()
            self.stop.wait(0.001)

    def __enter__(self):
        import threading
        try:
            self.nvml, self.handle = self._nvml_handle()
            self.max_mhz = self.nvml.nvmlDeviceGetMaxClockInfo(self.handle, self.nvml.NVML_CLOCK_SM)
            self.stop = threading.Event()
            self._sample()           # one reading as the timed region starts, one as it ends
            self.thread = threading.Thread(target=self._poll, daemon=True)
            self.thread.start()
            return self
        except Exception:
            self.nvml = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.thread is not None:
            self.stop.set()
            self.thread.join(timeout=5)
            self._sample()
            return False
        if self.proc is None:
            return False
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        names = [n for n, _ in self.REASONS]
        for line in out.splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9 and parts[1].replace(".", "").isdigit():
                self.samples.append((float(parts[1]), float(parts[2]),
                                     [names[i] for i in range(4) if parts[5 + i].lower() == "active"]))
        return False

    def summary(self):
        s = self.samples
        if not s:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": statistics.median(x[0] for x in s), "sm_max_mhz": max(x[1] for x in s),
                "reasons": sorted({r for x in s for r in x[2]}), "samples": len(s),
                "source": "nvml" if self.thread is not None else "nvidia-smi"}


def workload_config(name: str, world: int = 1):
    """The static description of a workload: identical for both arms of the bench."""
    cfg = CONFIGS[name]
    w_expert = 2 * cfg.F * (cfg.d // 2 + cfg.d // 32 + 2) + cfg.d * (cfg.F // 2 + cfg.F // 32 + 2)
    return {"workload": DESCRIPTIONS[name], "name": name, "T": cfg.T, "d_model": cfg.d, "d_ff": cfg.F,
            "experts": cfg.E, "top_k": cfg.k, "layers": cfg.layers, "seed": cfg.seed,
            "weights": "MXFP4 (E2M1 codes + E8M0 per 32)",
            "mma": "tcgen05 kind::mxf8f6f4 block-scaled: E2M1 weight codes (E8M0 per 32) straight from TMA x "
                   "activations as E4M3 terms (E8M0 per 32) -> fp32 in TMEM",
            "parallelism": "replicas (dp%d, no collective)" % world, "global_batch": cfg.T * world,
            "l2": "inputs larger than L2: a layer step streams the touched experts' MXFP4 weights (up to %.0f MB "
                  "per layer) vs a %d MB L2; no flush" % (cfg.E * w_expert / 1e6, L2_BYTES // 2 ** 20)}


def layer_inputs_of(cfg, layer: int, x=None):
    """One layer's inputs (a stack's layer l takes the stack's tokens)."""
    if cfg.layers == 1:
        return make_config_inputs(cfg)
    inp = make_config_inputs(cfg, layer)
    inp["x"] = x if x is not None else make_tokens(np.random.Generator(np.random.PCG64(cfg.seed)), cfg.T, cfg.d)
    return inp


# ----------------------------------------------------------------- CPU oracle

def oracle_tokens_per_s(inp, cfg, n_tokens: int, threads: int):
    """The CPU oracle as it stands on a bounded sample of the workload's tokens."""
    import oracle
    x = inp["x"][:n_tokens]
    t0 = time.perf_counter()
    oracle.moe_forward(inp, cfg.k, cfg.eps, x=x, threads=threads)
    dt = time.perf_counter() - t0
    return n_tokens / dt, dt


# tokens of a workload one reference (oracle) step processes: the whole batch of
# the decode workloads, a 64-token sample of the larger ones, always through one layer
REFERENCE_TOKENS_MAX = 64
# single-thread oracle runs reported beside the reference line: (workload, tokens)
SINGLE_THREAD_RUNS = (("tiny", 16), ("decode20b", 4), ("decode120b", 4))


def single_thread_baselines():
    out = []
    for name, n in SINGLE_THREAD_RUNS:
        cfg = CONFIGS[name]
        inp = layer_inputs_of(cfg, 0)
        tps, dt = oracle_tokens_per_s(inp, cfg, n, 1)
        out.append({"workload": name, "value": tps, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                    "sample": "%d of the workload's %d tokens through one layer (%.1f s)" % (n, cfg.T, dt)})
    return out


def run_reference(args, rank, world):
    """Reference arm: the CPU oracle, timed on the host cores (rank 0 only).

    Each step runs min(T, 64) of the workload's tokens through one layer (all of
    a decode batch); ms_per_step is the time of exactly that work, and the
    value is tokens per second per layer (divided by the layer count for a
    stack)."""
    if rank != 0:
        return 0
    import oracle
    cfg = CONFIGS[args.workload]
    inp = layer_inputs_of(cfg, 0)
    threads = oracle.max_threads()
    n = min(cfg.T, REFERENCE_TOKENS_MAX)
    for _ in range(min(args.warmup, 1)):
        oracle_tokens_per_s(inp, cfg, min(n, 2), threads)
    total_t = 0.0
    for _ in range(args.steps):
        _, dt = oracle_tokens_per_s(inp, cfg, n, threads)
        total_t += dt
    value = args.steps * n / total_t / cfg.layers
    sample = "%d of the workload's %d tokens through %s per step" % (
        n, cfg.T, "the layer" if cfg.layers == 1 else "layer 0 (value divided by %d layers)" % cfg.layers)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_t / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(args.workload, world),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                             "sample": sample},
            "cpu_baseline_single_thread": single_thread_baselines() if not args.no_cpu_baseline else None,
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------- replica plumbing

def max_over_ranks(ms: float, world: int, device=None) -> float:
    """The slowest rank's time: every rank takes part in the same all-reduce."""
    if world <= 1:
        return float(ms)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(ms_total: float, tokens_per_rank: int, steps: int, world: int) -> float:
    """Whole-job throughput: the tokens every replica processed over the slowest rank's time."""
    return world * tokens_per_rank * steps / (ms_total / 1e3)


def replica_tokens(cfg, rank: int):
    """Rank r's token batch: rank 0 uses the workload's own tokens, other ranks their own seed."""
    seed = cfg.seed if rank == 0 else cfg.seed + 1000 * rank
    return make_tokens(np.random.Generator(np.random.PCG64(seed)), cfg.T, cfg.d)


# ------------------------------------------------------------------ GPU arm

def algorithmic_counts(cfg, counts):
    """Algorithmic bytes and FLOPs of one layer step, from the actual routing.

    Bytes: the touched experts' codes + scales + biases, router weights and
    bias, RMSNorm scale, x read and y written (bf16).  FLOPs: 2*T*d*E for the
    router plus 2*(2F*d + d*F) per routed (token, expert) pair.  Per GEMM: its
    touched experts' weights, its activation rows in (bf16-sized: 2 bytes per
    element) and its output rows (h at 2 bytes, the weighted rows at 4).
    """
    T, d, F, E, k = cfg.T, cfg.d, cfg.F, cfg.E, cfg.k
    touched = int(np.count_nonzero(counts))
    w13_expert = 2 * F * (d // 2) + 2 * F * (d // 32) + 2 * F * 2
    w2_expert = d * (F // 2) + d * (F // 32) + d * 2
    pairs = T * k
    bytes_up = touched * w13_expert + T * d * 2 + pairs * F * 2          # weights, xn in, h out
    bytes_down = touched * w2_expert + pairs * F * 2 + pairs * d * 4      # weights, h in, weighted rows out
    flops_up = pairs * 2 * (2 * F) * d
    flops_down = pairs * 2 * d * F
    layer_bytes = touched * (w13_expert + w2_expert) + E * d * 2 + E * 4 + d * 2 + T * d * 2 * 2
    layer_flops = 2 * T * d * E + flops_up + flops_down
    return dict(touched=touched, bytes_up=bytes_up, bytes_down=bytes_down, flops_up=flops_up,
                flops_down=flops_down, bytes_ffn=bytes_up + bytes_down, flops_ffn=flops_up + flops_down,
                layer_bytes=layer_bytes, layer_flops=layer_flops, w13_expert=w13_expert, w2_expert=w2_expert)


def gemm_roofline(which, t_s, cnt, tensor_bound, peaks, peak_key, workload):
    """Roofline of one grouped GEMM launch from its live event time t_s (seconds)."""
    key = "expert_%s_%s" % (which, workload)
    if tensor_bound:
        flops = cnt["flops_" + which]
        achieved = flops / t_s / 1e12
        peak = peaks[peak_key]
        return {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                "traffic": committed_traffic(key), "kernel": "expert_gemm_kernel<%s>" % which,
                "algorithmic_flops_per_launch": flops,
                "peak_source": "%s bf16 dense%s (the roofline the block is specified against)" % (
                    peaks["source"], ", sustained" if peak_key.endswith("sustained") else ", burst")}
    byts = cnt["bytes_" + which]
    achieved = byts / t_s / 1e9
    return {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / peaks["hbm_gbs"], "traffic": committed_traffic(key),
            "kernel": "expert_gemm_kernel<%s>" % which, "algorithmic_bytes_per_launch": byts,
            "peak_source": peaks["source"] + " HBM copy"}


def measure_workload(name, args, rank, world, local_rank, main):
    """Time one workload: K steps of moe_forward (the value), then K steps of the stage calls
    with the GEMM launches bracketed by events, per-stage times, and (main line only) the end-to-end
    number and the CPU oracle sample.  Returns the measurements (rank 0) or None."""
    import torch
    import sparse_moe_rmsnorm_b200 as moe

    dev = torch.device("cuda", local_rank)
    cfg = CONFIGS[name]
    T, layers = cfg.T, cfg.layers
    x_np = replica_tokens(cfg, rank)
    # the weights (identical on every rank), made and uploaded one layer at a time
    weights = []
    first_inputs = None
    for l in range(layers):
        li = layer_inputs_of(cfg, l, x=x_np)
        if l == 0:
            first_inputs = li
        weights.append(moe.MoEWeights.from_numpy(li, device=dev))
    x = torch.from_numpy(x_np.view(np.int16)).view(torch.bfloat16).to(dev)
    m = moe.MoE(T, cfg.d, cfg.F, cfg.E, cfg.k, cfg.eps)
    bufs = [torch.empty_like(x) for _ in range(2)]
    stream = torch.cuda.current_stream()
    # moe_forward runs both GEMMs of a decode-sized batch as one launch (moe_expert_ffn)
    fused = T <= 64 and T * cfg.k <= 512 and cfg.d <= 3072 and cfg.d == cfg.F
    gemm_events = {"up": [], "down": [], "ffn": []}

    def step(timed=False):
        """One step: the block on every layer.  timed=False: moe_forward (the public call);
        timed=True: the stage calls moe_forward is made of, with the GEMM launches bracketed
        by events on the launching stream."""
        cur = x
        for l, w in enumerate(weights):
            out = bufs[l % 2]
            if not timed:
                m.forward(cur, w, y=out)
                cur = out
                continue
            moe.moe_route(m.ctx, T, cur, w.norm_scale, w.router_w, w.router_b, cfg.k)
            moe.moe_group(m.ctx, T, cfg.k)
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
            ev[0].record(stream)
            if fused:
                # decode-sized: both GEMMs in one launch, as moe_forward runs them
                moe.moe_expert_ffn(m.ctx, T, cfg.k, w.w13_codes, w.w13_scales, w.b13, w.w2_codes, w.w2_scales, w.b2)
                ev[1].record(stream)
                gemm_events["ffn"].append((ev[0], ev[1]))
            else:
                moe.moe_expert_up(m.ctx, T, cfg.k, w.w13_codes, w.w13_scales, w.b13, w.w2_scales)
                ev[1].record(stream)
                moe.moe_expert_down(m.ctx, T, cfg.k, w.w2_codes, w.w2_scales, w.b2)
                ev[2].record(stream)
                gemm_events["up"].append((ev[0], ev[1]))
                gemm_events["down"].append((ev[1], ev[2]))
            moe.moe_finalize(m.ctx, T, cfg.k, cur, out)
            cur = out
        return cur

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if m.sync_status() != moe.MOE_OK:
        raise RuntimeError("device-side error during warm-up (%s)" % name)

    # ---- timed region: K steps, device events, barrier + sync on both sides
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clocks:
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms_total = max_over_ranks(ev0.elapsed_time(ev1), world, dev)
    # ---- the GEMMs: K more steps, their launches bracketed by events
    for _ in range(args.steps):
        step(timed=True)
    torch.cuda.synchronize()
    gemm_ms = {k_: sum(a.elapsed_time(b) for a, b in v) / max(len(v), 1) for k_, v in gemm_events.items() if v}
    ms_per_step = ms_total / args.steps
    value = job_tokens_per_s(ms_total, T, args.steps, world)
    if m.sync_status() != moe.MOE_OK:
        raise RuntimeError("device-side error during the timed region (%s)" % name)

    # ---- per-stage times (layer 0) in a separate pass, for the report: events between
    # every kernel, so each stage is timed alone
    w0 = weights[0]
    stage_ms = {k_: 0.0 for k_ in ("route", "group", "up", "down", "finalize")}
    reps = max(3, min(args.steps, 20))
    y0 = bufs[0]
    for rep in range(reps + 1):     # (an untimed first pass loads the kernels moe_forward does not use)
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
        evs[0].record(stream)
        moe.moe_route(m.ctx, T, x, w0.norm_scale, w0.router_w, w0.router_b, cfg.k)
        evs[1].record(stream)
        moe.moe_group(m.ctx, T, cfg.k)
        evs[2].record(stream)
        moe.moe_expert_up(m.ctx, T, cfg.k, w0.w13_codes, w0.w13_scales, w0.b13, w0.w2_scales)
        evs[3].record(stream)
        moe.moe_expert_down(m.ctx, T, cfg.k, w0.w2_codes, w0.w2_scales, w0.b2)
        evs[4].record(stream)
        moe.moe_finalize(m.ctx, T, cfg.k, x, y0)
        evs[5].record(stream)
        torch.cuda.synchronize()
        if rep == 0:
            continue
        for i, k_ in enumerate(stage_ms):
            stage_ms[k_] += evs[i].elapsed_time(evs[i + 1]) / reps
    counts = m.workspace("counts", T).cpu().numpy()
    cnt = algorithmic_counts(cfg, counts)

    # ---- end to end through the public API: every step copies its tokens in from pinned host
    # memory, runs the block on every layer (moe_forward) and copies the result back.  As a serving
    # loop would, the copies run on two copy streams against double-buffered device tokens, so a
    # step's copies overlap the compute of the steps around it; events order each buffer's reuse.
    e2e = None
    if main:
        x_host = torch.from_numpy(x_np.view(np.int16)).view(torch.bfloat16).pin_memory()
        y_host = torch.empty_like(x_host).pin_memory()
        h2d_s, d2h_s = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        xd = [torch.empty_like(x) for _ in range(2)]
        yd = [torch.empty_like(x) for _ in range(2)]
        ev = {k_: [torch.cuda.Event() for _ in range(2)] for k_ in ("h2d", "fwd", "d2h")}

        def e2e_step(i):
            b = i % 2
            with torch.cuda.stream(h2d_s):
                h2d_s.wait_event(ev["fwd"][b])          # the step before last has read xd[b]
                xd[b].copy_(x_host, non_blocking=True)
                ev["h2d"][b].record(h2d_s)
            stream.wait_event(ev["h2d"][b])
            stream.wait_event(ev["d2h"][b])             # ... and its result has left yd[b]
            cur = xd[b]
            for l, w in enumerate(weights):
                out = yd[b] if l == layers - 1 else bufs[l % 2]
                m.forward(cur, w, y=out, stream=stream)
                cur = out
            ev["fwd"][b].record(stream)
            with torch.cuda.stream(d2h_s):
                d2h_s.wait_event(ev["fwd"][b])
                y_host.copy_(yd[b], non_blocking=True)
                ev["d2h"][b].record(d2h_s)
            return b

        for i in range(max(1, args.warmup)):
            e2e_step(i)
        torch.cuda.synchronize()
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        h2d_s.wait_event(e0)
        d2h_s.wait_event(e0)
        for i in range(args.steps):
            last = e2e_step(i)
        stream.wait_event(ev["d2h"][last])               # the last result is on the host
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
        # the host result is the block's output on these tokens, bit for bit
        y_ref = step()
        torch.cuda.synchronize()
        if not torch.equal(y_host, y_ref.cpu()):
            raise RuntimeError("end-to-end result differs from moe_forward's (%s)" % name)
        e2e = {"value": job_tokens_per_s(e2e_ms, T, args.steps, world), "unit": "tokens/s",
               "h2d_bytes_per_step": T * cfg.d * 2, "d2h_bytes_per_step": T * cfg.d * 2}
    m.close()
    del weights
    torch.cuda.empty_cache()
    if rank != 0:
        return None

    peaks = measured_peaks()
    tensor_bound = cfg.T * cfg.k >= 4096
    # a stack runs for seconds at the power cap: its tensor-bound kernels take the sustained peak
    peak_key = "bf16_tflops_sustained" if layers > 1 else "bf16_tflops"
    if fused:
        # the one GEMM launch of the step: both GEMMs' algorithmic bytes over its time; the
        # separate launches' times come from the per-stage pass
        roof_up = gemm_roofline("ffn", gemm_ms["ffn"] / 1e3, cnt, tensor_bound, peaks, peak_key, name)
        roof_down = gemm_roofline("down", stage_ms["down"] / 1e3, cnt, tensor_bound, peaks, peak_key, name)
    else:
        roof_up = gemm_roofline("up", gemm_ms["up"] / 1e3, cnt, tensor_bound, peaks, peak_key, name)
        roof_down = gemm_roofline("down", gemm_ms["down"] / 1e3, cnt, tensor_bound, peaks, peak_key, name)
    tflops_layer = peaks[peak_key] if tensor_bound else peaks["bf16_tflops"]
    t_layer_roof = max(cnt["layer_flops"] / (tflops_layer * 1e12), cnt["layer_bytes"] / (peaks["hbm_gbs"] * 1e9))
    layer_ms = ms_per_step / layers

    cpu = None
    if main and world == 1 and not args.no_cpu_baseline:
        import oracle
        threads = oracle.max_threads()
        n = min(T, REFERENCE_TOKENS_MAX)
        tps, dt = oracle_tokens_per_s(first_inputs, cfg, n, threads)
        cpu = {"value": tps / layers, "unit": "tokens/s", "cores": threads, "kind": "oracle",
               "sample": "%d of the workload's %d tokens through %s (%.1f s)" % (
                   n, T, "the layer" if layers == 1 else "layer 0 (value divided by %d layers)" % layers, dt)}
    return {"value": value, "ms_per_step": ms_per_step, "roofline": roof_up, "roofline_down": roof_down,
            "layer_roofline": {"t_roof_us": t_layer_roof * 1e6, "t_us": layer_ms * 1e3,
                               "frac": t_layer_roof / (layer_ms / 1e3), "bytes": cnt["layer_bytes"],
                               "flops": cnt["layer_flops"]},
            "stage_ms": {k_: round(v, 4) for k_, v in stage_ms.items()},
            "gemm_ms_live": {k_: round(v, 4) for k_, v in gemm_ms.items()},
            "experts_touched": cnt["touched"], "clocks": clocks.summary(), "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": kernels_per_layer(T, cfg.k, cfg.d, cfg.F) * layers * args.steps}


EXTRA_WORKLOADS = ("prefill20b", "decode120b", "stack20b")


def run_ours(args, rank, world, local_rank):
    import torch

    torch.cuda.set_device(local_rank)
    main = measure_workload(args.workload, args, rank, world, local_rank, main=True)
    # the other full-size workloads, one GPU only: each with its own timed region and clocks
    extra = {}
    if world == 1 and not args.single and args.workload == "decode20b":
        for name in EXTRA_WORKLOADS:
            r = measure_workload(name, args, rank, world, local_rank, main=False)
            extra[name] = {"config": workload_config(name, world), "value": r["value"], "unit": "tokens/s",
                           "ms_per_step": r["ms_per_step"], "roofline": r["roofline"],
                           "roofline_down": r["roofline_down"], "layer_roofline": r["layer_roofline"],
                           "stage_ms": r["stage_ms"], "gemm_ms_live": r["gemm_ms_live"],
                           "experts_touched": r["experts_touched"], "clocks": r["clocks"],
                           "gpu_launches": r["gpu_launches"]}
    if rank != 0:
        return 0
    line = {"metric": METRIC, "value": main["value"], "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": main["ms_per_step"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "e2m1xe4m3->f32", "data": "synthetic",
            "config": workload_config(args.workload, world), "roofline": main["roofline"],
            "cpu_baseline": main["cpu_baseline"], "e2e": main["e2e"], "gpu_launches": main["gpu_launches"],
            "clocks": main["clocks"],
            "detail": {"roofline_down": main["roofline_down"], "layer_roofline": main["layer_roofline"],
                       "stage_ms": main["stage_ms"], "gemm_ms_live": main["gemm_ms_live"],
                       "experts_touched": main["experts_touched"], "kernel_src_sha": kernel_source_hash()}}
    if extra:
        line["workloads"] = extra
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="decode20b", choices=sorted(CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--single", action="store_true", help="time only --workload (no workloads object)")
    args = ap.parse_args(argv)
    if args.warmup < 3 and args.impl == "ours":
        print("note: fewer than 3 warm-up steps", file=sys.stderr)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        return run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
