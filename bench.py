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
# kernels of one moe_forward: route, group + permute, gate/up GEMM, down GEMM, combine
KERNELS_PER_LAYER = 5
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


def workload_config(name: str, T: int):
    cfg = CONFIGS[name]
    c = {"workload": DESCRIPTIONS[name], "name": name, "T": T, "d_model": cfg.d, "d_ff": cfg.F, "experts": cfg.E,
         "top_k": cfg.k, "layers": cfg.layers, "seed": cfg.seed, "weights": "MXFP4 (E2M1 codes + E8M0 per 32)",
         "mma": "tcgen05 kind::mxf8f6f4 block-scaled: E2M1 weight codes (E8M0 per 32) straight from TMA x "
                "activations as two E4M3 terms (E8M0 per 32) -> fp32 in TMEM"}
    return c


# ----------------------------------------------------------------- CPU oracle

def oracle_tokens_per_s(inp, cfg, n_tokens: int, threads: int):
    """The CPU oracle as it stands on a bounded sample of the workload's tokens."""
    import oracle
    x = inp["x"][:n_tokens]
    t0 = time.perf_counter()
    oracle.moe_forward(inp, cfg.k, cfg.eps, x=x, threads=threads)
    dt = time.perf_counter() - t0
    return n_tokens / dt, dt


def run_reference(args, rank, world):
    """Reference arm: the CPU oracle, timed on the host cores (rank 0 only)."""
    if rank != 0:
        return 0
    import oracle
    cfg = CONFIGS[args.workload]
    inp = make_config_inputs(cfg) if cfg.layers == 1 else dict(make_config_inputs(cfg, 0), x=make_tokens(
        np.random.Generator(np.random.PCG64(cfg.seed)), cfg.T, cfg.d))
    threads = oracle.max_threads()
    n = min(cfg.T, max(1, threads))                 # one token per core per step
    for _ in range(args.warmup if args.warmup <= 1 else 1):
        oracle_tokens_per_s(inp, cfg, min(n, 2), threads)
    total_t = 0.0
    for _ in range(args.steps):
        _, dt = oracle_tokens_per_s(inp, cfg, n, threads)
        total_t += dt
    # a step of the workload is T tokens; the reference processes n per timed step
    per_token = total_t / (args.steps * n)
    value = 1.0 / per_token / max(cfg.layers, 1)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_token * cfg.T * cfg.layers * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(args.workload, cfg.T),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                             "sample": "%d of the workload's %d tokens per step (layer 0)" % (n, cfg.T)},
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
    router plus 2*(2F*d + d*F) per routed (token, expert) pair.
    """
    T, d, F, E, k = cfg.T, cfg.d, cfg.F, cfg.E, cfg.k
    touched = int(np.count_nonzero(counts))
    w13_expert = 2 * F * (d // 2) + 2 * F * (d // 32) + 2 * F * 2
    w2_expert = d * (F // 2) + d * (F // 32) + d * 2
    pairs = T * k
    bytes_up = touched * w13_expert + T * d * 2 + pairs * F * 2          # weights, xn16 in, h out
    bytes_down = touched * w2_expert + pairs * F * 2 + pairs * d * 4      # weights, h in, weighted rows out
    flops_up = pairs * 2 * (2 * F) * d
    flops_down = pairs * 2 * d * F
    layer_bytes = touched * (w13_expert + w2_expert) + E * d * 2 + E * 4 + d * 2 + T * d * 2 * 2
    layer_flops = 2 * T * d * E + flops_up + flops_down
    return dict(touched=touched, bytes_up=bytes_up, bytes_down=bytes_down, flops_up=flops_up,
                flops_down=flops_down, layer_bytes=layer_bytes, layer_flops=layer_flops,
                w13_expert=w13_expert, w2_expert=w2_expert)


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    import sparse_moe_rmsnorm_b200 as moe

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    cfg = CONFIGS[args.workload]
    T = cfg.T
    layers = cfg.layers
    # the weights (identical on every rank) and this rank's token batch
    if layers == 1:
        inp = make_config_inputs(cfg)
        layer_inputs = [inp]
    else:
        layer_inputs = [make_config_inputs(cfg, l) for l in range(layers)]
    x_np = replica_tokens(cfg, rank)
    weights = [moe.MoEWeights.from_numpy(li, device=dev) for li in layer_inputs]
    x = torch.from_numpy(x_np.view(np.int16)).view(torch.bfloat16).to(dev)
    m = moe.MoE(T, cfg.d, cfg.F, cfg.E, cfg.k, cfg.eps)
    bufs = [torch.empty_like(x) for _ in range(2)]
    stream = torch.cuda.current_stream()

    # events around the gate/up GEMM (the dominant kernel) of every layer of every timed step
    up_events = []

    def step(timed=False):
        """One step: the block on every layer.  timed=False: moe_forward (the public call);
        timed=True: the five stage calls moe_forward is made of, with the gate/up GEMM
        bracketed by events on the launching stream."""
        cur = x
        for l, w in enumerate(weights):
            out = bufs[l % 2]
            if not timed:
                m.forward(cur, w, y=out)
                cur = out
                continue
            moe.moe_route(m.ctx, T, cur, w.norm_scale, w.router_w, w.router_b, cfg.k)
            moe.moe_group(m.ctx, T, cfg.k)
            if timed:
                ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                ea.record(stream)
            moe.moe_expert_up(m.ctx, T, cfg.k, w.w13_codes, w.w13_scales, w.b13)
            if timed:
                eb.record(stream)
                up_events.append((ea, eb))
            moe.moe_expert_down(m.ctx, T, cfg.k, w.w2_codes, w.w2_scales, w.b2)
            moe.moe_finalize(m.ctx, T, cfg.k, cur, out)
            cur = out
        return cur

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if m.sync_status() != moe.MOE_OK:
        raise RuntimeError("device-side error during warm-up")

    # ---- timed region: K steps, device events, barrier + sync on both sides
    if world > 1:
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
    # ---- the dominant kernel: K more steps, its launches bracketed by events
    for _ in range(args.steps):
        step(timed=True)
    torch.cuda.synchronize()
    up_ms_live = sum(a.elapsed_time(b) for a, b in up_events) / max(len(up_events), 1)
    ms_per_step = ms_total / args.steps
    value = job_tokens_per_s(ms_total, T, args.steps, world)
    if m.sync_status() != moe.MOE_OK:
        raise RuntimeError("device-side error during the timed region")

    # ---- per-stage times (layer 0) in a separate pass, for the report: events between
    # every kernel, so each stage is timed alone
    w0 = weights[0]
    stage_ms = {k_: 0.0 for k_ in ("route", "group", "up", "down", "finalize")}
    reps = max(3, min(args.steps, 20))
    y0 = bufs[0]
    for _ in range(reps):
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
        evs[0].record(stream)
        moe.moe_route(m.ctx, T, x, w0.norm_scale, w0.router_w, w0.router_b, cfg.k)
        evs[1].record(stream)
        moe.moe_group(m.ctx, T, cfg.k)
        evs[2].record(stream)
        moe.moe_expert_up(m.ctx, T, cfg.k, w0.w13_codes, w0.w13_scales, w0.b13)
        evs[3].record(stream)
        moe.moe_expert_down(m.ctx, T, cfg.k, w0.w2_codes, w0.w2_scales, w0.b2)
        evs[4].record(stream)
        moe.moe_finalize(m.ctx, T, cfg.k, x, y0)
        evs[5].record(stream)
        torch.cuda.synchronize()
        for i, k_ in enumerate(stage_ms):
            stage_ms[k_] += evs[i].elapsed_time(evs[i + 1]) / reps
    counts = m.workspace("counts", T).cpu().numpy()
    cnt = algorithmic_counts(cfg, counts)

    # ---- end to end through the public API: pinned host x in, y out, every step
    x_host = torch.from_numpy(x_np.view(np.int16)).view(torch.bfloat16).pin_memory()
    y_host = torch.empty_like(x_host).pin_memory()
    x_dev = torch.empty_like(x)
    for _ in range(max(1, args.warmup)):
        m.forward_host(x_host, w0, y_host, x_dev, bufs[0])
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        if layers == 1:
            m.forward_host(x_host, w0, y_host, x_dev, bufs[0])
        else:
            x_dev.copy_(x_host, non_blocking=True)
            cur = x_dev
            for l, w in enumerate(weights):
                out = bufs[l % 2]
                m.forward(cur, w, y=out)
                cur = out
            y_host.copy_(cur, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    e2e_value = job_tokens_per_s(e2e_ms, T, args.steps, world)

    if rank != 0:
        m.close()
        return 0

    peaks = measured_peaks()
    # dominant kernel and its roofline
    # the dominant kernel: the gate/up GEMM (2/3 of the weights and of the flops), timed live
    dom = "up"
    t_dom = up_ms_live / 1e3
    tensor_bound = cfg.T * cfg.k >= 4096
    key = "expert_%s_%s" % (dom, args.workload)
    if tensor_bound:
        flops = cnt["flops_" + dom]
        achieved = flops / t_dom / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": achieved / peaks["bf16_tflops"], "traffic": committed_traffic(key),
                "kernel": "expert_gemm_kernel<%s>" % dom, "algorithmic_flops_per_launch": flops,
                "peak_source": peaks["source"] + " bf16 dense (the roofline the block is specified against; the "
                               "fp8-kind MMAs run two activation terms per product, the same tensor time as bf16)"}
    else:
        byts = cnt["bytes_" + dom]
        achieved = byts / t_dom / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "traffic": committed_traffic(key),
                "kernel": "expert_gemm_kernel<%s>" % dom, "algorithmic_bytes_per_launch": byts,
                "peak_source": peaks["source"] + " HBM copy"}
    t_layer_roof = max(cnt["layer_flops"] / (peaks["bf16_tflops"] * 1e12), cnt["layer_bytes"] / (peaks["hbm_gbs"] * 1e9))
    layer_ms = ms_per_step / layers

    # CPU oracle baseline on a bounded sample (rank 0, N = 1 only)
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        import oracle
        threads = oracle.max_threads()
        n = min(T, max(1, threads))
        tps, dt = oracle_tokens_per_s(layer_inputs[0] if layers == 1 else dict(layer_inputs[0], x=x_np), cfg, n,
                                      threads)
        cpu = {"value": tps / layers, "unit": "tokens/s", "cores": threads, "kind": "oracle",
               "sample": "%d tokens of the workload through %s (%.1f s)" % (
                   n, "the layer" if layers == 1 else "layer 0 (value divided by %d layers)" % layers, dt)}

    config = workload_config(args.workload, T)
    config.update({"parallelism": "replicas (dp%d, no collective)" % world, "global_batch": T * world,
                   "l2": "inputs larger than L2: %.0f MB of touched expert weights per layer step vs %d MB L2" % (
                       (cnt["touched"] * (cnt["w13_expert"] + cnt["w2_expert"])) / 1e6, L2_BYTES // 2 ** 20),
                   "stage_ms": {k_: round(v, 4) for k_, v in stage_ms.items()},
                   "up_ms_live": round(up_ms_live, 4),
                   "experts_touched": cnt["touched"],
                   "layer_roofline": {"t_roof_us": t_layer_roof * 1e6, "t_us": layer_ms * 1e3,
                                      "frac": t_layer_roof / (layer_ms / 1e3),
                                      "bytes": cnt["layer_bytes"], "flops": cnt["layer_flops"]},
                   "kernel_src_sha": kernel_source_hash()})
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "e2m1xe4m3->f32", "data": "synthetic", "config": config,
            "roofline": roof, "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": T * cfg.d * 2,
                    "d2h_bytes_per_step": T * cfg.d * 2},
            "gpu_launches": KERNELS_PER_LAYER * layers * args.steps, "clocks": clocks.summary()}
    print(json.dumps(line), flush=True)
    m.close()
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="decode20b", choices=sorted(CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
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
