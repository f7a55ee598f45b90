#!/usr/bin/env python
"""Throughput of the top-8-of-128 MoE FFN layer on a 256-token canvas.

One step = one moe_forward (router -> plan -> gather -> expert GEMMs ->
combine) over one canvas of T=256 tokens, d=2816, 128 experts, top-8,
f=704, bf16 weights (synthetic, seeded; inputs resident in HBM).  The metric
is canvas tokens/s per MoE layer; the JSON line also carries the expert
kernel's HBM roofline fraction, an end-to-end figure through
moe_forward_host (host buffers, copies inside the timed region) and the CPU
oracle timed on a bounded sample.  The same line also carries, under their
own keys, the other workloads measured in the same run: "encode" (the T=2048
prompt+canvas layer, graded on its tensor-core fraction), "stack30" (the
30-layer denoising step), "canvas4" / "canvas8" / "canvas4f" (the canvas
layer with int4, fp8 and fp4 expert weights) and "lmhead" (the lm_head step
with entropy-bounded acceptance), each with its own step time, per-kernel
times, roofline fractions and clock record.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload NAME] [--extra NAME,... | --no-extra]

N > 1 runs N independent replicas (one canvas per GPU, no collective on the
data path), launched one process per GPU by torch.distributed.run.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "canvas tokens/s per MoE layer (T=256, bf16) and % of HBM/tensor roofline"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
_CSRC = "block_diffusion_moe_router_b200/csrc/"
# Committed ncu summaries of the expert kernel per workload, and the sources
# whose hash they record: the DRAM traffic is reported only while the kernel
# still hashes to the profiled version.
PROFILES = {
    "canvas": ("expert_kernel_canvas.txt", "expert.cu"),
    "canvas4": ("expert_w4_kernel_canvas4.txt", "expert_w4.cu"),
    "canvas8": ("expert_w8_kernel_canvas8.txt", "expert_w8.cu"),
    "canvas4f": ("expert_w4f_kernel_canvas4f.txt", "expert_w4f.cu"),
}


def expert_sources(workload: str):
    return [_CSRC + PROFILES[workload][1], _CSRC + "expert_common.cuh", _CSRC + "common.cuh"]


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=100)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default="canvas")
    p.add_argument("--sets", type=int, default=0, help="input sets rotated (0: enough to exceed L2)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-pdl", action="store_true", help="plain stream-ordered launches")
    p.add_argument("--y-fp32", action="store_true",
                   help="keep the expert outputs y in fp32 (default bf16)")
    p.add_argument("--router", choices=["auto", "ffma", "tc"], default="auto",
                   help="router path (auto: tensor cores when E <= 128)")
    p.add_argument("--prefetch-mb", type=int, default=None,
                   help="MiB of gate_up weights pulled into L2 during routing")
    p.add_argument("--extra", default="encode,stack30,canvas4,canvas8,canvas4f,lmhead",
                   help="other workloads measured in the same run, reported under their "
                        "own keys of the JSON line")
    p.add_argument("--no-extra", action="store_true", help="measure the main workload only")
    return p.parse_args()


# ---------------------------------------------------------------- helpers


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as fh:
            m = json.load(fh)
        return float(m["hbm_gbs"]), float(m["bf16_tflops"]), float(
            m.get("bf16_tflops_sustained", m["bf16_tflops"])), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


def source_hash(workload: str = "canvas") -> str:
    h = hashlib.sha256()
    for rel in expert_sources(workload):
        with open(os.path.join(ROOT, rel), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str):
    """DRAM bytes per launch of the expert kernel from the workload's committed
    ncu summary, or None if there is none or the kernel changed since."""
    if workload not in PROFILES:
        return None
    try:
        kv = {}
        for line in open(os.path.join(ROOT, "profiles", PROFILES[workload][0])):
            if ":" in line and not line.startswith("#"):
                k, v = line.split(":", 1)
                kv[k.strip()] = v.strip()
        if kv.get("source_sha256_16") != source_hash(workload):
            return None
        return float(kv["dram_bytes_per_launch"])
    except Exception:
        return None


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.period = period_s
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._h = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            try:
                uuid = str(torch.cuda.get_device_properties(device_index).uuid)
                self._h = pynvml.nvmlDeviceGetHandleByUUID(
                    uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            except Exception:
                self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self._nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._h = None

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                try:
                    r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                except AttributeError:
                    r = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self._h)
                self.reasons |= int(r)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self._h is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._h is not None:
            self._stop.set()
            self._t.join()

    def summary(self):
        if self._h is None or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "samples": len(self.samples),
                "reasons": [n for b, n in self.REASONS.items() if self.reasons & b]}


def router_on_tensor_cores(w, T: int, router: str) -> bool:
    """The library's router choice (MOE_OPT_ROUTER): tensor cores for E <= 128
    unless the FFMA router is asked for."""
    return w.E <= 128 and router != "ffma"


def launches_per_layer(w, T: int, router: str) -> int:
    """Kernels one moe_forward launches: router, route plan, gather, expert
    GEMMs, combine; the plan and the gather are one launch for one canvas
    (T <= 256, k <= 8)."""
    return 4 if (T <= 256 and w.k <= 8) else 5


# weight formats by moe_wdtype_t value (bf16, int4, fp8, fp4)
WFMT = {0: "bf16", 1: "int4 w4g128", 2: "fp8 E4M3 (fp32 row scales)",
        3: "fp4 E2M1 (E4M3 scales per 16 weights, fp32 row scales)"}


def layer_costs(w, touched: float, T: int):
    """Algorithmic bytes and FLOPs of one layer call: weights of the experts
    that receive a token (streamed once), x in, router tensors, out.  The
    expert kernel's share is those weights."""
    if w.wdtype == 0:  # bf16
        wbytes = 3 * w.f * w.d * 2
    elif w.wdtype == 2:  # fp8: E4M3 bytes + one fp32 scale per row
        wbytes = 3 * w.f * w.d + 4 * (2 * w.f + w.d)
    elif w.wdtype == 3:  # fp4: packed E2M1 + scale records (fp32 per row, E4M3 per 16)
        wbytes = 3 * w.f * w.d // 2 + 2 * w.f * (4 + w.d // 16) + w.d * (4 + w.f // 16)
    else:
        wbytes = 3 * w.f * w.d // 2 + 2 * (2 * w.f * w.n_groups_d + w.d * w.n_groups_f)
    expert_bytes = touched * wbytes
    act = T * w.d * 2 * (3 if w.residual else 2)
    router = w.E * w.d * 4 + w.d * 4 + (w.E * 4 if w.zipf_s > 0 else 0)
    flops = T * w.k * 2 * (3 * w.f * w.d) + 2 * T * w.E * w.d
    return expert_bytes, expert_bytes + act + router, flops, wbytes


# ---------------------------------------------------------------- CPU oracle timing


def oracle_sample_rate(lay_cpu, k, n_tokens, eps=1e-6):
    """Tokens/s of the oracle on the first n_tokens rows (all host threads)."""
    import oracle
    x = lay_cpu["x"][:n_tokens]
    t0 = time.perf_counter()
    oracle.moe_forward(x, lay_cpu["router_w"], lay_cpu["router_gamma"],
                       lay_cpu.get("router_bias"), lay_cpu["w_gate_up"], lay_cpu["w_down"], k,
                       scales_gate_up=lay_cpu.get("scales_gate_up"),
                       scales_down=lay_cpu.get("scales_down"), eps=eps,
                       expert_gamma=lay_cpu.get("expert_gamma"))
    return n_tokens / (time.perf_counter() - t0)


def cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def oracle_f32_sample_rate(lay_cpu, k, n_tokens, eps=1e-6):
    """Tokens/s of the oracle's single-precision timing build on the first
    n_tokens rows (all host threads)."""
    import oracle
    x = lay_cpu["x"][:n_tokens]
    t0 = time.perf_counter()
    oracle.moe_forward_f32(x, lay_cpu["router_w"], lay_cpu["router_gamma"],
                           lay_cpu.get("router_bias"), lay_cpu["w_gate_up"], lay_cpu["w_down"], k,
                           scales_gate_up=lay_cpu.get("scales_gate_up"),
                           scales_down=lay_cpu.get("scales_down"), eps=eps,
                           expert_gamma=lay_cpu.get("expert_gamma"))
    return n_tokens / (time.perf_counter() - t0)


def cpu_baseline(lay_cpu, w, budget_s=12.0):
    """The fp64 oracle as it stands (the value), and beside it the same
    definition compiled in single precision, each on a bounded sample."""
    import oracle
    cores = oracle.get_threads()
    probe = max(1, min(w.T, cores))
    r = oracle_sample_rate(lay_cpu, w.k, probe)
    n = int(max(probe, min(w.T, round(r * budget_s / cores) * cores)))
    r = oracle_sample_rate(lay_cpu, w.k, n)
    oracle.build_f32()
    r32 = oracle_f32_sample_rate(lay_cpu, w.k, probe)
    n32 = int(max(probe, min(w.T, round(r32 * budget_s / 2 / cores) * cores)))
    r32 = oracle_f32_sample_rate(lay_cpu, w.k, n32)
    return {"value": r, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "cpu_model": cpu_model(), "omp_threads": cores, "host_cpus": os.cpu_count(),
            "sample": f"first {n} of the {w.T} canvas tokens, fp64 oracle, one layer",
            "fp32_timing_build": {"value": r32, "unit": "tokens/s",
                                  "sample": f"first {n32} of the {w.T} canvas tokens, the "
                                            f"oracle compiled in single precision, one layer"}}


# ---------------------------------------------------------------- arms


def run_reference(args):
    from block_diffusion_moe_router_b200.replicas import dist_env
    rank, world, _ = dist_env()
    if rank != 0:
        return
    import torch
    import oracle
    from block_diffusion_moe_router_b200 import inputs
    w = inputs.WORKLOADS[args.workload]
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    lay = {k: (v.cpu() if isinstance(v, torch.Tensor) else v)
           for k, v in inputs.make_layer(w, device=dev).items()}
    cores = oracle.get_threads()
    r1 = oracle_sample_rate(lay, w.k, min(w.T, cores))
    steps = args.steps + args.warmup
    per = max(1, min(w.T, int(120.0 * r1 / steps)))
    pos = 0

    def step():
        nonlocal pos
        rows = [(pos + i) % w.T for i in range(per)]
        pos = (pos + per) % w.T
        sub = dict(lay)
        sub["x"] = lay["x"][rows]
        oracle.moe_forward(sub["x"], sub["router_w"], sub["router_gamma"],
                           sub.get("router_bias"), sub["w_gate_up"], sub["w_down"], w.k,
                           scales_gate_up=sub.get("scales_gate_up"),
                           scales_down=sub.get("scales_down"),
                           expert_gamma=sub.get("expert_gamma"))

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    value = args.steps * per / dt
    sample = f"{per} of the {w.T} canvas tokens per step (rotating), fp64 oracle, one layer"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000 * dt / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{w.name}: T={w.T} d={w.d} E={w.E} k={w.k} f={w.f} bf16 weights",
                   "sample_tokens_per_step": per},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "cpu_model": cpu_model(), "omp_threads": cores,
                         "host_cpus": os.cpu_count(), "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


class LayerRun:
    """One workload resident on this rank's GPU: its layers' weights, input
    sets rotated so that every step's working set (with the weights) exceeds
    L2, and a plan.  A step is one pass of the whole hot path: one moe_forward
    per layer (router -> plan -> gather -> expert GEMMs -> combine), layers
    chained through the residual."""

    def __init__(self, w, args, rank):
        import torch
        import block_diffusion_moe_router_b200 as moe
        from block_diffusion_moe_router_b200 import inputs
        from block_diffusion_moe_router_b200 import replicas as rep
        self.torch, self.moe, self.rep = torch, moe, rep
        self.w = w
        T, L = w.T, w.layers
        self.T, self.L = T, L
        self.lays = [inputs.make_layer(w, layer=l, device="cuda", with_x=False)
                     for l in range(L)]
        lay = self.lays[0]
        self.small = T * w.d * 2 * 2 + (w.E * w.d * 4 + w.d * 4 if L == 1 else 0)
        self.nsets = nsets = args.sets or max(2, math.ceil(1.1 * L2_BYTES / self.small))
        self.xs = [inputs._randn((T, w.d), 1.0, rep.replica_seed(rank, i), "cuda",
                                 torch.bfloat16) for i in range(nsets)]
        if L == 1:
            self.rws = [lay["router_w"]] + [
                lay["router_w"][torch.randperm(w.E, device="cuda")].contiguous()
                for _ in range(nsets - 1)]
            self.gms = [lay["router_gamma"]] + [lay["router_gamma"].roll(i).contiguous()
                                                for i in range(1, nsets)]
        self.outs = [torch.empty((T, w.d), dtype=torch.bfloat16, device="cuda")
                     for _ in range(nsets)]
        self.bufs = [torch.empty((T, w.d), dtype=torch.bfloat16, device="cuda")
                     for _ in range(2)]
        self.plan = moe.moe_plan_create(w.E, w.k, w.d, w.f, w.wdtype)
        moe.moe_plan_reserve(self.plan, T)
        moe.moe_plan_set_option(self.plan, moe.MOE_OPT_PDL, 0 if args.no_pdl else 1)
        moe.moe_plan_set_option(self.plan, moe.MOE_OPT_ROUTER,
                                {"auto": 0, "ffma": 1, "tc": 2}[args.router])
        if args.prefetch_mb is not None:
            moe.moe_plan_set_option(self.plan, moe.MOE_OPT_L2_PREFETCH_MB, args.prefetch_mb)
        moe.moe_plan_set_option(self.plan, moe.MOE_OPT_Y_BF16, 0 if args.y_fp32 else 1)
        self.stream = torch.cuda.current_stream()
        # experts that receive a token (their weights are the bytes the layer
        # must stream), per layer, averaged over the input sets
        self.touched = [0.0] * L
        off = torch.empty(w.E + 1, dtype=torch.int32, device="cuda")

        def count(l):
            moe.moe_plan_routing(self.plan, off, None, None, self.stream)
            self.touched[l] += float(((off[1:] - off[:-1]) > 0).sum().item()) / nsets

        for i in range(nsets):
            self.step(i, count)
        self.check()

    def layer_call(self, l, x, out, residual, rw=None, gm=None):
        ly = self.lays[l]
        self.moe.moe_forward(self.plan, self.T, x, ly["router_w"] if rw is None else rw,
                             ly["router_gamma"] if gm is None else gm, ly["router_bias"],
                             ly["w_gate_up"], ly["w_down"], ly["scales_gate_up"],
                             ly["scales_down"], residual, out, self.stream,
                             expert_gamma=ly["expert_gamma"])

    def step(self, i, per_layer=None):
        j = i % self.nsets
        if self.L == 1:
            self.layer_call(0, self.xs[j], self.outs[j], None, self.rws[j], self.gms[j])
            if per_layer is not None:
                per_layer(0)
            return self.outs[j]
        cur = self.xs[j]
        for l in range(self.L):  # x_{l+1} = x_l + MoE_l(x_l)
            nxt = self.bufs[l % 2]
            self.layer_call(l, cur, nxt, cur)
            if per_layer is not None:
                per_layer(l)
            cur = nxt
        return cur

    def check(self):
        st = self.moe.moe_plan_sync_status(self.plan, self.stream)
        if st != self.moe.MOE_OK:
            raise RuntimeError(self.moe.moe_status_str(st))

    def timed(self, K, profile, per_step=False):
        """Device time of K steps (CUDA events on the launching stream, barrier
        and synchronize on both sides, max over ranks), or the per-step list."""
        torch, moe, rep = self.torch, self.moe, self.rep
        moe.moe_plan_set_option(self.plan, moe.MOE_OPT_PROFILE, 1 if profile else 0)
        rep.barrier()
        torch.cuda.synchronize()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(K + 1 if per_step else 2)]
        ev[0].record(self.stream)
        for i in range(K):
            self.step(i)
            if per_step:
                ev[i + 1].record(self.stream)
        ev[-1].record(self.stream)
        torch.cuda.synchronize()
        rep.barrier()
        moe.moe_plan_set_option(self.plan, moe.MOE_OPT_PROFILE, 0)
        if per_step:
            return [ev[i].elapsed_time(ev[i + 1]) for i in range(K)]
        return rep.max_over_ranks(ev[0].elapsed_time(ev[-1]), "cuda")

    def warm(self, W):
        for i in range(W):
            self.step(i)
        self.torch.cuda.synchronize()
        for kk in range(len(self.moe.KERNEL_NAMES)):  # discard warm-up records
            self.moe.moe_plan_profile(self.plan, kk)

    def kernel_ms(self):
        kern = {}
        for kk, name in enumerate(self.moe.KERNEL_NAMES):
            tot, n = self.moe.moe_plan_profile(self.plan, kk)
            kern[name] = (tot / n) if n else None
        return kern

    def costs(self):
        """Per step: algorithmic bytes of the expert kernels (per launch), of
        the whole step, FLOPs, and the expert weight bytes per touched expert."""
        expert_bytes, layer_bytes, flops = 0.0, 0.0, 0.0
        for l in range(self.L):
            eb, lb, fl, wbytes = layer_costs(self.w, self.touched[l], self.T)
            expert_bytes += eb
            layer_bytes += lb
            flops += fl
        return expert_bytes / self.L, layer_bytes, flops, wbytes

    def forward_into(self, x, out):
        """One step on input x, the last layer writing into out (layers chained
        through the residual, as in step())."""
        if self.L == 1:
            self.layer_call(0, x, out, None, self.rws[0], self.gms[0])
            return out
        cur = x
        for l in range(self.L):
            nxt = out if l == self.L - 1 else self.bufs[l % 2]
            self.layer_call(l, cur, nxt, cur)
            cur = nxt
        return out

    def e2e_pipelined(self, K, x_host):
        """Device time of K end-to-end steps: each step copies its input from
        pinned host memory, runs the layer(s) and copies its result back to
        pinned host memory.  Two input and two output buffers; the copies run
        on two side streams, so step i+1's input and step i-1's result move
        while step i computes (the layer calls stay in order on the plan's
        stream)."""
        torch = self.torch
        T, d = self.T, self.w.d
        comp = self.stream
        cin, cout = torch.cuda.Stream(), torch.cuda.Stream()
        xin = [torch.empty((T, d), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
        outd = [torch.empty((T, d), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
        hout = [torch.empty((T, d), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_done = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]
        for b in range(2):
            ev_done[b].record(comp)
            ev_out[b].record(cout)
        self.rep.barrier()
        torch.cuda.synchronize()
        h0 = torch.cuda.Event(enable_timing=True)
        h1 = torch.cuda.Event(enable_timing=True)
        h0.record(cin)
        for i in range(K):
            b = i % 2
            cin.wait_event(ev_done[b])  # step i-2 no longer reads xin[b]
            with torch.cuda.stream(cin):
                xin[b].copy_(x_host[i % len(x_host)], non_blocking=True)
            ev_in[b].record(cin)
            comp.wait_event(ev_in[b])
            comp.wait_event(ev_out[b])  # step i-2's result has left outd[b]
            self.forward_into(xin[b], outd[b])
            ev_done[b].record(comp)
            cout.wait_event(ev_done[b])
            with torch.cuda.stream(cout):
                hout[b].copy_(outd[b], non_blocking=True)
            ev_out[b].record(cout)
        h1.record(cout)
        torch.cuda.synchronize()
        return h0.elapsed_time(h1)

    def close(self):
        self.moe.moe_plan_destroy(self.plan)
        self.lays = self.xs = self.outs = self.bufs = None
        self.torch.cuda.empty_cache()


def sub_record(name, args, rank, steps, warmup):
    """A second workload measured in the same run, for the same JSON line:
    its step time (events around the K steps), per-kernel times (a second run
    with events between the launches) and its roofline fractions against the
    measured HBM copy bandwidth and both measured bf16 GEMM peaks."""
    import torch
    from block_diffusion_moe_router_b200 import inputs
    w = inputs.WORKLOADS[name]
    run = LayerRun(w, args, rank)
    run.warm(warmup)
    _, local = rank, int(os.environ.get("LOCAL_RANK", "0"))
    with ClockSampler(local) as clk:
        ms = run.timed(steps, profile=False)
        run.timed(steps, profile=True)
    kern = run.kernel_ms()
    per_step = sorted(run.timed(steps, profile=False, per_step=True))
    run.check()
    expert_bytes, step_bytes, flops, wbytes = run.costs()
    hbm, bf16, bf16_sus, basis = peaks()
    ms_step = ms / steps
    t = ms_step * 1e-3
    rec = {
        "workload": f"{w.name}: T={w.T}, d={w.d}, E={w.E}, top-{w.k}, f={w.f}, "
                    f"{WFMT[w.wdtype]} weights, {w.layers} layer(s) per step",
        "steps": steps, "warmup": warmup,
        "ms_per_step": ms_step,
        "ms_per_layer": ms_step / w.layers,
        "tokens_per_s_per_layer": w.T * w.layers / t,
        "canvas_tokens_per_s_per_step": w.T / t,  # T tokens through all the step's layers
        "step_ms_p10_p50_p90": [per_step[int(q * (len(per_step) - 1))] for q in (0.1, 0.5, 0.9)],
        "touched_experts_per_layer": sum(run.touched) / w.layers,
        "alg_bytes_per_step": step_bytes,
        "flops_per_step": flops,
        "hbm_frac": step_bytes / t / (hbm * 1e9),
        "tensor_frac_of_burst_peak": flops / t / (bf16 * 1e12),
        "tensor_frac_of_sustained_peak": flops / t / (bf16_sus * 1e12),
        "frac_of_roofline": max(step_bytes / (hbm * 1e9), flops / (bf16_sus * 1e12)) / t,
        "peak_basis": f"{basis}: HBM {hbm} GB/s, bf16 {bf16} TFLOP/s burst, "
                      f"{bf16_sus} TFLOP/s sustained",
        "kernel_ms_per_layer": kern,
        "expert_kernel_hbm_frac": (expert_bytes / (kern["expert"] * 1e-3) / 1e9 / hbm)
        if kern.get("expert") else None,
        "clocks": clk.summary(),
        "gpu_launches": launches_per_layer(w, w.T, args.router) * w.layers * steps,
    }
    run.close()
    del run
    torch.cuda.empty_cache()
    return rec


def lmhead_record(args, rank, steps, warmup):
    """The lm_head step over a 256-token canvas (V=262144, d=2816) measured in
    the same run: step time, GEMM time and its fractions of the measured HBM
    bandwidth and of the sustained bf16 peak."""
    import torch
    import block_diffusion_moe_router_b200 as moe
    from block_diffusion_moe_router_b200 import inputs
    T, V, d = 256, inputs.LMHEAD_V, inputs.LMHEAD_D
    temp, bound = 0.8, 0.1
    nsets = 4
    hs, W, _ = inputs.make_lmhead(T * nsets, V, d, seed=11 + rank, device="cuda")
    hs = [hs[i * T:(i + 1) * T].contiguous() for i in range(nsets)]
    g = torch.Generator().manual_seed(3)
    masked = (torch.rand(T, generator=g) < 0.75).to(torch.uint8).cuda()
    lh = moe.LmHead(V, d)
    stream = torch.cuda.current_stream()
    outs = [torch.empty(T, dtype=dt, device="cuda")
            for dt in (torch.int32, torch.float32, torch.float32, torch.uint8)]

    def run(K):
        for i in range(K):
            moe.moe_lmhead_forward(lh.handle, T, hs[i % nsets], W, temp, 0.0, masked, bound,
                                   *outs, stream)

    run(warmup)
    torch.cuda.synchronize()
    local = int(os.environ.get("LOCAL_RANK", "0"))
    with ClockSampler(local) as clk:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        run(steps)
        e1.record(stream)
        torch.cuda.synchronize()
        moe.moe_lmhead_set_profile(lh.handle, True)
        run(steps)
        moe.moe_lmhead_set_profile(lh.handle, False)
    ms = e0.elapsed_time(e1) / steps
    gemm_ms, n = moe.moe_lmhead_profile(lh.handle)
    gemm_ms /= max(n, 1)
    if lh.sync_status() != moe.MOE_OK:
        raise RuntimeError("lm_head step reported a device error")
    lh.close()
    del hs, W
    torch.cuda.empty_cache()
    hbm, bf16, bf16_sus, basis = peaks()
    alg_bytes = V * d * 2 + T * d * 2
    flops = 2.0 * T * V * d
    return {
        "workload": f"lmhead: T={T} canvas tokens, V={V}, d={d}, bf16 h and W, temperature "
                    f"{temp}, entropy bound {bound}, 75% of positions masked",
        "steps": steps, "warmup": warmup,
        "ms_per_step": ms, "tokens_per_s": T / (ms * 1e-3),
        "gemm_ms": gemm_ms,
        "gemm_hbm_frac": alg_bytes / (gemm_ms * 1e-3) / 1e9 / hbm,
        "gemm_tensor_frac_of_sustained_peak": flops / (gemm_ms * 1e-3) / 1e12 / bf16_sus,
        "gemm_tensor_frac_of_burst_peak": flops / (gemm_ms * 1e-3) / 1e12 / bf16,
        "peak_basis": f"{basis}: HBM {hbm} GB/s, bf16 {bf16} / {bf16_sus} TFLOP/s",
        "clocks": clk.summary(),
        "gpu_launches": 3 * steps,
    }


def run_ours(args):
    import torch
    import block_diffusion_moe_router_b200 as moe
    from block_diffusion_moe_router_b200 import inputs
    from block_diffusion_moe_router_b200 import replicas as rep

    rank, world, local = rep.dist_env()
    torch.cuda.set_device(local)
    rep.init("nccl", torch.device("cuda", local), timeout_s=120)
    w = inputs.WORKLOADS[args.workload]
    T, L = w.T, w.layers
    run = LayerRun(w, args, rank)
    lay, plan, stream = run.lays[0], run.plan, run.stream
    nsets = run.nsets
    run.warm(args.warmup)
    with ClockSampler(local) as clk:
        # the reported time: K steps, CUDA events around the region only
        ms = run.timed(args.steps, profile=False)
        # diagnostics: the same K steps with per-kernel events between the
        # launches (they break the launch overlap, so this run is slower)
        ms_prof = run.timed(args.steps, profile=True)
    kern = run.kernel_ms()
    per_step = sorted(run.timed(args.steps, profile=False, per_step=True))
    pct = {f"p{q}": per_step[min(len(per_step) - 1, int(q / 100 * len(per_step)))]
           for q in (10, 50, 90)}
    run.check()

    # end to end: host x in, host result out, every step, through the C ABI.
    # Reported: the pipelined form (copies on side streams overlap the layer,
    # two buffers each way); beside it the blocking form, one
    # moe_forward_host call per step (copy in, layer, copy out, synchronise).
    x_host = [run.xs[i].cpu().pin_memory() for i in range(min(nsets, 4))]
    out_host = torch.empty((T, w.d), dtype=torch.bfloat16).pin_memory()
    K2 = args.steps
    run.e2e_pipelined(min(K2, 5), x_host)  # warm the side streams
    e2e_s = rep.max_over_ranks(run.e2e_pipelined(K2, x_host), "cuda") * 1e-3
    rep.barrier()
    torch.cuda.synchronize()
    h0 = torch.cuda.Event(enable_timing=True)
    h1 = torch.cuda.Event(enable_timing=True)
    h0.record(stream)
    for i in range(K2):
        if L == 1:
            moe.moe_forward_host(plan, T, x_host[i % len(x_host)], run.rws[0], run.gms[0],
                                 lay["router_bias"], lay["w_gate_up"], lay["w_down"],
                                 lay["scales_gate_up"], lay["scales_down"], None, out_host,
                                 stream, expert_gamma=lay["expert_gamma"])
        else:
            run.xs[0].copy_(x_host[i % len(x_host)], non_blocking=True)
            out_host.copy_(run.step(0), non_blocking=True)
            stream.synchronize()
    h1.record(stream)
    torch.cuda.synchronize()
    e2e_block_s = rep.max_over_ranks(h0.elapsed_time(h1), "cuda") * 1e-3
    run.check()

    hbm, bf16, bf16_sus, basis = peaks()
    expert_bytes, layer_bytes, flops, wbytes = run.costs()
    ms_step = ms / args.steps
    k_ms = kern["expert"]
    achieved = expert_bytes / (k_ms * 1e-3) / 1e9 if k_ms else None
    traffic = recorded_traffic(args.workload)
    touched = run.touched
    lay_cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        lay_cpu = {k: (v.cpu() if isinstance(v, torch.Tensor) else v) for k, v in lay.items()}
        lay_cpu["x"] = run.xs[0].cpu()
    run.close()
    del run
    desc = {
        "canvas": "one MoE layer over a T=256 token canvas",
        "canvas4": "one MoE layer over a T=256 token canvas, int4 w4g128 weights",
        "canvas8": "one MoE layer over a T=256 token canvas, fp8 E4M3 weights",
        "canvas4f": "one MoE layer over a T=256 token canvas, fp4 E2M1 weights",
        "encode": "one MoE layer over T=2048 tokens (1792 prompt + 256 canvas)",
        "stack30": "one denoising step: 30 stacked MoE layers (distinct weights, Zipf(1.1) "
                   "router bias, residual chained) over a T=256 canvas",
        "tiny": "tiny MoE layer",
    }[w.name]
    line = {
        "metric": METRIC,
        "value": rep.job_rate(T, world, args.steps, ms),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "fp16" if w.wdtype in (2, 3) else "bf16",
        "data": "synthetic",
        "config": {
            "workload": f"{w.name}: {desc}, d={w.d}, E={w.E}, top-{w.k}, f={w.f}, "
                        f"{WFMT[w.wdtype]} weights",
            "global_batch": world * T, "seq_len": T, "layers_per_step": L,
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "l2": f"weights {wbytes * w.E * L / 1e9:.2f} GB > L2; x/out rotated over "
                  f"{nsets} sets ({nsets * run_small(w, nsets) / 2**20:.0f} MiB)",
            "timed_region": "CUDA events around the K steps; per-kernel times from a second "
                            "timed run with events between the launches",
            "ms_per_step_with_kernel_events": ms_prof / args.steps,
            "step_ms_percentiles_rank0": pct,
            "pdl": not args.no_pdl,
            "y_dtype": "fp32" if args.y_fp32 else "bf16",
            "router": "tensor cores" if router_on_tensor_cores(w, T, args.router) else "ffma",
        },
        "roofline": {
            "bound": "hbm", "kernel": "expert (grouped gate_up + down GEMMs)",
            "achieved": achieved, "peak": hbm, "unit": "GB/s",
            "frac": (achieved / hbm) if achieved else None, "traffic": traffic,
            "peak_basis": f"{basis} HBM copy bandwidth",
            "alg_bytes_per_launch": expert_bytes,
            "alg_bytes_rule": f"{sum(touched) / L:.2f} touched experts per layer x {wbytes} B "
                              f"of expert weights",
            "kernel_ms": k_ms,
        },
        "layer_roofline": {
            "alg_bytes_per_step": layer_bytes, "flops_per_step": flops,
            "t_hbm_ms": layer_bytes / (hbm * 1e9) * 1e3,
            "t_tensor_ms": flops / (bf16 * 1e12) * 1e3,
            "frac_of_roofline": (max(layer_bytes / (hbm * 1e9), flops / (bf16 * 1e12)) * 1e3)
                                / ms_step,
            "tensor_frac_of_burst_peak": flops / (ms_step * 1e-3) / (bf16 * 1e12),
        },
        "kernel_ms": kern,
        "gpu_launches": launches_per_layer(w, T, args.router) * L * args.steps,
        "e2e": {"value": rep.job_rate(T, world, K2, e2e_s * 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": T * w.d * 2, "d2h_bytes_per_step": T * w.d * 2,
                "form": "every step: x from pinned host memory, the layer call(s), the "
                        "result to pinned host memory; copies on two side streams overlap "
                        "the layer (two buffers each way), device time by CUDA events",
                "blocking": {"value": rep.job_rate(T, world, K2, e2e_block_s * 1e3),
                             "unit": "tokens/s",
                             "form": "one synchronous moe_forward_host call per step"
                                     if L == 1 else "copy in, step, copy out, synchronise"}},
        "clocks": clk.summary(),
    }
    # the other workloads the layer is graded on, measured in the same run:
    # the T=2048 encode layer (tensor-core target) and the 30-layer step
    extras = [] if args.no_extra else [x for x in args.extra.split(",") if x and x != w.name]
    for name in extras:
        steps, warm = {"encode": (100, 20), "stack30": (20, 5)}.get(name, (100, 20))
        if name == "lmhead":
            line[name] = lmhead_record(args, rank, steps, warm)
        else:
            line[name] = sub_record(name, args, rank, steps, warm)
    if lay_cpu is not None:
        cb = cpu_baseline(lay_cpu, w)
        if L > 1:
            cb["value"] /= L
            cb["sample"] += f"; per step = {L} layers"
        line["cpu_baseline"] = cb
    if rank == 0:
        print(json.dumps(line), flush=True)
    rep.barrier()
    rep.shutdown()


def run_small(w, nsets):
    return w.T * w.d * 2 * 2 + (w.E * w.d * 4 + w.d * 4 if w.layers == 1 else 0)


LMHEAD_METRIC = ("canvas tokens/s through the lm_head step (T=256 logits over V=262144, "
                 "entropy and argmax folded on chip, entropy-bound acceptance)")


def run_lmhead(args):
    """The step after the layer stack: one moe_lmhead_forward over a 256-token
    canvas (V=262144, d=2816; W is 1.48 GB, far above L2, so no flush is
    needed).  Same JSON contract as the layer bench."""
    import torch
    import block_diffusion_moe_router_b200 as moe
    from block_diffusion_moe_router_b200 import inputs
    from block_diffusion_moe_router_b200 import replicas as rep

    rank, world, local = rep.dist_env()
    torch.cuda.set_device(local)
    rep.init("nccl", torch.device("cuda", local), timeout_s=120)
    T, V, d = 256, inputs.LMHEAD_V, inputs.LMHEAD_D
    temp, bound = 0.8, 0.1
    nsets = 4
    hs, W, _ = inputs.make_lmhead(T * nsets, V, d, seed=11 + rank, device="cuda")
    hs = [hs[i * T:(i + 1) * T].contiguous() for i in range(nsets)]
    g = torch.Generator().manual_seed(3)
    masked = (torch.rand(T, generator=g) < 0.75).to(torch.uint8).cuda()
    lh = moe.LmHead(V, d)
    stream = torch.cuda.current_stream()
    tok = torch.empty(T, dtype=torch.int32, device="cuda")
    ent = torch.empty(T, dtype=torch.float32, device="cuda")
    lz = torch.empty(T, dtype=torch.float32, device="cuda")
    acc = torch.empty(T, dtype=torch.uint8, device="cuda")

    def step(i):
        moe.moe_lmhead_forward(lh.handle, T, hs[i % nsets], W, temp, 0.0, masked, bound, tok, ent,
                               lz, acc, stream)

    def timed(K, per_step=False):
        rep.barrier()
        torch.cuda.synchronize()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(K + 1 if per_step else 2)]
        ev[0].record(stream)
        for i in range(K):
            step(i)
            if per_step:
                ev[i + 1].record(stream)
        ev[-1].record(stream)
        torch.cuda.synchronize()
        rep.barrier()
        if per_step:
            return [ev[i].elapsed_time(ev[i + 1]) for i in range(K)]
        return rep.max_over_ranks(ev[0].elapsed_time(ev[-1]), "cuda")

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        ms = timed(args.steps)
        moe.moe_lmhead_set_profile(lh.handle, True)
        ms_prof = timed(args.steps)
        moe.moe_lmhead_set_profile(lh.handle, False)
    gemm_ms, n = moe.moe_lmhead_profile(lh.handle)
    gemm_ms /= max(n, 1)
    per_step = sorted(timed(args.steps, per_step=True))
    pct = {f"p{q}": per_step[min(len(per_step) - 1, int(q / 100 * len(per_step)))]
           for q in (10, 50, 90)}
    if lh.sync_status() != moe.MOE_OK:
        raise RuntimeError("lm_head step reported a device error")

    # end to end: host h in, host token / entropy / accept out, every step
    h_host = [x.cpu().pin_memory() for x in hs]
    outs = [torch.empty(T, dtype=t.dtype).pin_memory() for t in (tok, ent, acc)]
    rep.barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(args.steps):
        hs[0].copy_(h_host[i % nsets], non_blocking=True)
        moe.moe_lmhead_forward(lh.handle, T, hs[0], W, temp, 0.0, masked, bound, tok, ent, lz,
                               acc, stream)
        for o, t in zip(outs, (tok, ent, acc)):
            o.copy_(t, non_blocking=True)
        stream.synchronize()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = rep.max_over_ranks(e0.elapsed_time(e1), "cuda")
    lh.close()

    # a kernel timed inside a long run of steps: the sustained bf16 figure
    hbm_gbs, _, bf16_tf, basis = peaks()
    w_bytes = V * d * 2
    alg_bytes = w_bytes + T * d * 2
    flops = 2.0 * T * V * d
    t_hbm = alg_bytes / (hbm_gbs * 1e9)
    t_tc = flops / (bf16_tf * 1e12)
    hbm_frac = (alg_bytes / (gemm_ms * 1e-3) / 1e9) / hbm_gbs
    tc_frac = (flops / (gemm_ms * 1e-3) / 1e12) / bf16_tf
    # the roofline is the slower of the two floors (they are within 1% here)
    if t_tc >= t_hbm:
        roof = {"bound": "tensor", "achieved": flops / (gemm_ms * 1e-3) / 1e12,
                "peak": bf16_tf, "unit": "TFLOP/s", "frac": tc_frac,
                "peak_basis": f"{basis} dense bf16 GEMM (sustained, under the power cap)"}
    else:
        roof = {"bound": "hbm", "achieved": alg_bytes / (gemm_ms * 1e-3) / 1e9,
                "peak": hbm_gbs, "unit": "GB/s", "frac": hbm_frac,
                "peak_basis": f"{basis} HBM copy bandwidth"}
    roof.update({"traffic": None, "kernel": "lm_head GEMM with the fused softmax statistics",
                 "kernel_ms": gemm_ms, "hbm_fraction": hbm_frac, "tensor_fraction": tc_frac,
                 "alg_bytes_per_launch": alg_bytes, "flops_per_launch": flops})
    line = {
        "metric": LMHEAD_METRIC,
        "value": rep.job_rate(T, world, args.steps, ms),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {
            "workload": f"lmhead: T={T} canvas tokens, V={V}, d={d}, bf16 h and W, temperature "
                        f"{temp}, entropy bound {bound}, 75% of positions masked",
            "global_batch": world * T, "seq_len": T,
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "l2": f"W {w_bytes / 1e9:.2f} GB > L2; h rotated over {nsets} sets",
            "timed_region": "CUDA events around the K steps; GEMM time from a second run "
                            "with events around the GEMM launch",
            "ms_per_step_with_kernel_events": ms_prof / args.steps,
            "step_ms_percentiles_rank0": pct,
            "t_hbm_ms": t_hbm * 1e3, "t_tensor_ms": t_tc * 1e3,
        },
        "roofline": roof,
        "gpu_launches": 3 * args.steps,
        "e2e": {"value": rep.job_rate(T, world, args.steps, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": T * d * 2, "d2h_bytes_per_step": T * (4 + 4 + 1)},
        "clocks": clk.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        oracle.build()
        h_cpu, W_cpu = hs[0][:2].cpu(), W.cpu()
        t0 = time.perf_counter()
        oracle.lmhead_stats(h_cpu, W_cpu, temperature=temp)
        dt = time.perf_counter() - t0
        line["cpu_baseline"] = {"value": 2 / dt, "unit": "tokens/s",
                                "cores": oracle.get_threads(), "kind": "oracle",
                                "sample": "2 of the 256 canvas tokens over the full vocabulary, "
                                          "fp64 oracle (one thread per token)"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    rep.barrier()


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    elif args.workload == "lmhead":
        run_lmhead(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
