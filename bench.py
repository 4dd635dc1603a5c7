#!/usr/bin/env python
"""Benchmark: one sparse MoE layer forward pass on B200 (gpt-oss-120b-shaped decode).

Workload: d_model=2880, 128 experts, top-4, SwiGLU d_ff=2880, MXFP4 expert
weights (E2M1 + E8M0 per 32), bf16 router and activations, T=64 tokens per
step (the largest decode batch of the configuration; seeded synthetic inputs).
A step is one moe_layer_forward: router, top-k, permutation, grouped SwiGLU
FFN over the routed experts, combine.

    python bench.py [--gpus N --steps K --warmup W] [--tokens T] [--impl ours|reference]

Prints one JSON line (rank 0).  Under torchrun each rank runs its own batch on
its own GPU (independent decode batches; no data-path collective), times are
the max over ranks, and ``value`` is all ranks' tokens per second.
``--impl reference`` times the fp64 CPU oracle on the host cores instead.
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

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import moe_inputs as mi  # noqa: E402

METRIC = "MoE-layer tokens/s and achieved HBM GB/s (decode) / TFLOPS (prefill) vs B200 peak"
SHAPE = mi.GPTOSS
PROFILE_EVERY = 10


def profile_every(steps):
    """Which timed steps carry per-kernel CUDA events (every n-th, never the
    first).  Events between launches stop a kernel from overlapping its
    predecessor, which costs a layer of a few tokens ~30 us on the steps that
    carry them, so long runs sample sparsely: every 50th step from 500 steps
    (10+ samples), every 10th from 100, else every step."""
    if steps >= 50 * PROFILE_EVERY:
        return 5 * PROFILE_EVERY
    return PROFILE_EVERY if steps >= 10 * PROFILE_EVERY else 1
DEFAULT_TOKENS = {"tiny": 16, "gptoss_decode": 64, "mixtral_prefill": 4096, "kimi_decode": 128,
                  "offload_bank": 16, "mixtral_prefill_mxfp4": 4096, "mixtral_prefill_nvfp4": 4096,
                  "mixtral_prefill_int4": 4096}
L2_BYTES = 126 * 2 ** 20


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "src": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "src": "fallback"}


def expert_bytes_split(shape):
    """(W13 bytes, W2 bytes) of one expert, codes + scales."""
    d, f = shape.d_model, shape.d_ff
    blk = mi.BLOCK[shape.wdtype]
    sb = {"mxfp4": 1, "nvfp4": 1, "int4": 2}.get(shape.wdtype, 0)
    if shape.wdtype == "bf16":
        return 2 * f * d * 2, d * f * 2
    return 2 * f * d // 2 + 2 * f * (d // blk) * sb, d * f // 2 + d * (f // blk) * sb


def workload_name(shape, T):
    return (f"{shape.name}: d_model={shape.d_model} E={shape.n_experts} top-{shape.top_k} "
            f"d_ff={shape.d_ff} {shape.wdtype.upper()} experts, T={T} tokens/step")


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi samples of the GPU's SM clock and throttle reasons while running."""

    FIELDS = ("index,pci.bus_id,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, bus: int = -1):
        self.bus = bus  # PCI bus number of the GPU under test (-1: take every row)
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 10:
                continue
            try:
                bus = int(parts[1].split(":")[1], 16)
            except (IndexError, ValueError):
                bus = -1
            if self.bus >= 0 and bus != self.bus:
                continue
            rows.append(parts)
        if not rows:
            return None
        sm = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        mx = max(float(r[3]) for r in rows if r[3].replace(".", "").isdigit())
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[6 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": reasons,
                "samples": len(rows)}


# --------------------------------------------------------------- oracle leg
def oracle_subset_layer(dlay, tokens):
    """A host layer holding x/router/bias and only the experts the given tokens need."""
    import torch
    from oracle import layer as OL
    hl = {"shape": dlay["shape"], "x": dlay["x"].cpu(), "router": dlay["router"].cpu(),
          "bias": dlay["bias"].cpu() if dlay.get("bias") is not None else None, "shared": None}
    logits = OL.router_logits(OL.to_f64(hl["x"])[tokens], OL.to_f64(hl["router"]),
                              OL.to_f64(hl["bias"]) if hl["bias"] is not None else None)
    idx, _, _ = OL.topk_select(logits, dlay["shape"].top_k)
    need = sorted(set(idx.reshape(-1).tolist()))

    class Lazy:
        def __init__(self, src):
            self.cache = {e: src[e].cpu() for e in need}

        def __getitem__(self, e):
            return self.cache[int(e)]

    hl["experts"] = {k: Lazy(v) for k, v in dlay["experts"].items()}
    if dlay.get("shared"):
        hl["shared"] = {k: v.cpu() for k, v in dlay["shared"].items()}
    _ = torch
    return hl, need


def time_oracle(hl, tokens):
    from oracle import layer as OL
    t0 = time.perf_counter()
    OL.moe_layer(hl, tokens=tokens)
    return time.perf_counter() - t0


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def host_mem_available():
    """MemAvailable of the host in bytes (None when unknown)."""
    try:
        for ln in open("/proc/meminfo"):
            if ln.startswith("MemAvailable:"):
                return int(ln.split()[1]) * 1024
    except OSError:
        pass
    return None


def cpu_model():
    try:
        for ln in open("/proc/cpuinfo"):
            if ln.startswith("model name"):
                return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def oracle_parallel(hl, tokens, n_threads):
    """The oracle as it stands on ``n_threads`` host cores: the tokens split into
    one contiguous chunk per thread, each chunk one oracle call with one BLAS
    thread (numpy releases the GIL inside its array operations).  Returns the
    wall time."""
    import concurrent.futures as cf
    from threadpoolctl import threadpool_limits
    from oracle import layer as OL
    chunks = [c.tolist() for c in np.array_split(np.asarray(tokens), min(n_threads, len(tokens))) if c.size]
    with threadpool_limits(limits=1):
        t0 = time.perf_counter()
        with cf.ThreadPoolExecutor(max_workers=len(chunks)) as ex:
            list(ex.map(lambda c: OL.moe_layer(hl, tokens=c), chunks))
        return time.perf_counter() - t0


def cpu_baseline(dlay, T, budget_s=12.0):
    """Oracle tokens/s on bounded samples of the batch: on every host core
    (the reported value) and, beside it, on one core."""
    from threadpoolctl import threadpool_limits
    cores = host_cores()
    with threadpool_limits(limits=1):
        hl, _ = oracle_subset_layer(dlay, [0])
        t1 = time_oracle(hl, [0])
        n1 = int(max(1, min(T, budget_s / 2 / max(t1, 1e-3))))
        hl, need1 = oracle_subset_layer(dlay, list(range(n1)))
        el1 = time_oracle(hl, list(range(n1)))
    # all cores: as many tokens as the cores clear in about the budget
    n = int(max(1, min(T, cores * budget_s / 2 / max(el1 / n1, 1e-3))))
    toks = list(range(n))
    hl, need = oracle_subset_layer(dlay, toks)
    el = oracle_parallel(hl, toks, cores)
    return {"value": n / el, "unit": "tokens/s", "cores": min(cores, n), "kind": "oracle",
            "cpu": cpu_model(),
            "sample": f"{n} of the {T} tokens of one batch ({len(need)} distinct experts decoded in fp64), "
                      f"{el:.1f} s on {min(cores, n)} threads (one token chunk and one BLAS thread each, "
                      f"numpy float64)",
            "single_core": {"value": n1 / el1, "unit": "tokens/s", "cores": 1,
                            "sample": f"{n1} tokens ({len(need1)} experts), {el1:.1f} s, one BLAS thread"}}


# ------------------------------------------------------------- reference arm
def run_reference(args):
    """The fp64 oracle on the host cores, same workload and metric.  Each step
    is one token per host core of the batch, the cores running the oracle side
    by side on their own tokens (one BLAS thread each); the number of timed
    steps is capped so the run ends within MOE_REF_BUDGET_S seconds (default
    150), and the line reports how many were timed."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import torch
    T = args.tokens or DEFAULT_TOKENS["gptoss_decode"]
    shape = SHAPE
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    budget = float(os.environ.get("MOE_REF_BUDGET_S", "150"))
    cores = host_cores()
    per_step = min(cores, T)
    t_draw = time.perf_counter()
    dlay = mi.draw_layer(shape, T, seed=1000, device=dev)  # the same inputs as the GPU arm
    hl, need = oracle_subset_layer(dlay, list(range(T)))
    del dlay
    t_draw = time.perf_counter() - t_draw

    def tokens_of(step):
        return [(step * per_step + i) % T for i in range(per_step)]

    n_warm = 0
    t_step = None
    for s in range(args.warmup):
        t_step = oracle_parallel(hl, tokens_of(s), per_step)
        n_warm += 1
        if t_step * (s + 2) > budget / 4:
            break
    n = args.steps
    if t_step is not None:
        n = int(max(3, min(args.steps, (budget - n_warm * t_step) / t_step)))
    el = 0.0
    for s in range(n):
        el += oracle_parallel(hl, tokens_of(n_warm + s), per_step)
    value = n * per_step / el
    sample = (f"each step: {per_step} tokens of the T={T} batch, one per host thread, through the fp64 oracle "
              f"(router, top-k, {shape.top_k} MXFP4 experts decoded to fp64, SwiGLU, combine); numpy, one BLAS "
              f"thread per token; {n} timed steps of {args.steps} requested (time budget {budget:.0f} s)")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": n, "steps_requested": args.steps, "warmup": n_warm, "ms_per_step": 1000 * el / n,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": workload_name(shape, T), "tokens": T, "input_setup_s": round(t_draw, 1)},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": per_step, "kind": "oracle",
                             "cpu": cpu_model(), "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------- multi-rank plumbing
def max_over_ranks(value: float, world: int, device="cpu") -> float:
    """The largest value over all ranks (timings are reported as the slowest rank's)."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tokens_per_s(world: int, tokens: int, steps: int, ms: float) -> float:
    """All ranks' tokens (each rank runs its own batch) over the slowest rank's time."""
    return world * tokens * steps / (ms * 1e-3)


# ----------------------------------------------------------------- our arm
def kernel_src_sha(name="ffn_stream.cu"):
    p = os.path.join(ROOT, "expert_ffn_layer_route_b200", "csrc", name)
    return hashlib.sha256(open(p, "rb").read()).hexdigest()[:16]


def stored_traffic(workload, T):
    """DRAM bytes per launch of the stage-1 kernel from a committed ncu summary,
    if it was taken on the current kernel source."""
    p = os.path.join(ROOT, "profiles", "ffn_stream_traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    ent = d.get(f"{workload}_T{T}")
    if not ent or ent.get("kernel_src_sha") != kernel_src_sha(ent.get("kernel_src_file", "ffn_stream.cu")):
        return None
    return ent.get("dram_bytes_per_launch")


def launches_per_step(prof, steps):
    """Kernel launches in the timed region: the sampled steps' launch count per
    step times the number of steps."""
    every = profile_every(steps)
    sampled = len([i for i in range(steps) if i > 0 and i % every == 0])
    per_step = sum(v[0] for v in prof.values()) / max(sampled, 1)
    return int(round(per_step * steps))


def run_ours(args):
    import torch
    import torch.distributed as dist
    import expert_ffn_layer_route_b200 as moe

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    shape = mi.CONFIGS[args.workload]
    if args.experts:
        # a reduced-expert variant of the layer (same d_model, d_ff, top-k and
        # format), for profiling captures that must stay a few GB on the device
        shape = shape.replace(n_experts=max(args.experts, shape.top_k))
    T = args.tokens or DEFAULT_TOKENS[args.workload]
    dlay = mi.draw_layer(shape, T, seed=1000 + rank, device=dev)
    desc = moe.make_desc(shape, T)
    ws = torch.empty(moe.moe_workspace_size(desc), dtype=torch.uint8, device=dev)
    out = torch.empty(T, shape.d_model, dtype=torch.bfloat16, device=dev)
    routed = moe.make_weights(dlay["experts"])
    shared = moe.make_weights(dlay["shared"]) if dlay.get("shared") else None
    stream = torch.cuda.current_stream(dev)

    def step(x=None):
        moe.moe_layer_forward(desc, dlay["x"] if x is None else x, dlay["router"], dlay["bias"], routed, shared,
                              out, ws, stream)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    # routing of this batch -> algorithmic bytes / flops
    L = moe.moe_workspace_layout_of(desc)
    offs = ws[L.offsets: L.offsets + 4 * (shape.n_experts + 1)].view(torch.int32).cpu().numpy()
    distinct = int((np.diff(offs) > 0).sum())
    b13, b2 = expert_bytes_split(shape)
    d, f, k, S = shape.d_model, shape.d_ff, shape.top_k, shape.n_shared
    act_bytes = 2 * T * d * 2
    router_bytes = shape.n_experts * d * (4 if shape.router_fp32 else 2)
    layer_bytes = (distinct + S) * (b13 + b2) + router_bytes + act_bytes
    rows = T * k + S * T
    layer_flops = 2.0 * rows * 3 * d * f + 2.0 * T * d * shape.n_experts
    stage1_bytes = (distinct + S) * b13 + rows * d * 2 + rows * f * 2
    stage1_flops = 2.0 * rows * d * 2 * f

    moe.moe_profile_enable(not args.no_kernel_timing)
    moe.moe_profile_collect()
    bus = -1
    try:
        bus = int(torch.cuda.get_device_properties(dev).pci_bus_id)
    except Exception:
        pass
    clocks = ClockSampler(bus) if rank == 0 else None
    if clocks:
        clocks.start()
        time.sleep(0.3)
    barrier()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # per-kernel CUDA events on a sample of the timed steps (profile_every:
    # every 50th of a run of 500+ steps, every 10th from 100, every step but
    # the first of a short one); events between launches also stop a kernel
    # from overlapping its predecessor, so they are sampled rather than put
    # around every launch
    every = profile_every(args.steps)
    e0.record(stream)
    for i in range(args.steps):
        if not args.no_kernel_timing:
            moe.moe_profile_enable(i > 0 and i % every == 0)
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    clk = clocks.stop() if clocks else None
    moe.moe_profile_enable(False)
    prof = moe.moe_profile_collect()
    launches = launches_per_step(prof, args.steps)
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev)

    # end to end: pinned host input -> device, layer, result -> pinned host, every step
    xh = dlay["x"].cpu().pin_memory()
    oh = torch.empty(T, d, dtype=torch.bfloat16).pin_memory()
    xd = torch.empty_like(dlay["x"])

    def e2e_step():
        xd.copy_(xh, non_blocking=True)
        step(xd)
        oh.copy_(out, non_blocking=True)

    for _ in range(max(3, args.warmup)):
        e2e_step()
    torch.cuda.synchronize(dev)
    barrier()
    e2 = torch.cuda.Event(enable_timing=True)
    e3 = torch.cuda.Event(enable_timing=True)
    e2.record(stream)
    for _ in range(args.steps):
        e2e_step()
    e3.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    ms_e2e = max_over_ranks(e2.elapsed_time(e3), world, dev)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(dlay, T)

    if rank == 0:
        pk = peaks()
        # the stage-1 kernel that ran: the tensor-core GEMM (bf16 or 4-bit
        # weights) for prefill-sized groups, else the weight-streaming kernel
        kname = next((kk for kk in ("ffn_gemm_stage1_gate_up", "ffn_gemm_q4_stage1_gate_up") if kk in prof),
                     "ffn_stage1_gate_up")
        tensor_path = kname != "ffn_stage1_gate_up"
        s1 = prof.get(kname, (0, 0.0))
        s1_ms = s1[1] / max(s1[0], 1)
        step_s = ms / args.steps * 1e-3
        if tensor_path:
            # the kernel is timed inside steps of a few ms: the burst peak, unless
            # a single step runs for seconds (then the sustained one)
            long_step = ms / args.steps > 1000.0
            peak = pk["bf16_tflops_sustained"] if long_step else pk["bf16_tflops"]
            achieved = stage1_flops / (s1_ms * 1e-3) / 1e12 if s1_ms else 0.0
            roof = {"bound": "tensor", "kernel": kname, "achieved": achieved, "peak": peak,
                    "peak_source": pk["src"] + (" sustained" if long_step else " burst"), "unit": "TFLOP/s",
                    "frac": achieved / peak, "traffic": stored_traffic(args.workload, T),
                    "algorithmic_flops_per_launch": stage1_flops, "avg_launch_us": 1000 * s1_ms}
        else:
            achieved = stage1_bytes / (s1_ms * 1e-3) / 1e9 if s1_ms else 0.0
            roof = {"bound": "hbm", "kernel": kname, "achieved": achieved, "peak": pk["hbm_gbs"],
                    "peak_source": pk["src"], "unit": "GB/s", "frac": achieved / pk["hbm_gbs"],
                    "traffic": stored_traffic(args.workload, T),
                    "algorithmic_bytes_per_launch": stage1_bytes, "avg_launch_us": 1000 * s1_ms}
        per_kernel = {kk: {"launches": v[0], "avg_us": 1000.0 * v[1] / max(v[0], 1),
                           "share": v[1] / max(sum(w[1] for w in prof.values()), 1e-12)} for kk, v in prof.items()}
        value = whole_job_tokens_per_s(world, T, args.steps, ms)
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": workload_name(shape, T), "tokens": T, "weights": shape.wdtype,
                       "parallelism": f"replicas x{world} (independent batches)",
                       "l2": f"inputs larger than L2: {distinct + S} distinct experts = "
                             f"{(distinct + S) * (b13 + b2) / 1e9:.2f} GB of weights per step vs "
                             f"{L2_BYTES / 2**20:.0f} MiB L2",
                       "distinct_experts": distinct + S, "layer_algorithmic_bytes": layer_bytes,
                       "layer_achieved_gbs": layer_bytes / step_s / 1e9,
                       "layer_algorithmic_flops": layer_flops, "layer_achieved_tflops": layer_flops / step_s / 1e12},
            "roofline": roof,
            "kernels": per_kernel,
            "gpu_launches": launches,
            "e2e": {"value": whole_job_tokens_per_s(world, T, args.steps, ms_e2e), "unit": "tokens/s",
                    "h2d_bytes_per_step": T * d * 2, "d2h_bytes_per_step": T * d * 2},
            "clocks": clk,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_offload(args):
    """Offloaded bank: decode steps through --bank-layers NVFP4 layers (default
    all 48) whose experts live in pinned host memory, 25% of each layer
    resident in HBM under LRU, with next-layer prefetch.  Reports hit rate,
    H2D GB/s against a measured pinned host-to-device copy peak, tokens/s of
    the layer stack, and the copy time prefetch hides: a second run of
    --bank-noprefetch-steps steps without prefetch, and the time of one layer
    with every expert resident (compute alone)."""
    import torch
    import expert_ffn_layer_route_b200 as moe
    from expert_ffn_layer_route_b200.offload import OffloadedBank
    shape = mi.BANK
    T = args.tokens or DEFAULT_TOKENS["offload_bank"]
    L = args.bank_layers
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    # pinned host -> device copy peak (1 GiB, best of 5)
    hb = torch.empty(1 << 30, dtype=torch.uint8).pin_memory()
    db = torch.empty(1 << 30, dtype=torch.uint8, device=dev)
    best = 0.0
    for _ in range(5):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        db.copy_(hb, non_blocking=True)
        b.record()
        torch.cuda.synchronize()
        best = max(best, (1 << 30) / (a.elapsed_time(b) * 1e-3) / 1e9)
    del hb, db
    # the pinned bank must leave the host room: take fewer layers when it would not
    note = None
    per_layer_bytes = shape.n_experts * (mi.expert_bytes(shape) + 4 * 256)
    avail = host_mem_available()
    if avail is not None:
        fit = int((avail - 40 * 2 ** 30) // per_layer_bytes)
        if fit < L:
            note = f"layers reduced from {L} to {max(fit, 1)} to fit the host's available memory ({avail / 2**30:.0f} GiB)"
            L = max(fit, 1)
    bank = OffloadedBank(shape, L, mi.BANK_SLOTS_PER_LAYER, T)
    t0 = time.perf_counter()
    resident_ms = None
    for l in range(L):
        lay = mi.bank_layer(shape, l, 0, dev)
        bank.fill_layer(l, lay)
        if l == 0:
            # one layer with all 256 experts resident in HBM: the compute alone
            desc = moe.make_desc(shape, T)
            ws = torch.empty(moe.moe_workspace_size(desc), dtype=torch.uint8, device=dev)
            out = torch.empty(T, shape.d_model, dtype=torch.bfloat16, device=dev)
            w = moe.make_weights(lay["experts"])
            xs = [mi.bank_step_tokens(10_000 + i, T, shape.d_model, 0, dev) for i in range(8)]
            for i in range(5):
                moe.moe_layer_forward(desc, xs[i % 8], lay["router"], lay["bias"], w, None, out, ws)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            for i in range(40):
                moe.moe_layer_forward(desc, xs[i % 8], lay["router"], lay["bias"], w, None, out, ws)
            b.record()
            torch.cuda.synchronize()
            resident_ms = a.elapsed_time(b) / 40
            del ws, out, w
        del lay
    fill_s = time.perf_counter() - t0
    for s_ in range(args.warmup):
        bank.decode_step(mi.bank_step_tokens(s_, T, shape.d_model, 0, dev))
    torch.cuda.synchronize()

    def timed(n, first, prefetch):
        st0 = bank.stats()
        xs = [mi.bank_step_tokens(first + s_, T, shape.d_model, 0, dev) for s_ in range(n)]
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for s_ in range(n):
            bank.decode_step(xs[s_], prefetch=prefetch)
        e1.record()
        torch.cuda.synchronize()
        st1 = bank.stats()
        return e0.elapsed_time(e1), {k: st1[k] - st0[k] for k in st1}

    sweep = None
    if args.bank_prefetch_sweep:
        # short runs over the prefetch depth (experts prefetched per token), same bank
        sweep = []
        first = args.warmup
        for p_top in [int(v) for v in args.bank_prefetch_sweep.split(",")]:
            bank.prefetch_top = p_top
            n_sw = args.bank_sweep_steps
            ms_sw, d_sw = timed(n_sw, first, p_top > 0)
            first += n_sw
            sweep.append({"prefetch_top": p_top, "steps": n_sw, "tokens_per_s": T * n_sw / (ms_sw * 1e-3),
                          "ms_per_layer": ms_sw / n_sw / L, "hit_rate": d_sw["hits"] / max(d_sw["lookups"], 1),
                          "bytes_h2d_per_step": d_sw["bytes_h2d"] / n_sw,
                          "prefetch_used_frac": d_sw["prefetch_used"] / max(d_sw["prefetch_issued"], 1)})
    bank.prefetch_top = args.bank_prefetch_top if args.bank_prefetch_top >= 0 else None
    if args.bank_prefetch_top == -2:
        bank.prefetch_top = 0
    clocks = ClockSampler()
    clocks.start()
    time.sleep(0.3)
    ms, d = timed(args.steps, args.warmup + (sum(e["steps"] for e in sweep) if sweep else 0), True)
    # a second run in the same steady state with the other prefetch choice
    # (every predicted expert when the main run had none, else none)
    n_np = args.bank_noprefetch_steps
    main_top = bank.prefetch_top
    other_top = shape.top_k if main_top == 0 else 0
    bank.prefetch_top = other_top
    ms_np, d_np = timed(n_np, 10 ** 6, True) if n_np > 0 else (None, None)
    bank.prefetch_top = main_top
    clk = clocks.stop()
    h2d = d["bytes_h2d"] / (ms * 1e-3) / 1e9
    per_layer = ms / args.steps / L
    line = {
        "metric": METRIC, "value": T * args.steps / (ms * 1e-3), "unit": "tokens/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"offload_bank: {L} of 48 layers x (d_model=4096 E=256 top-8 d_ff=1536 NVFP4), "
                               f"{mi.BANK_SLOTS_PER_LAYER} HBM slots per layer (25%), LRU + next-layer prefetch, "
                               f"T={T} tokens/step, residual chain x_l+1 = x_l + out_l",
                   "tokens": T, "layers": L, "bank_bytes": L * shape.n_experts * bank.blob.size,
                   "fill_s": round(fill_s, 1), "host_memory_note": note},
        "roofline": {"bound": "pcie_h2d", "achieved": h2d, "peak": best, "unit": "GB/s", "frac": h2d / best,
                     "peak_source": "measured pinned cudaMemcpy, 1 GiB", "traffic": None},
        "offload": {"hit_rate": d["hits"] / max(d["lookups"], 1), "lookups": d["lookups"], "hits": d["hits"],
                    "misses": d["misses"], "prefetch_issued": d["prefetch_issued"],
                    "prefetch_used": d["prefetch_used"], "bytes_h2d_per_step": d["bytes_h2d"] / args.steps,
                    "copy_ms_per_step": d["copy_ms"] / args.steps, "h2d_gbs": h2d,
                    "ms_per_layer": per_layer, "resident_ms_per_layer": resident_ms,
                    "exposed_ms_per_layer": per_layer - resident_ms if resident_ms is not None else None,
                    "prefetch_top": main_top if main_top is not None else "auto"},
        "prefetch_sweep": sweep,
        "clocks": clk,
    }
    if ms_np is not None:
        pl_np = ms_np / n_np / L
        line["offload_other_prefetch"] = {
            "prefetch_top": other_top, "steps": n_np, "ms_per_layer": pl_np,
            "hit_rate": d_np["hits"] / max(d_np["lookups"], 1), "bytes_h2d_per_step": d_np["bytes_h2d"] / n_np,
            "prefetch_used_frac": d_np["prefetch_used"] / max(d_np["prefetch_issued"], 1),
            "exposed_ms_per_layer": pl_np - resident_ms if resident_ms is not None else None,
            "tokens_per_s": T * n_np / (ms_np * 1e-3)}
    print(json.dumps(line), flush=True)
    bank.close()
    return 0


def run_verify(args):
    """Speculative verification blocks on the gpt-oss-shaped decode layer:
    n_seq sequences each verify depth drafted tokens plus their own position
    in one layer call (T = n_seq * (depth + 1) positions that read the union of
    their experts once), against ordinary decode of the same sequences (T =
    n_seq, one position each).  Accepted output per block follows seeded
    accept flags (probability alpha per draft, stopping at the first
    rejection).  Reports accepted tokens/s and layer bytes per accepted token
    for both."""
    import torch
    import expert_ffn_layer_route_b200 as moe
    from expert_ffn_layer_route_b200 import verify as V
    shape = mi.GPTOSS
    nseq, depth, rho, alpha = args.verify_seqs, args.verify_depth, args.verify_rho, args.verify_alpha
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    lay = mi.draw_layer(shape, 1, seed=1000, device=dev)
    routed = moe.make_weights(lay["experts"])
    b13, b2 = expert_bytes_split(shape)
    stream = torch.cuda.current_stream(dev)

    def measure(T, xs):
        desc = moe.make_desc(shape, T)
        ws = torch.empty(moe.moe_workspace_size(desc), dtype=torch.uint8, device=dev)
        out = torch.empty(T, shape.d_model, dtype=torch.bfloat16, device=dev)
        for i in range(args.warmup):
            moe.moe_layer_forward(desc, xs[i % len(xs)], lay["router"], None, routed, None, out, ws, stream)
        torch.cuda.synchronize()
        L = moe.moe_workspace_layout_of(desc)
        distinct = []
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(args.steps):
            moe.moe_layer_forward(desc, xs[i % len(xs)], lay["router"], None, routed, None, out, ws, stream)
        e1.record(stream)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / args.steps
        for x in xs:  # experts each input reads (union over its positions), untimed
            moe.moe_layer_forward(desc, x, lay["router"], None, routed, None, out, ws, stream)
            offs = ws[L.offsets: L.offsets + 4 * (shape.n_experts + 1)].view(torch.int32).cpu().numpy()
            distinct.append(int((np.diff(offs) > 0).sum()))
        d_mean = float(np.mean(distinct))
        layer_bytes = d_mean * (b13 + b2) + shape.n_experts * shape.d_model * 2 + 2 * T * shape.d_model * 2
        return ms, d_mean, layer_bytes

    n_inputs = 8
    xv = [mi.draw_verify_tokens(nseq, depth, shape.d_model, rho, 2000 + i, dev) for i in range(n_inputs)]
    x1 = [xi.view(nseq, depth + 1, -1)[:, 0].contiguous() for xi in xv]  # the sequences' own positions
    clocks = ClockSampler()
    clocks.start()
    time.sleep(0.3)
    ms_v, dv, bytes_v = measure(nseq * (depth + 1), xv)
    ms_o, do, bytes_o = measure(nseq, x1)
    clk = clocks.stop()
    acc = [sum(V.accepted_tokens(a) for a in mi.draw_accepts(nseq, depth, alpha, 3000 + i).tolist())
           for i in range(args.steps)]
    acc_mean = float(np.mean(acc))
    value = acc_mean / (ms_v * 1e-3)
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_v, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"verify: gpt-oss-shaped decode layer (d_model=2880 E=128 top-4 d_ff=2880 MXFP4), "
                               f"{nseq} sequences x (1 + {depth} drafted) positions per call, positions of a "
                               f"sequence correlated (rho={rho}), accept probability {alpha} per draft",
                   "tokens": nseq * (depth + 1), "l2": "inputs larger than L2 (each call reads >= 1 GB of experts)"},
        "verify": {"accepted_per_step": acc_mean, "expected_accepted_per_step": nseq * V.expected_accepted_tokens(depth, alpha),
                   "distinct_experts": dv, "layer_bytes": bytes_v,
                   "bytes_per_accepted_token": V.bytes_per_accepted_token(bytes_v, acc_mean),
                   "ms_per_call": ms_v},
        "ordinary_decode": {"tokens_per_step": nseq, "distinct_experts": do, "layer_bytes": bytes_o,
                            "bytes_per_token": V.bytes_per_accepted_token(bytes_o, nseq), "ms_per_call": ms_o,
                            "tokens_per_s": nseq / (ms_o * 1e-3)},
        "clocks": clk,
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--tokens", type=int, default=0, help="tokens per step (default: the workload's)")
    ap.add_argument("--experts", type=int, default=0,
                    help="routed experts of a reduced layer variant (default: the workload's); for profiling captures")
    ap.add_argument("--workload", choices=sorted(DEFAULT_TOKENS) + ["verify"], default="gptoss_decode")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--bank-layers", type=int, default=mi.BANK_LAYERS, help="layers of the offloaded bank (of 48)")
    ap.add_argument("--bank-noprefetch-steps", type=int, default=128,
                    help="offload_bank: steps of a second run with the other prefetch choice (0: none)")
    ap.add_argument("--bank-prefetch-top", type=int, default=-2,
                    help="offload_bank: experts prefetched per token, its most likely ones (-2: none, the "
                         "default; -1: every prediction when they fit a quarter of the slots, else one)")
    ap.add_argument("--bank-prefetch-sweep", default="",
                    help="offload_bank: comma-separated prefetch depths timed first, --bank-sweep-steps each")
    ap.add_argument("--bank-sweep-steps", type=int, default=48)
    ap.add_argument("--verify-seqs", type=int, default=16, help="verify: sequences per call")
    ap.add_argument("--verify-depth", type=int, default=3, help="verify: drafted tokens per sequence")
    ap.add_argument("--verify-rho", type=float, default=0.5, help="verify: correlation of a sequence's positions")
    ap.add_argument("--verify-alpha", type=float, default=0.7, help="verify: accept probability per draft")
    ap.add_argument("--no-kernel-timing", action="store_true",
                    help="no per-kernel CUDA events in the timed region (the roofline fields are then empty)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    if args.workload == "offload_bank":
        return run_offload(args)
    if args.workload == "verify":
        return run_verify(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
