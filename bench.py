#!/usr/bin/env python3
"""Benchmark of the B200 routed-MoE layer: one JSON line on rank 0.

A step is one pass of the whole layer (route -> bucket -> gate/up -> down ->
combine) over one batch of synthetic tokens.  Default workload: the
full-shape decode layer (d=2048, 512 experts, top-10 + 1 shared, f=768,
2-bit), 4 tokens per step (one token plus three draft tokens verified
together).  Inputs are larger than L2: the step rotates through R distinct
layers (R * 756 MB of packed weights) with fresh activations, so the touched
experts of a layer are evicted before it comes round again.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload decode|chain48|prefill|sweep|tiny]
                  [--tokens T] [--bits B] [--impl ours|reference]

Multi-GPU (torchrun): independent replicas, one per GPU (weak scaling); the
time is the max over ranks of the device-timed region.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "routed-MoE layer tokens/s (decode 1-4 tok, 8K prefill); % of HBM/TC roofline"


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default="decode", choices=["decode", "chain48", "prefill", "sweep", "tiny"])
    p.add_argument("--tokens", type=int, default=None)
    p.add_argument("--bits", type=int, default=2)
    p.add_argument("--bits-down", type=int, default=0, help="code width of the down matrices (sweep; 0: --bits)")
    p.add_argument("--rotate", type=int, default=8, help="distinct layers cycled through (decode/sweep)")
    p.add_argument("--flags", default="", help="extra forward flags, '+'-separated: gemv, gemm, tailskip "
                   "(the route-tail skip approximation)")
    p.add_argument("--expert-shard", default="", help="r/w: time one rank's partial layer of a w-way expert "
                   "split (the routed experts of range r, plus the shared one on rank 0)")
    p.add_argument("--cpu-seconds", type=float, default=12.0, help="budget of the oracle CPU-baseline sample")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-graph", action="store_true", help="time eager launches instead of a CUDA graph")
    p.add_argument("--no-sub", action="store_true", help="skip the decode T=1 and prefill sub-measurements")
    p.add_argument("--chain-two-calls", action="store_true", help="chain48: a norm launch, then the layer (default: "
                   "one call per layer with MOE_NORM_INPUT)")
    return p.parse_args()


# ---------------------------------------------------------------- ncu traffic of the dominant kernel
# kernel -> (source file, first line of its section or None for the whole file, first line after it)
_SEC = "// ---------------------------------------------------------------- "
_KERNEL_SOURCE = {"gemm_gateup": ("gemm_sm100.cu", _SEC + "grouped expert GEMM", _SEC + "router GEMM"),
                  "gemm_down": ("gemm_sm100.cu", _SEC + "grouped expert GEMM", _SEC + "router GEMM"),
                  "router_gemm": ("gemm_sm100.cu", _SEC + "router GEMM", _SEC + "activation gather, combine"),
                  "decode_fused": ("decode_pair.cu", None, None), "gemv_gateup": ("gemv.cu", None, None),
                  "gemv_down": ("gemv.cu", None, None)}


def kernel_source_hash(kernel: str):
    """First 16 hex digits of the sha256 of the kernel's source section (its file when it has none)."""
    import hashlib
    src = _KERNEL_SOURCE.get(kernel)
    if not src:
        return None
    path = os.path.join(ROOT, "bit_expert_ffn_gemv_b200", "csrc", src[0])
    try:
        text = open(path, "rb").read()
    except OSError:
        return None
    if src[1] is not None:
        a, b = src[1].encode(), src[2].encode()
        i = text.find(a)
        j = text.find(b, i + 1) if i >= 0 else -1
        if i < 0 or j < 0:
            return None
        text = text[i:j]
    return hashlib.sha256(text).hexdigest()[:16]


def profile_traffic(kernel: str, tokens=None):
    """DRAM bytes per launch of `kernel` from a committed ncu summary (profiles/*.md lines
    `traffic: kernel=K source_sha256_16=H tokens=T dram_bytes_per_launch=B`), or None when no capture of
    this workload size exists or the kernel's source changed since it was taken."""
    import glob
    cur = kernel_source_hash(kernel)
    if cur is None:
        return None
    for f in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md"))):
        for line in open(f):
            if not line.startswith("traffic:"):
                continue
            kv = dict(t.split("=", 1) for t in line.split()[1:] if "=" in t)
            if kv.get("kernel") == kernel and kv.get("source_sha256_16") == cur and \
                    (tokens is None or kv.get("tokens") == str(tokens)):
                return int(kv["dram_bytes_per_launch"])
    return None


# ---------------------------------------------------------------- replicas (one process per GPU)
def rank_master(master: int, rank: int) -> int:
    """Seed of a replica's weights and inputs: every rank draws its own data."""
    return master + 1000 * rank


def max_over_ranks(value: float, world: int, device="cuda") -> float:
    """The slowest rank's time (all ranks call this at the same point)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(tokens_per_step: int, steps: int, world: int, ms_max: float) -> float:
    """Whole-job tokens/s: every rank processes its own batches; time is the slowest rank's."""
    return tokens_per_step * steps * world / (ms_max / 1000.0)


# ---------------------------------------------------------------- workload description
def workload(args):
    from synth import WORKLOADS, MoeShape
    wl = WORKLOADS[args.workload]
    sh = wl.shape
    if args.workload == "sweep":
        sh = MoeShape(sh.d, sh.f, sh.E, sh.k, sh.n_shared, args.bits, bits_down=args.bits_down)
    T = args.tokens or {"decode": 4, "chain48": 1, "prefill": 8192, "sweep": 4, "tiny": 8}[args.workload]
    layers = 48 if args.workload == "chain48" else (1 if args.workload == "tiny" else max(1, args.rotate))
    return wl, sh, T, layers


def expert_bytes(sh):
    n = sh.f * sh.d
    return n * (2 * sh.bits + sh.bd) // 8 + 3 * (n // 32) * 2


def mat_bytes(sh, mat=0):
    """Bytes of one matrix (0 gate, 1 up, 2 down) at its own code width."""
    n = sh.f * sh.d
    return n * (sh.bd if mat == 2 else sh.bits) // 8 + (n // 32) * 2


# ---------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.out = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out = ""

    def summary(self):
        if not self.out:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        sm.sort()
        return {"sm_mhz": sm[len(sm) // 2] if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d.get("hbm_gbs", 6650.0), d.get("bf16_tflops", 1590.0), d.get("bf16_tflops_sustained", 1400.0), \
            "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


# ---------------------------------------------------------------- oracle CPU baseline
def oracle_sample(sh, wl, T, seconds, steps=None, warmup=0, layer_of=lambda i: 0, tokens_after_warmup=None):
    """Time the fp64 oracle on batches of T tokens of the workload; returns (tok/s, tokens, secs, threads).

    Runs `warmup` untimed batches, then either `steps` timed batches or timed batches until `seconds` of
    oracle time.  tokens_after_warmup(sec_per_token) may shrink the timed batches (>= 1 token) so that a
    fixed step count stays within a time budget.
    """
    import oracle
    import synth
    threads = oracle.threads()
    routers, experts = {}, {}
    done_tok, spent, i = 0, 0.0, 0
    warm_tok, warm_s = 0, 0.0
    Tb = T
    while True:
        if steps is not None and i >= steps + warmup:
            break
        if steps is None and spent >= seconds:
            break
        if i == warmup and tokens_after_warmup is not None and warm_tok:
            Tb = max(1, min(T, tokens_after_warmup(warm_s / warm_tok)))
        layer = layer_of(i)
        if layer not in routers:
            routers[layer] = synth.router_host(sh, wl.master, layer, wl.zipf)
        wr, bias = routers[layer]
        x = synth.x_host(sh, wl.master, 50000 + i, Tb)
        ids, _ = oracle.route(sh, x, wr, bias)
        need = sorted(set(ids.ravel().tolist()) | ({sh.E} if sh.n_shared else set()))
        codes = [None] * sh.n_experts_total
        scales = [None] * sh.n_experts_total
        for e in need:
            key = (layer, e)
            if key not in experts:
                pair = synth.expert_host(sh, wl.master, layer, e)
                if len(experts) >= 1024:  # bounded host cache (~1.5 GB at the full shape)
                    codes[e], scales[e] = pair
                    continue
                experts[key] = pair
            codes[e], scales[e] = experts[key]
        t0 = time.perf_counter()
        oracle.layer(sh, x, wr, bias, codes, scales)
        dt = time.perf_counter() - t0
        if i >= warmup:
            spent += dt
            done_tok += Tb
        else:
            warm_s += dt
            warm_tok += Tb
        i += 1
    return done_tok / spent, done_tok, spent, threads


def reference_arm(args):
    """The oracle as the reference arm: rank 0 alone, on the host cores.

    Exactly `--warmup` untimed and `--steps` timed batches.  Each timed batch is a bounded sample of the
    workload: up to 16 of its tokens, fewer when the step count would otherwise take more than about
    150 s of oracle time (the warm-up batches give the time per token).
    """
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    wl, sh, T, layers = workload(args)
    Tref = min(T, 16)
    steps, warmup = max(1, args.steps), max(0, args.warmup)
    budget_s = 150.0
    tps, ntok, secs, threads = oracle_sample(
        sh, wl, Tref, None, steps=steps, warmup=warmup, layer_of=lambda i: i % layers,
        tokens_after_warmup=lambda s_tok: int(budget_s / (steps * s_tok)))
    per_step = ntok // steps
    line = {"metric": METRIC, "value": tps, "unit": "tok/s", "n_gpus": 0, "steps": steps, "warmup": warmup,
            "ms_per_step": 1000.0 * secs / steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": args.workload, "tokens_per_step": T, "bits": sh.bits, "d": sh.d, "f": sh.f,
                       "experts": sh.E, "top_k": sh.k, "shared": sh.n_shared, "layers": layers},
            "cpu_baseline": {"value": tps, "unit": "tok/s", "cores": threads, "kind": "oracle",
                             "sample": f"{ntok} tokens in {steps} timed batches of {per_step} "
                                       f"(workload batches hold {T}; fp64 C oracle)"},
            "e2e": {"value": tps, "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def _graph_launches(h, step, n):
    """Kernels the library launches for n steps (counted eagerly, outside the timed region)."""
    import torch
    a = h.stats()["launches"]
    for i in range(n):
        step(i)
    torch.cuda.synchronize()
    return h.stats()["launches"] - a


def _capture(step, first, n):
    """A CUDA graph of steps first .. first + n - 1 (each step enqueued once while capturing)."""
    import torch
    cap_stream = torch.cuda.Stream()
    cap_stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(cap_stream):
        for i in range(n):  # settle any lazy per-kernel setup outside capture
            step(first + i)
    torch.cuda.current_stream().wait_stream(cap_stream)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(n):
            step(first + i)
    torch.cuda.synchronize()
    return g


def time_steps(step, steps, warmup, n_cap, use_graph, clock_index=None, world=1):
    """Device time (ms) of exactly `steps` steps after `warmup` untimed ones.

    With graphs: replays of a graph of n_cap consecutive steps, then one graph of
    the remaining steps % n_cap, so exactly `steps` steps run.  Returns
    (ms, clocks summary or None).
    """
    import torch
    import torch.distributed as dist
    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    graphs = []
    if use_graph:
        n_cap = max(1, min(n_cap, steps))
        full, rest = divmod(steps, n_cap)
        g_full = _capture(step, warmup, n_cap)
        graphs = [g_full] * full
        if rest:
            graphs.append(_capture(step, warmup, rest))
    if world > 1:
        dist.barrier()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clk = ClockSampler(clock_index) if clock_index is not None else None
    if clk:
        clk.__enter__()
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_push("timed")
    ev0.record()
    if use_graph:
        for g in graphs:
            g.replay()
    else:
        for i in range(steps):
            step(warmup + i)
    ev1.record()
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    if clk:
        clk.__exit__()
    return ev0.elapsed_time(ev1), (clk.summary() if clk else None)


def kernel_profile(h, step, first, n):
    """Per-kernel device time of n steps (events on the library's launch stream), behind a device-side
    sleep so that the events bracket back-to-back device work: {name: (total ms, launches)}."""
    import torch
    torch.cuda.synchronize()
    h.profile(True)
    torch.cuda._sleep(int(2e8))
    for i in range(n):
        step(first + i)
    prof = h.profile_read()
    h.profile(False)
    return prof


def roofline_of(prof, alg_bytes, flops, nprof, tokens=None):
    """Roofline entry of the dominant kernel of a per-kernel profile."""
    hbm, tc_burst, tc_sus, peak_kind = measured_peaks()
    if not prof:
        return None
    dom = max(prof.items(), key=lambda kv: kv[1][0])[0]
    if dom in flops:
        dom_ms = prof[dom][0] / prof[dom][1]
        ach = flops[dom] / (dom_ms / 1000.0) / 1e12
        r = {"bound": "tensor", "kernel": dom, "achieved": ach, "peak": tc_burst, "unit": "TFLOP/s",
             "frac": ach / tc_burst, "traffic": profile_traffic(dom, tokens),
             "peak_kind": peak_kind + " bf16 dense (burst)", "flops_per_launch": flops[dom],
             "avg_launch_us": 1000.0 * dom_ms}
        if alg_bytes.get(dom):
            # a grouped GEMM over small expert groups is bound by its weight bytes, not its FLOPs:
            # report against whichever bound takes longer
            bpl = alg_bytes[dom] / max(1, prof[dom][1])
            ach_b = bpl / (dom_ms / 1000.0) / 1e9
            r["hbm_frac"] = ach_b / hbm
            r["bytes_per_launch"] = bpl
            if bpl / (hbm * 1e9) > flops[dom] / (tc_burst * 1e12):
                r.update({"bound": "hbm", "achieved": ach_b, "peak": hbm, "unit": "GB/s", "frac": ach_b / hbm,
                          "peak_kind": peak_kind, "tensor_frac": ach / tc_burst})
        return r
    if dom in alg_bytes:
        dom_ms = prof[dom][0]
        ach = alg_bytes[dom] / (dom_ms / 1000.0) / 1e9
        r = {"bound": "hbm", "kernel": dom, "achieved": ach, "peak": hbm, "unit": "GB/s", "frac": ach / hbm,
             "traffic": profile_traffic(dom, tokens), "peak_kind": peak_kind,
             "bytes_per_launch": alg_bytes[dom] / max(1, prof[dom][1]),
             "avg_launch_us": 1000.0 * dom_ms / max(1, prof[dom][1])}
        if dom == "decode_fused":
            r["traffic_note"] = ("the clustered decode kernel needs a cooperative launch, which ncu's replay "
                                 "cannot reproduce; profiles/decode_pair_T4_phases.md has its device-side trace")
        return r
    return None


def layer_bytes(sh, D, T):
    """Algorithmic HBM bytes of one layer step: router, the D distinct routed experts and the shared one,
    activations in and out."""
    return sh.E * sh.d * 2 + (D + sh.n_shared) * expert_bytes(sh) + 4 * T * sh.d


def measure_decode(moe, h, sh, xs, layers, T, flags, args, steps, warmup, clock_index, world, chain=False):
    """Throughput and per-kernel breakdown of decode steps of T tokens (layers rotated)."""
    import torch
    n_x = len(xs)
    resid = [torch.empty_like(xs[0]) for _ in range(2)]
    normed = torch.empty_like(xs[0])
    ys = [torch.empty(T, sh.d, dtype=torch.bfloat16, device="cuda") for _ in range(2)]

    def step(i, stream=None):
        if chain:
            # residual chain x_{l+1} = x_l + layer_l(rmsnorm(x_l)), in place; one call per layer
            # (MOE_NORM_INPUT), or the norm kernel then the layer with --chain-two-calls
            r = resid[i & 1]
            r.copy_(xs[i % n_x])
            for l in range(layers):
                if args.chain_two_calls:
                    moe.rms_normalize(r, normed, stream=stream)
                    h.forward(l, normed, r, flags=flags | moe.MOE_ACCUMULATE, stream=stream)
                else:
                    h.forward(l, r, r, flags=flags | moe.MOE_ACCUMULATE | moe.MOE_NORM_INPUT, stream=stream)
            return r
        return h.forward(i % layers, xs[i % n_x], ys[i & 1], flags=flags, stream=stream)

    n_cap = max(layers, n_x) if not chain else 1
    ms, clocks = time_steps(step, steps, warmup, n_cap, not args.no_graph, clock_index, world)
    launches = _graph_launches(h, step, steps)
    # per-kernel device time and the algorithmic bytes of the same steps
    nl = layers if chain else 1
    nprof = min(steps, 64)
    alg = {"gemv_gateup": 0.0, "gemv_down": 0.0, "gemm_gateup": 0.0, "gemm_down": 0.0, "decode_fused": 0.0,
           "layer": 0.0}
    for i in range(nprof):
        step(warmup + i)
        D = h.stats()["active_experts"]
        lb = nl * layer_bytes(sh, D, T)
        alg["gemv_gateup"] += nl * (D + sh.n_shared) * 2 * mat_bytes(sh, 0)
        alg["gemv_down"] += nl * (D + sh.n_shared) * mat_bytes(sh, 2)
        alg["gemm_gateup"] += nl * (D + sh.n_shared) * 2 * mat_bytes(sh, 0)
        alg["gemm_down"] += nl * (D + sh.n_shared) * mat_bytes(sh, 2)
        alg["decode_fused"] += lb
        alg["layer"] += lb
    prof = kernel_profile(h, step, warmup, nprof)
    rows = T * sh.k + T * sh.n_shared
    flops = {"gemm_gateup": 2.0 * rows * 2 * sh.f * sh.d, "gemm_down": 2.0 * rows * sh.d * sh.f}
    layer_time = sum(v[0] for v in prof.values())
    return {"ms": ms, "clocks": clocks, "launches": launches, "step": step,
            "roofline": roofline_of(prof, alg, flops, nprof, T),
            "layer_hbm_gbs": alg["layer"] / (layer_time / 1000.0) / 1e9 if layer_time else None,
            "kernels_ms_per_step": {k: v[0] / nprof for k, v in prof.items()}}


def sub_block(moe, sgpu, wl, sh, T, layers, rank, args, steps, warmup):
    """A separate measured workload (its own handle) reported inside the main line."""
    import torch
    h = moe.MoeLayer(sh.d, sh.f, sh.E, sh.k, sh.n_shared, layers, sh.bits, T, bits_down=sh.bits_down)
    keep = []
    for l in range(layers):
        w = sgpu.layer_device(sh, rank_master(wl.master, rank), l, wl.zipf)
        h.load_layer(l, *w)
        keep.append(w)
    n_x = 4 if T > 64 else 16
    xs = [sgpu.x_device(sh, rank_master(wl.master, rank), 20000 + i, T) for i in range(n_x)]
    torch.cuda.synchronize()
    r = measure_decode(moe, h, sh, xs, layers, T, 0, args, steps, warmup, None, 1)
    h.close()
    del keep
    torch.cuda.empty_cache()
    return {"tokens_per_step": T, "layers": layers, "steps": steps, "value": T * steps / (r["ms"] / 1000.0),
            "unit": "tok/s", "ms_per_step": r["ms"] / steps, "roofline": r["roofline"],
            "kernels_ms_per_step": r["kernels_ms_per_step"], "gpu_launches": r["launches"]}


# ---------------------------------------------------------------- our arm
def ours(args):
    import torch
    import torch.distributed as dist

    import bit_expert_ffn_gemv_b200 as moe
    from bit_expert_ffn_gemv_b200 import build
    from synth import gpu as sgpu

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))
    build.build()
    wl, sh, T, layers = workload(args)
    names = {"gemv": moe.MOE_FORCE_GEMV, "gemm": moe.MOE_FORCE_GEMM, "tailskip": moe.MOE_ROUTE_TAIL_SKIP}
    flags = 0
    for f in filter(None, args.flags.split("+")):
        if f not in names:
            raise SystemExit(f"--flags: unknown flag {f!r} (known: {', '.join(names)})")
        flags |= names[f]

    # ---- setup: layers generated on the device, one handle holding all of them
    h = moe.MoeLayer(sh.d, sh.f, sh.E, sh.k, sh.n_shared, layers, sh.bits, T, bits_down=sh.bits_down)
    weights = []
    for l in range(layers):
        w = sgpu.layer_device(sh, rank_master(wl.master, rank), l, wl.zipf)
        h.load_layer(l, *w)
        weights.append(w)
    if args.expert_shard:
        from bit_expert_ffn_gemv_b200.expert_parallel import expert_shard
        r, w = (int(v) for v in args.expert_shard.split("/"))
        h.set_expert_range(*expert_shard(sh.E, r, w))
    n_x = 16
    xs = [sgpu.x_device(sh, rank_master(wl.master, rank), 10000 + i, T) for i in range(n_x)]
    chain = args.workload == "chain48"
    torch.cuda.synchronize()

    res = measure_decode(moe, h, sh, xs, layers, T, flags, args, args.steps, args.warmup, local, world, chain)
    ms = max_over_ranks(res["ms"], world)
    if world > 1:
        dist.barrier()
    value = replica_throughput(T, args.steps, world, ms)

    # ---- end to end through the host-buffer entry point (pinned memory)
    e2e = None
    if not args.no_e2e and not chain:
        xh = [x.cpu().pin_memory() for x in xs]
        yh = torch.empty(T, sh.d, dtype=torch.bfloat16).pin_memory()
        for i in range(3):
            h.forward_host(i % layers, xh[i % n_x], yh, flags=flags)
        torch.cuda.synchronize()
        k2 = min(args.steps, 100)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for i in range(k2):
            h.forward_host(i % layers, xh[i % n_x], yh, flags=flags)
        e1.record()
        torch.cuda.synchronize()
        ems = max_over_ranks(e0.elapsed_time(e1), world)
        e2e = {"value": replica_throughput(T, k2, world, ems), "unit": "tok/s", "h2d_bytes_per_step": T * sh.d * 2,
               "d2h_bytes_per_step": T * sh.d * 2}

    # ---- the rest of the metric ("decode 1-4 tok, 8K prefill"): decode T = 1 and one 8192-token
    # prefill chunk, each on its own handle (rank 0 of a single-GPU run only: replicas repeat it)
    subs = {}
    if args.workload == "decode" and world == 1 and not args.no_sub and not flags:
        h.close()
        del weights
        torch.cuda.empty_cache()
        h = None
        subs["decode_t1"] = sub_block(moe, sgpu, wl, sh, 1, layers, rank, args, max(args.steps, 16), args.warmup)
        subs["prefill_8192"] = sub_block(moe, sgpu, WORKLOADS_PREFILL(), WORKLOADS_PREFILL().shape, 8192, 1, rank,
                                         args, 10, 3)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        Tc = min(T, 16)
        tps, ntok, secs, threads = oracle_sample(sh, wl, Tc, args.cpu_seconds, layer_of=lambda i: 0)
        cpu = {"value": tps, "unit": "tok/s", "cores": threads, "kind": "oracle",
               "sample": f"{ntok} tokens in batches of {Tc}, {secs:.1f} s of fp64 C oracle work"}

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "tok/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": {"workload": args.workload, "tokens_per_step": T, "d": sh.d, "f": sh.f, "experts": sh.E,
                           "top_k": sh.k, "shared": sh.n_shared, "bits": sh.bits,
                           **({"bits_down": sh.bits_down} if sh.bits_down and sh.bits_down != sh.bits else {}),
                           "layers": layers,
                           "l2": ("inputs larger than L2: 48 layers x 756 MB per step" if chain else
                                  f"inputs larger than L2: {layers} distinct layers cycled, {n_x} fresh inputs"),
                           "parallelism": f"replicas x{world}",
                           "timing": "CUDA graph replay" if not args.no_graph else "eager",
                           **({"flags": args.flags} if args.flags else {}),
                           **({"expert_shard": args.expert_shard} if args.expert_shard else {})},
                "roofline": res["roofline"], "layer_hbm_gbs": res["layer_hbm_gbs"],
                "kernels_ms_per_step": res["kernels_ms_per_step"],
                **subs,
                "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": res["launches"], "clocks": res["clocks"]}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if h is not None:
        h.close()


def WORKLOADS_PREFILL():
    from synth import WORKLOADS
    return WORKLOADS["prefill"]


def main():
    args = parse()
    if args.impl == "reference":
        reference_arm(args)
    else:
        ours(args)


if __name__ == "__main__":
    main()
