"""Device-side phase trace of the clustered decode kernel.

The kernel is launched cooperatively as clusters of two CTAs, a launch that a
kernel-replaying profiler cannot reproduce, so its timeline comes from the
kernel itself: built with -DMOE_PAIR_TRACE, thread 0 of every CTA stamps the
global timer at each phase boundary and sums clock64() differences per phase.
This tool builds that traced copy of the library (under _build/trace/, apart
from the product's libmoe.so), runs full-shape decode layers on synthetic
inputs, and prints per-phase times over the CTAs (min / median / max).

  python -m bit_expert_ffn_gemv_b200.phase_trace [--tokens 4] [--bits 2] [--reps 3] [--sm-mhz 1965]
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import ctypes
import os
import subprocess
import sys

import numpy as np

from . import build as _build

TRACE_DIR = os.path.join(_build.ROOT, "_build", "trace")
TRACE_LIB = os.path.join(TRACE_DIR, "libmoe.so")
SLOTS = 48      # boundary stamps per CTA
CYC_SLOTS = 32  # cycle accumulators per CTA

BOUNDARIES = {0: "start", 1: "router done", 2: "routing starts (shared-expert gate/up done)", 3: "router barrier passed",
              4: "top-k done", 5: "schedule done", 38: "routed units done", 39: "partial-sum barrier passed",
              40: "end"}
BOUNDARIES.update({6 + 2 * i: f"gate/up of routed unit {i} done" for i in range(16)})
CYCLES = {27: "router", 6: "top-k (own tokens)", 10: "top-k: loads + keys", 11: "top-k: extraction rounds",
          13: "top-k: ranking", 15: "top-k: exact-scan fallback", 14: "weights (softmax, after the schedule)",
          16: "schedule: wait for other warps' top-k", 17: "schedule: masks + compaction",
          18: "schedule: slot places + meta", 7: "top-k + schedule", 1: "gate/up: wait for weights",
          2: "gate/up: compute", 3: "gate/up: h exchange", 4: "down: wait for weights", 5: "down: compute",
          19: "tail: partial-sum barrier", 20: "tail: reduction"}


def build_traced(force: bool = False) -> str:
    """libmoe.so with the phase trace compiled in, under _build/trace/."""
    objdir = os.path.join(TRACE_DIR, "obj")
    os.makedirs(objdir, exist_ok=True)
    if not force and os.path.exists(TRACE_LIB) and all(
            os.path.getmtime(TRACE_LIB) >= os.path.getmtime(p) for p in _build._inputs()):
        return TRACE_LIB

    def one(src):
        out = os.path.join(objdir, os.path.basename(src)[:-3] + ".o")
        subprocess.check_call([_build.NVCC, *_build.ARCH, *_build.FLAGS, "-DMOE_PAIR_TRACE", "-c", src, "-o", out])
        return out

    srcs = _build.sources()
    with cf.ThreadPoolExecutor(max_workers=min(len(srcs), os.cpu_count() or 4)) as ex:
        objs = list(ex.map(one, srcs))
    subprocess.check_call([_build.NVCC, *_build.ARCH, "-shared", "-o", TRACE_LIB, *objs])
    return TRACE_LIB


def _stats(v):
    return float(np.min(v)), float(np.median(v)), float(np.max(v))


def main(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--tokens", type=int, default=4)
    p.add_argument("--bits", type=int, default=2)
    p.add_argument("--layers", type=int, default=4, help="distinct layers cycled (larger than L2 together)")
    p.add_argument("--reps", type=int, default=3)
    p.add_argument("--sm-mhz", type=float, default=1965.0, help="SM clock for converting cycles to us")
    args = p.parse_args(argv)

    import torch

    import bit_expert_ffn_gemv_b200 as moe
    from synth import WORKLOADS, MoeShape
    from synth import gpu as sgpu

    moe.library_path = build_traced()
    L = moe.lib()
    L.moe_debug_pair_trace.argtypes = [ctypes.c_void_p, ctypes.c_int]
    L.moe_debug_pair_cycles.argtypes = [ctypes.c_void_p, ctypes.c_int]
    wl = WORKLOADS["decode"]
    b = wl.shape
    sh = MoeShape(b.d, b.f, b.E, b.k, b.n_shared, args.bits)
    T = args.tokens
    h = moe.MoeLayer(sh.d, sh.f, sh.E, sh.k, sh.n_shared, args.layers, sh.bits, T)
    keep = [sgpu.layer_device(sh, wl.master, l, wl.zipf) for l in range(args.layers)]
    for l, w in enumerate(keep):
        h.load_layer(l, *w)
    xs = [sgpu.x_device(sh, wl.master, 10000 + i, T) for i in range(8)]
    y = torch.empty(T, sh.d, dtype=torch.bfloat16, device="cuda")
    for i in range(20):
        h.forward(i % args.layers, xs[i % 8], y)
    torch.cuda.synchronize()
    G = torch.cuda.get_device_properties(0).multi_processor_count
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    print(f"# decode phase trace: d {sh.d}, E {sh.E}, k {sh.k}, f {sh.f}, {sh.bits}-bit, T = {T}; "
          f"{G} CTAs; cycles at {args.sm_mhz:.0f} MHz\n")
    for rep in range(args.reps):
        torch.cuda._sleep(10_000_000)  # the launch starts on an idle GPU, not behind the previous one
        ev0.record()
        h.forward(rep % args.layers, xs[rep % 8], y)
        ev1.record()
        torch.cuda.synchronize()
        if h.check_status() != 0:
            raise RuntimeError("device status set during the traced launch")
        tr = np.zeros(1024 * SLOTS, dtype=np.uint64)
        cy = np.zeros(1024 * CYC_SLOTS, dtype=np.uint64)
        if L.moe_debug_pair_trace(tr.ctypes.data, tr.size) or L.moe_debug_pair_cycles(cy.ctypes.data, cy.size):
            raise RuntimeError("reading the trace failed")
        tr = tr.reshape(1024, SLOTS)[:G].astype(np.int64)
        cy = cy.reshape(1024, CYC_SLOTS)[:G].astype(np.float64) / args.sm_mhz
        t0 = tr[:, 0].min()
        st = h.stats()
        print(f"## launch {rep}: {ev0.elapsed_time(ev1) * 1000:.1f} us between events, "
              f"{st['active_experts']} routed experts active\n")
        print("| boundary (us after the first CTA started) | CTAs | min | median | max |\n|---|---|---|---|---|")
        for s, name in BOUNDARIES.items():
            col = tr[:, s]
            ok = col >= t0  # stale stamps of earlier launches are older than this start
            if ok.sum() == 0:
                continue
            lo, md, hi = _stats((col[ok] - t0) / 1000.0)
            print(f"| {name} | {ok.sum()} | {lo:.2f} | {md:.2f} | {hi:.2f} |")
        print("\n| phase (us of SM cycles per CTA) | min | median | max |\n|---|---|---|---|")
        for s, name in CYCLES.items():
            lo, md, hi = _stats(cy[:, s])
            if hi > 0:
                print(f"| {name} | {lo:.2f} | {md:.2f} | {hi:.2f} |")
        print()
        tr[:] = 0
    h.close()
    return 0


if __name__ == "__main__":
    sys.exit(main())
