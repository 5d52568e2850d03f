"""Route-tail skip (MOE_ROUTE_TAIL_SKIP) on every path, against the oracle with the same drop rule.

The oracle decides the dropped experts from its own routing of the whole batch
(oracle.tail_skip) and evaluates the layer without their terms; the GPU must
select the same experts, compute only the kept ones (checked through the
active-expert count) and match that sum.  Each case also prints how far the
approximation moves the output from the full layer.
"""
import numpy as np
import pytest

import oracle
import synth
from synth import WORKLOADS, MoeShape
from tests.gpu_util import MAX_ABS, REL_L2, REL_L2_FP32, max_abs, rel_l2, upload_layer, x_to_device, y_to_f64

pytestmark = pytest.mark.gpu

REL_L2_FP32_TC = 8e-4  # tensor-core path: fp16 operands and partials
SMALL = MoeShape(d=256, f=128, E=64, k=10, n_shared=1, bits=2)
WIDE_E = MoeShape(d=256, f=128, E=1024, k=10, n_shared=1, bits=2)


@pytest.fixture(scope="module")
def torch_cuda():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import bit_expert_ffn_gemv_b200.build as b
    b.build()
    return torch


def _check(torch, h, shape, L, xb, flags, tc, label, rows=None):
    import bit_expert_ffn_gemv_b200 as moe
    T = xb.shape[0]
    x = x_to_device(xb)
    fl = flags | moe.MOE_ROUTE_TAIL_SKIP
    y32 = h.forward(0, x, flags=fl | moe.MOE_OUT_FP32)
    y16 = h.forward(0, x, flags=fl)
    ids_g, _ = h.last_routing(T)
    torch.cuda.synchronize()
    assert h.check_status() == 0, label
    st = h.stats()
    ids, _ = oracle.route(shape, xb, L["router_w"], L["bias"])
    assert np.array_equal(ids_g.cpu().numpy(), ids), f"{label}: expert selection differs"
    drop = oracle.tail_skip(ids, shape.E, moe.MOE_TAIL_SKIP_RANK)
    kept = np.setdiff1d(np.unique(ids), np.flatnonzero(drop))
    assert drop.any(), f"{label}: the batch drops nothing, so it tests nothing"
    assert st["active_experts"] == kept.size, (label, st, kept.size)
    rows = np.arange(T) if rows is None else np.asarray(rows)
    y_ref, _, _ = oracle.layer(shape, xb[rows], L["router_w"], L["bias"], L["codes"], L["scales"], drop=drop)
    y_full, _, _ = oracle.layer(shape, xb[rows], L["router_w"], L["bias"], L["codes"], L["scales"])
    g16, g32 = y_to_f64(y16)[rows], y_to_f64(y32)[rows]
    r16, m16, r32 = rel_l2(g16, y_ref), max_abs(g16, y_ref), rel_l2(g32, y_ref)
    print(f"{label} T={T}: dropped {int(drop.sum())} of {np.unique(ids).size} experts "
          f"({int(drop[ids].sum())} of {ids.size} pairs); rel_l2 bf16 {r16:.3e} fp32 {r32:.3e}; "
          f"deviation from the full layer {rel_l2(y_ref, y_full):.3e}")
    assert r16 <= REL_L2 and m16 <= MAX_ABS, label
    assert r32 <= (REL_L2_FP32_TC if tc else REL_L2_FP32), label
    # without the flag the same handle computes the full layer again
    yf = h.forward(0, x, flags=flags | moe.MOE_OUT_FP32)
    torch.cuda.synchronize()
    assert rel_l2(y_to_f64(yf)[rows], y_full) <= (REL_L2_FP32_TC if tc else REL_L2_FP32), label


def _layer(shape, master, max_tokens):
    import bit_expert_ffn_gemv_b200 as moe
    L = synth.layer_host(shape, master, 0, True)
    h = moe.MoeLayer(shape.d, shape.f, shape.E, shape.k, shape.n_shared, 1, shape.bits, max_tokens)
    h.load_layer(0, *upload_layer(L))
    return L, h


@pytest.fixture(scope="module")
def small(torch_cuda):
    L, h = _layer(SMALL, 4242, 256)
    yield L, h
    h.close()


@pytest.mark.parametrize("T,seed,path", [(1, 1, "fused"), (4, 1, "fused"), (16, 2, "fused"), (4, 1, "unfused"),
                                         (64, 3, "gemv"), (200, 4, "gemv"), (40, 3, "gemm"), (200, 4, "gemm")])
def test_tail_skip_small(torch_cuda, small, T, seed, path):
    """E = 64, k = 10 through each path: the fused kernel, the one-kernel-per-step GEMV path, the fused
    kernel / grouped GEMV forced onto CUDA cores above 16 tokens, and the tensor-core path."""
    import bit_expert_ffn_gemv_b200 as moe
    L, h = small
    flags = {"fused": 0, "unfused": moe.MOE_FORCE_UNFUSED, "gemv": moe.MOE_FORCE_GEMV,
             "gemm": moe.MOE_FORCE_GEMM}[path]
    xb = synth.x_host(SMALL, 4242, seed, T)
    _check(torch_cuda, h, SMALL, L, xb, flags, path == "gemm", f"tail-skip {path}")


@pytest.mark.parametrize("path", ["gemm", "gemv"])
def test_tail_skip_multi_cta_bucket(torch_cuda, path):
    """E = 1024 and T * k = 9000 >= 8192 pairs: the three-kernel bucketing carries the per-chunk best
    ranks through its scan."""
    import bit_expert_ffn_gemv_b200 as moe
    L, h = _layer(WIDE_E, 4242, 900)
    try:
        xb = synth.x_host(WIDE_E, 4242, 5, 900)
        rows = np.unique(np.r_[0, 899, np.random.default_rng(9).choice(900, 40, False)])
        flags = moe.MOE_FORCE_GEMM if path == "gemm" else moe.MOE_FORCE_GEMV
        _check(torch_cuda, h, WIDE_E, L, xb, flags, path == "gemm", f"tail-skip wide-E {path}", rows=rows)
    finally:
        h.close()


@pytest.mark.parametrize("T", [1, 4, 16])
def test_tail_skip_full_shape_decode(torch_cuda, T):
    """The full-shape layer (E = 512, k = 10, d = 2048, f = 768) at decode batch sizes."""
    import bit_expert_ffn_gemv_b200 as moe
    from synth import gpu as sgpu
    wl = WORKLOADS["decode"]
    sh = wl.shape
    h = moe.MoeLayer(sh.d, sh.f, sh.E, sh.k, sh.n_shared, 1, sh.bits, 16)
    try:
        h.load_layer(0, *sgpu.layer_device(sh, wl.master, 0, wl.zipf))
        xb = synth.x_host(sh, wl.master, 1, T)
        wr, bias = synth.router_host(sh, wl.master, 0, wl.zipf)
        ids, _ = oracle.route(sh, xb, wr, bias)
        L = synth.layer_host(sh, wl.master, 0, wl.zipf, experts=set(ids.ravel().tolist()) | {sh.E})
        _check(torch_cuda, h, sh, L, xb, 0, False, "tail-skip full-shape")
    finally:
        h.close()
