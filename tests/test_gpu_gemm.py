"""Parity of the tensor-core (tcgen05) path with the fp64 oracle.

The path runs for T > 16 tokens, or for any T with MOE_FORCE_GEMM: router
logits from a bf16 GEMM (certified against their error bound, then re-ranked
in fp64 where the order is open), grouped gate/up and down GEMMs over expert
groups with weights dequantised to fp16 in shared memory, and a fixed-order
combine of fp16 partial outputs.
"""
import numpy as np
import pytest

import oracle
import synth
from synth import WORKLOADS, MoeShape
from tests.gpu_util import (MAX_ABS, REL_L2, make_layer_host, max_abs, rel_l2, tile_cover_rows, upload_layer,
                            x_to_device, y_to_f64)

pytestmark = pytest.mark.gpu

# Routing weights: the tensor-core logits carry fp32 accumulation error
# (measured below 1.1e-5 on the full-shape layer, far inside the certified
# bound); a logit error e moves a renormalised weight by a factor within
# exp(+-2e), so 1e-4 relative leaves a 4x margin.
W_RTOL = 1e-4
# fp32 output: three fp16 roundings on the way (dequantised weight q*s when
# |q| > 2, h, the weighted partial outputs), each about 2e-4 relative rms;
# 8e-4 bounds their sum with margin.  The bf16 bar is the layer's own.
REL_L2_FP32_TC = 8e-4


@pytest.fixture(scope="module")
def torch_cuda():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import bit_expert_ffn_gemv_b200.build as b
    b.build()
    return torch


def _handle(shape, max_tokens, n_layers=1):
    import bit_expert_ffn_gemv_b200 as moe
    return moe.MoeLayer(shape.d, shape.f, shape.E, shape.k, shape.n_shared, n_layers, shape.bits, max_tokens)


def _check(torch, h, shape, L, x_bits, flags, label, sample=None):
    """Forward on all of x; compare routing of every token and outputs of `sample` rows (default all)."""
    import bit_expert_ffn_gemv_b200 as moe
    T = x_bits.shape[0]
    x = x_to_device(x_bits)
    y16 = h.forward(0, x, flags=flags)
    y32 = h.forward(0, x, flags=flags | moe.MOE_OUT_FP32)
    ids_f, w_f = h.last_routing(T)
    torch.cuda.synchronize()
    assert h.check_status() == 0, label
    rows = np.arange(T) if sample is None else np.asarray(sample)
    ids_all, w_all = oracle.route(shape, x_bits, L["router_w"], L["bias"])
    assert np.array_equal(ids_f.cpu().numpy(), ids_all), f"{label}: expert selection differs"
    assert np.allclose(w_f.cpu().numpy(), w_all, rtol=W_RTOL, atol=1e-7), label
    y_ref, _, _ = oracle.layer(shape, x_bits[rows], L["router_w"], L["bias"], L["codes"], L["scales"])
    g16, g32 = y_to_f64(y16)[rows], y_to_f64(y32)[rows]
    r16, m16, r32 = rel_l2(g16, y_ref), max_abs(g16, y_ref), rel_l2(g32, y_ref)
    print(f"{label} T={T} rows={len(rows)}: rel_l2 bf16 {r16:.3e} max_abs {m16:.3e} fp32 {r32:.3e} "
          f"stats {h.stats()}")
    assert r16 <= REL_L2 and m16 <= MAX_ABS, label
    assert r32 <= REL_L2_FP32_TC, label
    return y16, y32


# ------------------------------------------------------------------ tiny layer, every token
@pytest.fixture(scope="module")
def tiny(torch_cuda):
    wl = WORKLOADS["tiny"]
    L = make_layer_host(wl)
    dev = upload_layer(L)
    h = _handle(wl.shape, max_tokens=600)
    h.load_layer(0, *dev)
    yield wl, L, h
    h.close()


@pytest.mark.parametrize("T", [8, 1, 13, 64, 65, 300, 513])
def test_tiny_gemm(torch_cuda, tiny, T):
    """Token tiles of 256 with ragged tails; E = 16 fills only part of a 128-row router tile."""
    import bit_expert_ffn_gemv_b200 as moe
    wl, L, h = tiny
    x = synth.x_host(wl.shape, wl.master, 500 + T, T)
    _check(torch_cuda, h, wl.shape, L, x, moe.MOE_FORCE_GEMM, "tiny-gemm")


def test_tiny_gemm_matches_gemv(torch_cuda, tiny):
    """Both large-T paths compute the same layer; they differ only by rounding (fp16 vs fp32 partials)."""
    import bit_expert_ffn_gemv_b200 as moe
    wl, L, h = tiny
    x = x_to_device(synth.x_host(wl.shape, wl.master, 77, 200))
    a = h.forward(0, x, flags=moe.MOE_OUT_FP32 | moe.MOE_FORCE_GEMM)
    b = h.forward(0, x, flags=moe.MOE_OUT_FP32 | moe.MOE_FORCE_GEMV)
    torch_cuda.cuda.synchronize()
    assert rel_l2(y_to_f64(a), y_to_f64(b)) < REL_L2_FP32_TC


def test_tiny_gemm_deterministic(torch_cuda, tiny):
    import bit_expert_ffn_gemv_b200 as moe
    wl, L, h = tiny
    x = x_to_device(synth.x_host(wl.shape, wl.master, 78, 333))
    a = h.forward(0, x, flags=moe.MOE_OUT_FP32).clone()
    b = h.forward(0, x, flags=moe.MOE_OUT_FP32)
    torch_cuda.cuda.synchronize()
    assert torch_cuda.equal(a, b)


def test_gemm_accumulate_inplace(torch_cuda, tiny):
    """y == x with MOE_ACCUMULATE on the tensor-core path (x is read before y is written)."""
    import bit_expert_ffn_gemv_b200 as moe
    wl, L, h = tiny
    x = x_to_device(synth.x_host(wl.shape, wl.master, 79, 100))
    ref = (x.float() + h.forward(0, x, flags=moe.MOE_OUT_FP32)).to(torch_cuda.bfloat16)
    r = x.clone()
    h.forward(0, r, r, flags=moe.MOE_ACCUMULATE)
    torch_cuda.cuda.synchronize()
    assert torch_cuda.equal(r, ref)


def test_fp16_range_is_reported(torch_cuda, tiny):
    """An activation beyond the fp16 range sets MOE_ERR_RANGE instead of silently producing inf."""
    wl, L, h = tiny
    xb = synth.x_host(wl.shape, wl.master, 80, 100)
    xb[3, 5] = 0x4789  # bf16 70144.0 > 65504
    h.forward(0, x_to_device(xb))
    assert h.check_status() == 7
    assert h.check_status() == 0  # cleared


def test_uniform_routing_gemm(torch_cuda):
    """W_r = 0, no bias: every logit is exactly 0, the top-k is 0..k-1 with weights 1/k (all re-ranked)."""
    torch = torch_cuda
    sh = MoeShape(d=256, f=128, E=16, k=4, n_shared=1, bits=2)
    L = synth.layer_host(sh, 123, 0, False)
    L["router_w"][:] = 0
    h = _handle(sh, max_tokens=300)
    h.load_layer(0, *upload_layer(L))
    x = x_to_device(synth.x_host(sh, 5, 1, 300))
    ids, w = h.route(0, x)
    torch.cuda.synchronize()
    assert (ids.cpu().numpy() == np.arange(4)).all()
    assert (w.cpu().numpy() == 0.25).all()
    assert h.stats()["fixup_tokens"] == 300
    h.close()


@pytest.mark.parametrize("bits", [3, 4])
def test_small_layer_other_widths(torch_cuda, bits):
    """3- and 4-bit codes through the tensor-core path (several 128-row tiles in d and f)."""
    sh = MoeShape(d=512, f=256, E=32, k=4, n_shared=1, bits=bits)
    L = synth.layer_host(sh, 900 + bits, 0, True)
    h = _handle(sh, max_tokens=400)
    h.load_layer(0, *upload_layer(L))
    x = synth.x_host(sh, 900 + bits, 3, 400)
    _check(torch_cuda, h, sh, L, x, 0, f"b{bits}-gemm")
    h.close()


# ------------------------------------------------------------------ full-shape layer
@pytest.fixture(scope="module")
def full(torch_cuda):
    wl = WORKLOADS["prefill"]
    L = make_layer_host(wl)
    dev = upload_layer(L)
    h = _handle(wl.shape, max_tokens=8192)
    h.load_layer(0, *dev)
    yield wl, L, h, dev
    h.close()


@pytest.mark.parametrize("T", [16, 64, 1024])
def test_router_gemm_error_bound(torch_cuda, full, T):
    """Every tensor-core logit lies within the certified interval around the exact logit, at the
    batch's own K-chunk count (32 chunks at 16 tokens, 8 at 64, 4 at 128 or more)."""
    import bit_expert_ffn_gemv_b200 as moe
    wl, L, h, dev = full
    sh = wl.shape
    xb = synth.x_host(sh, wl.master, 11, T)
    lg = h.router_logits(0, x_to_device(xb), tensor_cores=True).cpu().numpy().astype(np.float64)
    _, _, exact = oracle.route(sh, xb, L["router_w"], L["bias"], with_logits=True)
    from tests.gpu_util import bf16_bits_to_f64
    xf = bf16_bits_to_f64(xb)
    wf = bf16_bits_to_f64(L["router_w"])
    depth = moe.moe_router_error_depth(sh.d, True, T)
    assert depth <= moe.moe_router_error_depth(sh.d, True)  # the any-batch bound is the loosest
    bound = 2 * depth * 2.0 ** -24 * (np.linalg.norm(xf, axis=1)[:, None] * np.linalg.norm(wf, axis=1)[None, :] +
                                      np.abs(L["bias"])[None, :])
    err = np.abs(lg - exact)
    print(f"tensor-core logits: max err {err.max():.3e}, max err / bound {(err / bound).max():.3e}")
    assert (err <= bound).all()


@pytest.mark.parametrize("T", [17, 33, 65, 1000, 8192])
def test_full_layer_gemm(torch_cuda, full, T):
    """Full shape (E = 512, k = 10, d = 2048, f = 768); outputs checked on tokens that cover every tile
    the tensor-core path forms (every expert group, every 256-token tile, every 32-row box of the small
    groups, the ragged ends), plus a random sample."""
    wl, L, h, dev = full
    x = synth.x_host(wl.shape, wl.master, 600 + T, T)
    ids, _ = oracle.route(wl.shape, x, L["router_w"], L["bias"])
    rng = np.random.default_rng(T)
    sample = np.unique(np.concatenate([tile_cover_rows(ids, wl.shape.E), rng.choice(T, size=min(T, 16),
                                                                                        replace=False)]))
    _check(torch_cuda, h, wl.shape, L, x, 0, "full-gemm", sample=sample)


def test_prefill_four_chunks(torch_cuda, full):
    """The 32K-token prompt as four consecutive 8192-token chunks through one handle, enqueued back to
    back; every chunk's routing checked on all tokens and its outputs on a tile-covering set of rows."""
    import bit_expert_ffn_gemv_b200 as moe
    torch = torch_cuda
    wl, L, h, dev = full
    sh, T = wl.shape, 8192
    xs = [synth.x_host(sh, wl.master, 800 + c, T) for c in range(wl.chunks)]
    xd = [x_to_device(xb) for xb in xs]
    outs = []
    for x in xd:  # no synchronisation between the chunks
        y16 = h.forward(0, x)
        y32 = h.forward(0, x, flags=moe.MOE_OUT_FP32)
        outs.append((y16, y32))
    ids_gpu = [h.route(0, x)[0] for x in xd]
    torch.cuda.synchronize()
    assert h.check_status() == 0
    for c, xb in enumerate(xs):
        ids_ref, _ = oracle.route(sh, xb, L["router_w"], L["bias"])
        assert np.array_equal(ids_gpu[c].cpu().numpy(), ids_ref), f"chunk {c}: expert selection differs"
        rows = tile_cover_rows(ids_ref, sh.E)
        y_ref, _, _ = oracle.layer(sh, xb[rows], L["router_w"], L["bias"], L["codes"], L["scales"])
        g16, g32 = y_to_f64(outs[c][0])[rows], y_to_f64(outs[c][1])[rows]
        r16, m16, r32 = rel_l2(g16, y_ref), max_abs(g16, y_ref), rel_l2(g32, y_ref)
        print(f"chunk {c} rows={len(rows)}: rel_l2 bf16 {r16:.3e} max_abs {m16:.3e} fp32 {r32:.3e}")
        assert r16 <= REL_L2 and m16 <= MAX_ABS, c
        assert r32 <= REL_L2_FP32_TC, c


def test_full_layer_forced_small(torch_cuda, full):
    """MOE_FORCE_GEMM on a handful of tokens: groups of one token (N = 16 MMAs)."""
    import bit_expert_ffn_gemv_b200 as moe
    wl, L, h, dev = full
    x = synth.x_host(wl.shape, wl.master, 700, 4)
    _check(torch_cuda, h, wl.shape, L, x, moe.MOE_FORCE_GEMM, "full-gemm-T4")
