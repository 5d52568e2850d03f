"""Full-shape parity beyond one 2-bit layer: the 48-layer residual chain and 3/4-bit layers.

The oracle materialises only the experts the checked tokens select (plus the
shared one), so full-shape layers stay cheap on the host; the GPU holds
every layer, generated on the device by the bit-identical generator twin.
"""
import numpy as np
import pytest

import oracle
import synth
from synth import WORKLOADS, MoeShape
from tests.gpu_util import MAX_ABS, REL_L2, max_abs, rel_l2, tile_cover_rows, x_to_device, y_to_f64

pytestmark = pytest.mark.gpu

REL_L2_FP32 = 5e-4     # fused decode path: fp16 h, fp32 sums
REL_L2_FP32_TC = 8e-4  # tensor-core path: fp16 operands and partials


@pytest.fixture(scope="module")
def torch_cuda():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import bit_expert_ffn_gemv_b200.build as b
    b.build()
    return torch


def _host_layer(shape, master, layer, zipf, x_bits):
    """Router + the experts the tokens of x select (and the shared expert), on the host."""
    wr, bias = synth.router_host(shape, master, layer, zipf)
    ids, _ = oracle.route(shape, x_bits, wr, bias)
    return synth.layer_host(shape, master, layer, zipf, experts=set(ids.ravel().tolist()) | {shape.E})


def _compare(shape, L, x_bits, y32, y16=None, label="", fp32_tol=REL_L2_FP32, rows=None, scaled_abs=False):
    """scaled_abs: the max-abs bar is the larger of MAX_ABS and one bf16 ulp (2^-7 relative) of the
    largest output -- deep in the residual chain outputs reach |y| ~ 30, where rounding y itself to
    bf16 already costs more than MAX_ABS."""
    rows = np.arange(x_bits.shape[0]) if rows is None else np.asarray(rows)
    y_ref, _, _ = oracle.layer(shape, x_bits[rows], L["router_w"], L["bias"], L["codes"], L["scales"])
    g32 = y_to_f64(y32)[rows]
    r32, m32 = rel_l2(g32, y_ref), max_abs(g32, y_ref)
    msg = f"{label}: rel_l2 fp32 {r32:.3e} max_abs fp32 {m32:.3e}"
    if y16 is not None:
        g16 = y_to_f64(y16)[rows]
        r16, m16 = rel_l2(g16, y_ref), max_abs(g16, y_ref)
        bar = max(MAX_ABS, 2.0 ** -7 * float(np.abs(y_ref).max())) if scaled_abs else MAX_ABS
        msg += f" bf16 {r16:.3e} max_abs {m16:.3e} (bar {bar:.3e}, max|y| {np.abs(y_ref).max():.2f})"
        assert r16 <= REL_L2 and m16 <= bar, msg
    print(msg)
    # the fp32 output carries no bf16 rounding of y: held to the absolute bar at any |y|
    assert r32 <= fp32_tol and m32 <= MAX_ABS, msg


# ------------------------------------------------------------------ 48-layer chain
@pytest.fixture(scope="module")
def chain(torch_cuda):
    from synth import gpu as sgpu
    import bit_expert_ffn_gemv_b200 as moe
    wl = WORKLOADS["chain48"]
    sh = wl.shape
    h = moe.MoeLayer(sh.d, sh.f, sh.E, sh.k, sh.n_shared, wl.layers, sh.bits, 4)
    keep = []
    for l in range(wl.layers):
        w = sgpu.layer_device(sh, wl.master, l, wl.zipf)
        h.load_layer(l, *w)
        keep.append(w)
    yield wl, h
    h.close()


def test_rms_normalize(torch_cuda):
    """The chain's pre-norm helper: bf16(x / sqrt(mean x^2 + 1e-6)) per row, within one bf16 rounding."""
    import bit_expert_ffn_gemv_b200 as moe
    torch = torch_cuda
    x = x_to_device(synth.x_host(MoeShape(2048, 768, 512, 10, 1, 2), 7, 3, 33)) * 3
    u = moe.rms_normalize(x)
    xf = x.double()
    ref = xf / torch.sqrt((xf * xf).mean(dim=1, keepdim=True) + 1e-6)
    assert ((u.double() - ref).abs() <= ref.abs() * 2.0 ** -8 + 1e-30).all()


@pytest.mark.parametrize("T", [1, 4])
def test_chain48_teacher_forced(torch_cuda, chain, T):
    """Residual chain through 48 layers: u_l = rmsnorm(x_l), x_{l+1} = bf16(x_l + y_l(u_l)), the
    residual updated in place; sampled layers checked against the oracle on the GPU's own u_l
    (teacher forcing), and the residual update checked exactly."""
    import bit_expert_ffn_gemv_b200 as moe
    torch = torch_cuda
    wl, h = chain
    sh = wl.shape
    checked = {0, 17, 47}
    r = x_to_device(synth.x_host(sh, wl.master, 1, T))
    u = torch.empty_like(r)
    saved = {}
    for l in range(wl.layers):
        moe.rms_normalize(r, u)
        if l in checked:
            saved[l] = (r.clone(), u.clone())
        h.forward(l, u, r, flags=moe.MOE_ACCUMULATE)
    torch.cuda.synchronize()
    assert h.check_status() == 0
    assert torch.isfinite(r.float()).all()
    for l in sorted(checked):
        xl, ul = saved[l]
        y32 = h.forward(l, ul, flags=moe.MOE_OUT_FP32)
        y16 = h.forward(l, ul)
        # the residual step equals bf16(x_l + y_l)
        step = xl.clone()
        h.forward(l, ul, step, flags=moe.MOE_ACCUMULATE)
        torch.cuda.synchronize()
        assert torch.equal(step, (xl.float() + y32).to(torch.bfloat16)), l
        ub = ul.cpu().view(torch.int16).numpy().view(np.uint16)
        L = _host_layer(sh, wl.master, l, wl.zipf, ub)
        h.forward(l, ul)
        ids, _ = h.last_routing(T)
        ids_ref, _ = oracle.route(sh, ub, L["router_w"], L["bias"])
        assert np.array_equal(ids.cpu().numpy(), ids_ref), f"layer {l}: expert selection differs"
        _compare(sh, L, ub, y32, y16, label=f"chain48 T={T} layer {l}", scaled_abs=True)


# ------------------------------------------------------------------ 3- and 4-bit full-shape layers
@pytest.fixture(scope="module", params=[3, 4])
def wide(torch_cuda, request):
    from synth import gpu as sgpu
    import bit_expert_ffn_gemv_b200 as moe
    wl = WORKLOADS["sweep"]
    b = wl.shape
    sh = MoeShape(b.d, b.f, b.E, b.k, b.n_shared, request.param)
    w = sgpu.layer_device(sh, wl.master, 0, wl.zipf)
    h = moe.MoeLayer(sh.d, sh.f, sh.E, sh.k, sh.n_shared, 1, sh.bits, 8192)
    h.load_layer(0, *w)
    yield wl, sh, h, w
    h.close()


@pytest.mark.parametrize("T", [1, 4, 16, 64, 512, 8192])
def test_wide_full_layer(torch_cuda, wide, T):
    """3/4-bit full shape at every batch of the sweep: fused decode path up to 16 tokens, tensor-core path
    above; every row up to 64 tokens, above that rows covering every tile the tensor-core path forms."""
    import bit_expert_ffn_gemv_b200 as moe
    wl, sh, h, w = wide
    xb = synth.x_host(sh, wl.master, 300 + T, T)
    if T <= 64:
        rows = np.arange(T)
    else:
        wr, bias = synth.router_host(sh, wl.master, 0, wl.zipf)
        rows = tile_cover_rows(oracle.route(sh, xb, wr, bias)[0], sh.E)
    x = x_to_device(xb)
    y32 = h.forward(0, x, flags=moe.MOE_OUT_FP32)
    y16 = h.forward(0, x)
    ids, _ = h.last_routing(T)
    torch_cuda.cuda.synchronize()
    assert h.check_status() == 0
    L = _host_layer(sh, wl.master, 0, wl.zipf, xb[rows])
    ids_ref, _ = oracle.route(sh, xb, L["router_w"], L["bias"])
    assert np.array_equal(ids.cpu().numpy(), ids_ref), f"b{sh.bits} T={T}: expert selection differs"
    _compare(sh, L, xb, y32, y16, label=f"b{sh.bits} T={T}", rows=rows,
             fp32_tol=REL_L2_FP32 if T <= 16 else REL_L2_FP32_TC)


# ------------------------------------------------------------------ Coder shape (256 routed experts)
@pytest.fixture(scope="module")
def coder(torch_cuda):
    from synth import gpu as sgpu
    import bit_expert_ffn_gemv_b200 as moe
    wl = WORKLOADS["sweep"]
    b = wl.shape
    sh = MoeShape(b.d, b.f, 256, b.k, b.n_shared, 2)
    w = sgpu.layer_device(sh, wl.master + 256, 0, wl.zipf)
    h = moe.MoeLayer(sh.d, sh.f, sh.E, sh.k, sh.n_shared, 1, sh.bits, 512)
    h.load_layer(0, *w)
    yield wl, sh, h
    h.close()


@pytest.mark.parametrize("T", [1, 4, 16, 64, 512])
def test_coder_shape_layer(torch_cuda, coder, T):
    """E = 256 (the Coder variant keeps 256 of the 512 experts), k = 10, d = 2048, f = 768: fused decode
    path up to 16 tokens, tensor-core path above (sampled rows at 512)."""
    import bit_expert_ffn_gemv_b200 as moe
    wl, sh, h = coder
    master = wl.master + 256
    xb = synth.x_host(sh, master, 700 + T, T)
    rows = np.arange(T) if T <= 64 else np.unique(np.r_[0, T - 1, np.random.default_rng(T).choice(T, 30, False)])
    x = x_to_device(xb)
    y32 = h.forward(0, x, flags=moe.MOE_OUT_FP32)
    y16 = h.forward(0, x)
    ids, _ = h.last_routing(T)
    torch_cuda.cuda.synchronize()
    assert h.check_status() == 0
    L = _host_layer(sh, master, 0, wl.zipf, xb[rows])
    ids_ref, _ = oracle.route(sh, xb, L["router_w"], L["bias"])
    assert np.array_equal(ids.cpu().numpy(), ids_ref), f"E=256 T={T}: expert selection differs"
    _compare(sh, L, xb, y32, y16, label=f"E=256 T={T}", rows=rows,
             fp32_tol=REL_L2_FP32 if T <= 16 else REL_L2_FP32_TC)


# ------------------------------------------------------------------ pre-norm input (MOE_NORM_INPUT)
@pytest.fixture(scope="module")
def decode_layer(torch_cuda):
    from synth import gpu as sgpu
    import bit_expert_ffn_gemv_b200 as moe
    wl = WORKLOADS["decode"]
    sh = wl.shape
    h = moe.MoeLayer(sh.d, sh.f, sh.E, sh.k, sh.n_shared, 1, sh.bits, 512)
    w = sgpu.layer_device(sh, wl.master, 0, wl.zipf)
    h.load_layer(0, *w)
    yield wl, h, w
    h.close()


@pytest.mark.parametrize("T,path", [(1, "default"), (4, "default"), (16, "default"), (4, "unfused"),
                                    (40, "gemv"), (40, "default"), (300, "default")])
def test_norm_input_is_the_two_call_sequence(torch_cuda, decode_layer, T, path):
    """forward(x, MOE_NORM_INPUT) is bit for bit moe_rms_normalize then forward, on every path (the
    clustered decode kernel normalises inside its launch, the others run the norm kernel first), and
    with MOE_ACCUMULATE in place it is one residual step."""
    import bit_expert_ffn_gemv_b200 as moe
    torch = torch_cuda
    wl, h, _ = decode_layer
    sh = wl.shape
    pf = {"default": 0, "unfused": moe.MOE_FORCE_UNFUSED, "gemv": moe.MOE_FORCE_GEMV}[path]
    x = x_to_device(synth.x_host(sh, wl.master, 900 + T, T)) * 3
    u = moe.rms_normalize(x)
    for out in (0, moe.MOE_OUT_FP32):
        ref = h.forward(0, u, flags=pf | out)
        got = h.forward(0, x, flags=pf | out | moe.MOE_NORM_INPUT)
        torch.cuda.synchronize()
        assert h.check_status() == 0
        assert torch.equal(got.view(torch.int16 if got.dtype != torch.float32 else torch.int32),
                           ref.view(torch.int16 if ref.dtype != torch.float32 else torch.int32)), (T, path, out)
    r = x.clone()
    h.forward(0, r, r, flags=pf | moe.MOE_ACCUMULATE | moe.MOE_NORM_INPUT)
    y32 = h.forward(0, u, flags=pf | moe.MOE_OUT_FP32)
    torch.cuda.synchronize()
    assert torch.equal(r, (x.float() + y32).to(torch.bfloat16)), (T, path)


@pytest.mark.parametrize("T", [1, 4])
def test_chain48_with_norm_input_equals_two_calls(torch_cuda, chain, T):
    """The 48-layer chain as one call per layer (MOE_NORM_INPUT | MOE_ACCUMULATE, in place) ends bit for
    bit where the two-call chain (norm, then layer) ends."""
    import bit_expert_ffn_gemv_b200 as moe
    torch = torch_cuda
    wl, h = chain
    sh = wl.shape
    x0 = x_to_device(synth.x_host(sh, wl.master, 2, T))
    r1, r2 = x0.clone(), x0.clone()
    u = torch.empty_like(x0)
    for l in range(wl.layers):
        moe.rms_normalize(r1, u)
        h.forward(l, u, r1, flags=moe.MOE_ACCUMULATE)
        h.forward(l, r2, r2, flags=moe.MOE_ACCUMULATE | moe.MOE_NORM_INPUT)
    torch.cuda.synchronize()
    assert h.check_status() == 0
    assert torch.isfinite(r2.float()).all()
    assert torch.equal(r1, r2)
