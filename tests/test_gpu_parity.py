"""Parity of the CUDA path (through the C ABI) with the fp64 oracle."""
import numpy as np
import pytest

import oracle
import synth
from synth import WORKLOADS, MoeShape
from tests.gpu_util import (MAX_ABS, REL_L2, REL_L2_FP32, bf16_bits_to_f64, make_layer_host, max_abs, rel_l2,
                            upload_layer, x_to_device, y_to_f64)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import bit_expert_ffn_gemv_b200.build as b
    b.build()
    return torch


def _handle(shape, n_layers=1, max_tokens=64):
    import bit_expert_ffn_gemv_b200 as moe
    return moe.MoeLayer(shape.d, shape.f, shape.E, shape.k, shape.n_shared, n_layers, shape.bits, max_tokens)


def _check_layer(torch, h, shape, L, x_bits, layer=0, flags_extra=0, label=""):
    import bit_expert_ffn_gemv_b200 as moe
    T = x_bits.shape[0]
    x = x_to_device(x_bits)
    y_ref, ids_ref, w_ref = oracle.layer(shape, x_bits, L["router_w"], L["bias"], L["codes"], L["scales"])
    ids, w = h.route(layer, x)
    torch.cuda.synchronize()
    assert np.array_equal(ids.cpu().numpy(), ids_ref), f"{label}: expert selection differs"
    assert np.allclose(w.cpu().numpy(), w_ref, rtol=2e-6, atol=1e-7), label
    y16 = h.forward(layer, x, flags=flags_extra)
    y32 = h.forward(layer, x, flags=moe.MOE_OUT_FP32 | flags_extra)
    ids_f, w_f = h.last_routing(T)
    torch.cuda.synchronize()
    # above 16 tokens (unless forced onto the CUDA-core paths) moe_forward takes the
    # tensor-core path: fp32 tensor-core logits (1e-4 on the weights) and fp16 operands
    tc = T > 16 and not (flags_extra & (moe.MOE_FORCE_GEMV | moe.MOE_FORCE_UNFUSED))
    assert np.array_equal(ids_f.cpu().numpy(), ids_ref), f"{label}: forward's expert selection differs"
    assert np.allclose(w_f.cpu().numpy(), w_ref, rtol=1e-4 if tc else 2e-6, atol=1e-7), label
    assert h.check_status() == 0
    g16, g32 = y_to_f64(y16), y_to_f64(y32)
    r16, m16, r32 = rel_l2(g16, y_ref), max_abs(g16, y_ref), rel_l2(g32, y_ref)
    print(f"{label} T={T}: rel_l2 bf16 {r16:.3e} max_abs {m16:.3e} fp32 {r32:.3e} stats {h.stats()}")
    assert r16 <= REL_L2 and m16 <= MAX_ABS, label
    assert r32 <= (8e-4 if tc else REL_L2_FP32), label
    return y16, y32


# ------------------------------------------------------------------ tiny layer
@pytest.fixture(scope="module")
def tiny(torch_cuda):
    wl = WORKLOADS["tiny"]
    L = make_layer_host(wl)
    dev = upload_layer(L)
    h = _handle(wl.shape, max_tokens=64)
    h.load_layer(0, *dev)
    yield wl, L, h
    h.close()


@pytest.mark.parametrize("T", [8, 1, 3, 13, 64])
def test_tiny_layer(torch_cuda, tiny, T):
    wl, L, h = tiny
    x = synth.x_host(wl.shape, wl.master, 100 + T, T)
    _check_layer(torch_cuda, h, wl.shape, L, x, label="tiny")


def test_tiny_dequant_bit_exact(torch_cuda, tiny):
    wl, L, h = tiny
    sh = wl.shape
    for e in range(sh.E + sh.n_shared):
        cb = synth.codes_bytes(sh.f, sh.d, sh.bits)
        sb = sh.f * sh.d // 32
        for m in range(3):
            N, K = synth.mat_dims(sh, m)
            got = h.debug_dequant(0, e, m).cpu().numpy().astype(np.float64)
            want = oracle.dequant(L["codes"][e][m * cb:(m + 1) * cb], L["scales"][e][m * sb:(m + 1) * sb], N, K,
                                  sh.bits)
            assert np.array_equal(got, want), (e, m)


def test_zero_tokens_is_a_noop(torch_cuda, tiny):
    wl, L, h = tiny
    import bit_expert_ffn_gemv_b200 as moe
    y = torch_cuda.full((1, wl.shape.d), 7.0, device="cuda", dtype=torch_cuda.float32)
    moe.moe_forward(h.handle, 0, 0, 0, y.data_ptr(), moe.MOE_OUT_FP32, 0)
    torch_cuda.cuda.synchronize()
    assert (y == 7.0).all()


def test_too_many_tokens_rejected(torch_cuda, tiny):
    wl, L, h = tiny
    import bit_expert_ffn_gemv_b200 as moe
    x = x_to_device(synth.x_host(wl.shape, wl.master, 5, 65))
    with pytest.raises(moe.MoeError) as ei:
        h.forward(0, x)
    assert ei.value.status == 1


def test_accumulate_and_host_buffers(torch_cuda, tiny):
    wl, L, h = tiny
    import bit_expert_ffn_gemv_b200 as moe
    torch = torch_cuda
    T = 8
    xb = synth.x_host(wl.shape, wl.master, 7, T)
    x = x_to_device(xb)
    base = torch.randn(T, wl.shape.d, device="cuda", dtype=torch.float32)
    y = base.clone()
    h.forward(0, x, y, flags=moe.MOE_OUT_FP32 | moe.MOE_ACCUMULATE)
    plain = h.forward(0, x, flags=moe.MOE_OUT_FP32)
    torch.cuda.synchronize()
    assert torch.allclose(y, base + plain, rtol=0, atol=1e-6)
    # host buffers: identical kernels, so identical bits
    xh = x.cpu().pin_memory()
    yh = torch.empty(T, wl.shape.d, dtype=torch.float32).pin_memory()
    h.forward_host(0, xh, yh, flags=moe.MOE_OUT_FP32)
    assert torch.equal(yh, plain.cpu())


def test_deterministic(torch_cuda, tiny):
    wl, L, h = tiny
    import bit_expert_ffn_gemv_b200 as moe
    x = x_to_device(synth.x_host(wl.shape, wl.master, 9, 13))
    a = h.forward(0, x, flags=moe.MOE_OUT_FP32).clone()
    b = h.forward(0, x, flags=moe.MOE_OUT_FP32)
    assert torch_cuda.equal(a, b)


def test_uniform_routing_closed_form(torch_cuda):
    """W_r = 0, no bias: every logit is exactly 0, so ids = 0..k-1 and w = 1/k."""
    torch = torch_cuda
    sh = MoeShape(d=256, f=128, E=16, k=4, n_shared=1, bits=2)
    L = synth.layer_host(sh, 123, 0, False)
    L["router_w"][:] = 0
    dev = upload_layer(L)
    h = _handle(sh, max_tokens=16)
    h.load_layer(0, *dev)
    x = x_to_device(synth.x_host(sh, 5, 1, 16))
    ids, w = h.route(0, x)
    torch.cuda.synchronize()
    assert (ids.cpu().numpy() == np.arange(4)).all()
    assert (w.cpu().numpy() == 0.25).all()
    assert h.stats()["fixup_tokens"] == 16
    h.close()


# ------------------------------------------------------------------ full-shape decode layer
@pytest.fixture(scope="module")
def decode_layer(torch_cuda):
    wl = WORKLOADS["decode"]
    L = make_layer_host(wl)
    dev = upload_layer(L)
    h = _handle(wl.shape, max_tokens=64)
    h.load_layer(0, *dev)
    yield wl, L, h
    h.close()


@pytest.mark.parametrize("T", [1, 4, 16, 64, 7, 33])
def test_decode_layer(torch_cuda, decode_layer, T):
    """The fused persistent kernel (the default up to 16 tokens, MOE_FORCE_GEMV up to 64)."""
    import bit_expert_ffn_gemv_b200 as moe
    wl, L, h = decode_layer
    x = synth.x_host(wl.shape, wl.master, 200 + T, T)
    _check_layer(torch_cuda, h, wl.shape, L, x, flags_extra=moe.MOE_FORCE_GEMV if T > 16 else 0, label="decode")


@pytest.mark.parametrize("T", [1, 4, 64])
def test_decode_layer_unfused(torch_cuda, decode_layer, T):
    """The one-kernel-per-step path meets the same bar, and agrees with the fused kernel to fp32 rounding."""
    import bit_expert_ffn_gemv_b200 as moe
    wl, L, h = decode_layer
    xb = synth.x_host(wl.shape, wl.master, 400 + T, T)
    _check_layer(torch_cuda, h, wl.shape, L, xb, flags_extra=moe.MOE_FORCE_UNFUSED, label="decode-unfused")
    x = x_to_device(xb)
    a = h.forward(0, x, flags=moe.MOE_OUT_FP32 | moe.MOE_FORCE_GEMV)  # the fused kernel up to 64 tokens
    b = h.forward(0, x, flags=moe.MOE_OUT_FP32 | moe.MOE_FORCE_UNFUSED)
    torch_cuda.cuda.synchronize()
    assert rel_l2(y_to_f64(a), y_to_f64(b)) < 1e-5


def test_inplace_residual(torch_cuda, decode_layer):
    """y == x with MOE_ACCUMULATE updates a residual stream in place."""
    import bit_expert_ffn_gemv_b200 as moe
    wl, L, h = decode_layer
    x = x_to_device(synth.x_host(wl.shape, wl.master, 77, 4))
    ref = (x.float() + h.forward(0, x, flags=moe.MOE_OUT_FP32)).to(torch_cuda.bfloat16)
    r = x.clone()
    h.forward(0, r, r, flags=moe.MOE_ACCUMULATE)
    torch_cuda.cuda.synchronize()
    assert torch_cuda.equal(r, ref)
