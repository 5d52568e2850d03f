"""Per-tensor mixed code widths (gate/up at one width, down at another) against the oracle.

Every path reads each matrix at its own width: the fused decode kernel up to
16 tokens, the tensor-core grouped GEMM above (or forced), the grouped GEMV
when forced.  The tests cover the dequantisation of each matrix, the layer on
each path at decode and batch sizes, and the full-shape layer on the fused and
tensor-core paths.
"""
import numpy as np
import pytest

import oracle
import synth
from synth import WORKLOADS, MoeShape
from tests.gpu_util import MAX_ABS, REL_L2, REL_L2_FP32, max_abs, rel_l2, upload_layer, x_to_device, y_to_f64

REL_L2_FP32_TC = 8e-4  # tensor-core path: fp16 operands and partials

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import bit_expert_ffn_gemv_b200.build as b
    b.build()
    return torch


def _handle(sh, max_tokens):
    import bit_expert_ffn_gemv_b200 as moe
    return moe.MoeLayer(sh.d, sh.f, sh.E, sh.k, sh.n_shared, 1, sh.bits, max_tokens, bits_down=sh.bits_down)


def _check(torch, h, sh, L, xb, label, flags=0):
    import bit_expert_ffn_gemv_b200 as moe
    T = xb.shape[0]
    x = x_to_device(xb)
    y16 = h.forward(0, x, flags=flags)
    y32 = h.forward(0, x, flags=flags | moe.MOE_OUT_FP32)
    ids, _ = h.last_routing(T)
    torch.cuda.synchronize()
    assert h.check_status() == 0, label
    y_ref, ids_ref, _ = oracle.layer(sh, xb, L["router_w"], L["bias"], L["codes"], L["scales"])
    assert np.array_equal(ids.cpu().numpy(), ids_ref), f"{label}: expert selection differs"
    g16, g32 = y_to_f64(y16), y_to_f64(y32)
    r16, m16, r32 = rel_l2(g16, y_ref), max_abs(g16, y_ref), rel_l2(g32, y_ref)
    print(f"{label} T={T}: rel_l2 bf16 {r16:.3e} max_abs {m16:.3e} fp32 {r32:.3e}")
    assert r16 <= REL_L2 and m16 <= MAX_ABS, label
    tc = (T > 16 and not flags & (moe.MOE_FORCE_GEMV | moe.MOE_FORCE_UNFUSED)) or flags & moe.MOE_FORCE_GEMM
    assert r32 <= (REL_L2_FP32_TC if tc else REL_L2_FP32), label


@pytest.mark.parametrize("bits,bits_down", [(2, 3), (2, 4), (3, 2)])
def test_mixed_small_layer(torch_cuda, bits, bits_down):
    import bit_expert_ffn_gemv_b200 as moe
    torch = torch_cuda
    sh = MoeShape(d=256, f=128, E=32, k=4, n_shared=1, bits=bits, bits_down=bits_down)
    L = synth.layer_host(sh, 5000 + 10 * bits + bits_down, 0, True)
    h = _handle(sh, 300)
    try:
        h.load_layer(0, *upload_layer(L))
        # every matrix of two experts dequantises bit-exactly at its own width
        for e in (3, sh.E):
            blk = L["codes"][e]
            mc = sh.f * sh.d * bits // 8
            for mat in range(3):
                N, K = synth.mat_dims(sh, mat)
                b = synth.mat_bits(sh, mat)
                c = blk[mat * mc: mat * mc + N * K * b // 8]
                s = L["scales"][e][mat * (N * K // 32):(mat + 1) * (N * K // 32)]
                got = torch.empty(N, K, dtype=torch.float32, device="cuda")
                moe.moe_debug_dequant(h.handle, 0, e, mat, got.data_ptr(), 0)
                torch.cuda.synchronize()
                assert np.array_equal(got.cpu().numpy().astype(np.float64), oracle.dequant(c, s, N, K, b)), (e, mat)
        for T in (1, 4, 16, 64, 300):  # fused decode kernel, then the tensor-core path
            _check(torch, h, sh, L, synth.x_host(sh, 5000, T, T), f"b{bits}/{bits_down}")
        for T in (4, 37):
            _check(torch, h, sh, L, synth.x_host(sh, 5001, T, T), f"b{bits}/{bits_down} gemm", moe.MOE_FORCE_GEMM)
        for T in (64, 300):
            _check(torch, h, sh, L, synth.x_host(sh, 5002, T, T), f"b{bits}/{bits_down} gemv", moe.MOE_FORCE_GEMV)
    finally:
        h.close()


@pytest.mark.parametrize("T", [4, 16, 96])
def test_mixed_full_shape(torch_cuda, T):
    """The full-shape layer with 2-bit gate/up and 3-bit down: the fused decode kernel at 4 and 16
    tokens, the tensor-core path at 96.  Only the experts the tokens select (and the shared one) are
    written into the device buffer; the kernels read no other."""
    torch = torch_cuda
    base = WORKLOADS["decode"]
    sh = MoeShape(base.shape.d, base.shape.f, base.shape.E, base.shape.k, 1, 2, bits_down=3)
    master = base.master + 23
    xb = synth.x_host(sh, master, 1, T)
    wr, bias = synth.router_host(sh, master, 0, True)
    ids, _ = oracle.route(sh, xb, wr, bias)
    L = synth.layer_host(sh, master, 0, True, experts=set(ids.ravel().tolist()) | {sh.E})
    cb, sb = synth.expert_bytes(sh)
    n = sh.n_experts_total
    codes = torch.zeros(n * cb, dtype=torch.uint8, device="cuda")
    scales = torch.zeros(n * sb // 2, dtype=torch.int16, device="cuda")
    for e, (c, s) in enumerate(zip(L["codes"], L["scales"])):
        if c is not None:
            codes[e * cb:(e + 1) * cb] = torch.from_numpy(c).cuda()
            scales[e * sb // 2:(e + 1) * sb // 2] = torch.from_numpy(s.view(np.int16)).cuda()
    h = _handle(sh, 96)
    try:
        h.load_layer(0, codes, scales, torch.from_numpy(wr.view(np.int16)).cuda(), torch.from_numpy(bias).cuda())
        _check(torch, h, sh, L, xb, "full b2/3")
    finally:
        h.close()
