"""moe_route_noalloc: routing for callers that cannot allocate device memory.

Callers inside a CUDA-graph capture, inside a framework that owns all device
memory, or in loops that cannot afford cudaMalloc's synchronisation use this
entry point; it keeps its intermediates in a fixed array inside the library.
These tests call it through the C ABI and compare each result with the
handle-based moe_route on the same inputs, token by token on its CUDA-core
router (at most 64 tokens per handle call): two calls in a row, the scratch's
exact capacity (T * E = 65536), the widest expert count (E = 1024, whose top-k
takes 128 KB of shared memory at 64 tokens), and a call captured in a CUDA graph and
replayed on new activations.  The file sorts last so
that a run stopping at the first failure has already run everything else.
"""
import numpy as np
import pytest

import synth
from synth import WORKLOADS
from synth.layer import MoeShape

pytestmark = pytest.mark.gpu


def _noalloc(moe, torch, x, sh, wr, bias):
    T = x.shape[0]
    ids = torch.full((T, sh.k), -1, dtype=torch.int32, device="cuda")
    w = torch.full((T, sh.k), -1.0, dtype=torch.float32, device="cuda")
    moe.moe_route_noalloc(x.data_ptr(), T, sh.d, sh.E, sh.k, wr.data_ptr(),
                          bias.data_ptr() if bias is not None else None, ids.data_ptr(), w.data_ptr(),
                          torch.cuda.current_stream().cuda_stream)
    return ids, w


@pytest.mark.parametrize("name,T", [("tiny", 8), ("decode", 64)])
def test_noalloc_route_matches_handle_route(name, T):
    import torch

    import bit_expert_ffn_gemv_b200 as moe
    from bit_expert_ffn_gemv_b200 import build
    from synth import gpu
    build.build()
    wl = WORKLOADS[name]
    sh = wl.shape
    codes, scales, wr, bias = gpu.layer_device(sh, wl.master, 0, wl.zipf)
    h = moe.MoeLayer(sh.d, sh.f, sh.E, sh.k, sh.n_shared, 1, sh.bits, T)
    h.load_layer(0, codes, scales, wr, bias)
    try:
        for call in range(2):  # two calls in a row share the fixed scratch
            x = gpu.x_device(sh, wl.master, 300 + call, T)
            ids_ref, w_ref = h.route(0, x)
            ids, w = _noalloc(moe, torch, x, sh, wr, bias)
            torch.cuda.synchronize()
            assert torch.equal(ids, ids_ref), f"call {call}: expert selection differs"
            assert torch.allclose(w, w_ref, rtol=2e-6, atol=1e-7), f"call {call}: weights differ"
            assert np.allclose(w.sum(1).cpu().numpy(), 1.0, atol=1e-5)
    finally:
        h.close()


def _handle_route(h, x, chunk=64):
    """moe_route on the CUDA-core router: chunks of at most 64 tokens."""
    import torch
    parts = [h.route(0, x[t0:t0 + chunk]) for t0 in range(0, x.shape[0], chunk)]
    return torch.cat([p[0] for p in parts]), torch.cat([p[1] for p in parts])


def _layer(sh, master, zipf, max_tokens):
    import bit_expert_ffn_gemv_b200 as moe
    from synth import gpu
    codes, scales, wr, bias = gpu.layer_device(sh, master, 0, zipf)
    h = moe.MoeLayer(sh.d, sh.f, sh.E, sh.k, sh.n_shared, 1, sh.bits, max_tokens)
    h.load_layer(0, codes, scales, wr, bias)
    return h, (codes, scales, wr, bias)


@pytest.mark.parametrize("case", ["capacity", "wide_e"])
def test_noalloc_route_at_its_limits(case):
    """T * E exactly 65536 (T = 128, E = 512), and E = 1024 at 64 tokens."""
    import torch

    import bit_expert_ffn_gemv_b200 as moe
    from bit_expert_ffn_gemv_b200 import build
    from synth import gpu
    build.build()
    if case == "capacity":
        wl = WORKLOADS["decode"]
        sh, master, zipf, T = wl.shape, wl.master, wl.zipf, 128
    else:
        sh, master, zipf, T = MoeShape(d=256, f=128, E=1024, k=10, n_shared=1, bits=2), 0x5EED_0A11, True, 64
    assert T * sh.E <= 65536
    h, keep = _layer(sh, master, zipf, T)
    try:
        x = gpu.x_device(sh, master, 310, T)
        ids_ref, w_ref = _handle_route(h, x)
        ids, w = _noalloc(moe, torch, x, sh, keep[2], keep[3])
        torch.cuda.synchronize()
        assert torch.equal(ids, ids_ref), "expert selection differs"
        assert torch.allclose(w, w_ref, rtol=2e-6, atol=1e-7), "weights differ"
    finally:
        h.close()


def test_noalloc_route_in_a_cuda_graph():
    """First call outside capture, then one call captured and replayed on new activations."""
    import torch

    import bit_expert_ffn_gemv_b200 as moe
    from bit_expert_ffn_gemv_b200 import build
    from synth import gpu
    build.build()
    wl = WORKLOADS["decode"]
    sh, T = wl.shape, 16
    h, keep = _layer(sh, wl.master, wl.zipf, T)
    wr, bias = keep[2], keep[3]
    try:
        x = gpu.x_device(sh, wl.master, 320, T)
        _noalloc(moe, torch, x, sh, wr, bias)  # first call: module loaded, address known
        torch.cuda.synchronize()
        ids = torch.full((T, sh.k), -1, dtype=torch.int32, device="cuda")
        w = torch.full((T, sh.k), -1.0, dtype=torch.float32, device="cuda")
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            moe.moe_route_noalloc(x.data_ptr(), T, sh.d, sh.E, sh.k, wr.data_ptr(),
                                  bias.data_ptr() if bias is not None else None, ids.data_ptr(), w.data_ptr(),
                                  torch.cuda.current_stream().cuda_stream)
        for call in range(2):
            x.copy_(gpu.x_device(sh, wl.master, 321 + call, T))
            g.replay()
            torch.cuda.synchronize()
            ids_ref, w_ref = h.route(0, x)
            torch.cuda.synchronize()
            assert torch.equal(ids, ids_ref), f"replay {call}: expert selection differs"
            assert torch.allclose(w, w_ref, rtol=2e-6, atol=1e-7), f"replay {call}: weights differ"
        del g
    finally:
        h.close()


def test_noalloc_route_rejects_oversize():
    import torch

    import bit_expert_ffn_gemv_b200 as moe
    sh = WORKLOADS["decode"].shape
    x = torch.zeros(129, sh.d, dtype=torch.bfloat16, device="cuda")  # 129 * 512 > 65536
    wr = torch.zeros(sh.E, sh.d, dtype=torch.bfloat16, device="cuda")
    ids = torch.empty(129, sh.k, dtype=torch.int32, device="cuda")
    w = torch.empty(129, sh.k, dtype=torch.float32, device="cuda")
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_route_noalloc(x.data_ptr(), 129, sh.d, sh.E, sh.k, wr.data_ptr(), None, ids.data_ptr(),
                              w.data_ptr(), 0)
    assert ei.value.status == 1
