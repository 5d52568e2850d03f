"""moe_route_noalloc: routing for callers that cannot allocate device memory.

Callers inside a CUDA-graph capture, inside a framework that owns all device
memory, or in loops that cannot afford cudaMalloc's synchronisation use this
entry point; it keeps its intermediates in a fixed array inside the library.
These tests call it through the C ABI twice in a row and compare each result
with the handle-based moe_route on the same inputs.  The file sorts last so
that a run stopping at the first failure has already run everything else.
"""
import numpy as np
import pytest

import synth
from synth import WORKLOADS

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
