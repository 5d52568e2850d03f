"""Host-side failure handling through the C ABI: every bad call is refused with its status before any
work is enqueued, and the handle stays usable.  Nothing here faults, traps or hangs a GPU: no kernel
is launched with a bad argument, and the one allocation failure asks for more memory than exists."""
import ctypes

import numpy as np
import pytest

import synth
from synth import WORKLOADS
from tests.gpu_util import make_layer_host, upload_layer, x_to_device

pytestmark = pytest.mark.gpu

INVALID, NOT_LOADED, OOM = 1, 4, 3


@pytest.fixture(scope="module")
def tiny():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import bit_expert_ffn_gemv_b200 as moe
    import bit_expert_ffn_gemv_b200.build as b
    b.build()
    wl = WORKLOADS["tiny"]
    L = make_layer_host(wl)
    h = moe.MoeLayer(wl.shape.d, wl.shape.f, wl.shape.E, wl.shape.k, wl.shape.n_shared, 2, wl.shape.bits, 8)
    h.load_layer(0, *upload_layer(L))  # layer 1 stays unloaded
    yield wl, h
    h.close()


def _fwd(h, layer, x_ptr, T, y_ptr, flags=0):
    import bit_expert_ffn_gemv_b200 as moe
    return moe.lib().moe_forward(h.handle, layer, x_ptr, T, y_ptr, flags, None)


def test_bad_forward_arguments_are_refused(tiny):
    import torch
    import bit_expert_ffn_gemv_b200 as moe
    wl, h = tiny
    x = x_to_device(synth.x_host(wl.shape, wl.master, 3, 4))
    y = torch.empty(8, wl.shape.d, dtype=torch.bfloat16, device="cuda")
    xp, yp = x.data_ptr(), y.data_ptr()
    assert _fwd(h, 2, xp, 4, yp) == INVALID           # layer out of range
    assert _fwd(h, -1, xp, 4, yp) == INVALID
    assert _fwd(h, 1, xp, 4, yp) == NOT_LOADED        # layer never loaded
    assert _fwd(h, 0, xp, 9, yp) == INVALID           # T > max_tokens
    assert _fwd(h, 0, xp, -1, yp) == INVALID
    assert _fwd(h, 0, None, 4, yp) == INVALID         # null pointers
    assert _fwd(h, 0, xp, 4, None) == INVALID
    assert _fwd(h, 0, xp + 2, 4, yp) == INVALID       # misaligned pointers
    assert _fwd(h, 0, xp, 4, yp + 8) == INVALID
    assert _fwd(h, 0, xp, 4, yp, 1 << 31) == INVALID  # unknown flag
    assert _fwd(h, 0, xp, 4, yp, moe.MOE_FORCE_GEMV | moe.MOE_FORCE_GEMM) == INVALID
    assert moe.lib().moe_forward(None, 0, xp, 4, yp, 0, None) == INVALID
    ids = torch.empty(4, wl.shape.k, dtype=torch.int32, device="cuda")
    w = torch.empty(4, wl.shape.k, dtype=torch.float32, device="cuda")
    assert moe.lib().moe_route(h.handle, 0, xp, 4, ids.data_ptr() + 4, w.data_ptr(), None) == INVALID
    assert moe.lib().moe_route(h.handle, 1, xp, 4, ids.data_ptr(), w.data_ptr(), None) == NOT_LOADED
    # nothing was enqueued and no device status was raised; the handle still computes
    assert h.check_status() == 0
    h.forward(0, x, y[:4])
    torch.cuda.synchronize()
    assert h.check_status() == 0 and torch.isfinite(y[:4].float()).all()


def test_bad_load_arguments_are_refused(tiny):
    import torch
    import bit_expert_ffn_gemv_b200 as moe
    wl, h = tiny
    codes, scales, wr, bias = upload_layer(make_layer_host(wl))
    W = moe.MoeLayerWeights
    ok = dict(codes=codes.data_ptr(), scales=scales.data_ptr(), router_w=wr.data_ptr(), router_bias=None)
    for bad in [dict(codes=None), dict(scales=None), dict(router_w=None), dict(codes=codes.data_ptr() + 8),
                dict(router_w=wr.data_ptr() + 2)]:
        args = dict(ok, **bad)
        assert moe.lib().moe_load_layer(h.handle, 1, ctypes.byref(W(**args))) == INVALID, bad
    assert moe.lib().moe_load_layer(h.handle, 5, ctypes.byref(W(**ok))) == INVALID
    torch.cuda.synchronize()


def test_impossible_handle_size_is_a_clean_oom():
    """max_tokens 2^20 at d = f = 16384 and E = 1024 asks for terabytes of scratch: MOE_ERR_OOM, no
    handle, and the device stays usable."""
    import torch
    import bit_expert_ffn_gemv_b200 as moe
    cfg = moe.MoeConfig(d=16384, f=16384, n_experts=1024, top_k=32, n_shared=1, n_layers=1, bits=2,
                        max_tokens=1 << 20)
    out = ctypes.c_void_p(1234)
    assert moe.lib().moe_layer_init(ctypes.byref(cfg), ctypes.byref(out)) == OOM
    assert out.value is None
    a = torch.ones(1024, device="cuda")
    assert float(a.sum()) == 1024.0


def test_destroy_is_safe_on_null():
    import bit_expert_ffn_gemv_b200 as moe
    assert moe.lib().moe_destroy(None) == 0
