"""The device watchdog: a bounded wait that runs out reports MOE_ERR_TIMEOUT and the handle recovers.

The fused decode kernel's CTAs hand the router logits to one another through a
grid-wide arrival counter, and every wait on it gives up after a bounded number
of polls.  A test hook (moe_debug_wait_limit) shortens that bound and makes one
CTA withhold its arrival, so every other CTA's wait runs out: nothing traps or
hangs, the kernel finishes, and the status word carries the timeout.
moe_check_status must then report MOE_ERR_TIMEOUT, reset the kernel's counters,
and leave the same handle computing correct layers again.
"""
import numpy as np
import pytest

import oracle
import synth
from synth import WORKLOADS
from tests.gpu_util import MAX_ABS, REL_L2, make_layer_host, max_abs, rel_l2, upload_layer, x_to_device, y_to_f64

pytestmark = pytest.mark.gpu

SHORT_WAIT = 1 << 14  # polls of at most 128 ns: a few milliseconds
DEFAULT_WAIT = 1 << 21


@pytest.fixture(scope="module")
def torch_cuda():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import bit_expert_ffn_gemv_b200.build as b
    b.build()
    return torch


def _timeout_then_recover(torch, h, x, withhold):
    import bit_expert_ffn_gemv_b200 as moe
    assert h.check_status() == 0
    h.debug_wait_limit(SHORT_WAIT, withhold)
    h.forward(0, x)
    torch.cuda.synchronize()
    assert moe.STATUS[h.check_status()] == "MOE_ERR_TIMEOUT"
    assert h.stats()["cuda_error"] == 0, "the timed-out launch must end without a CUDA error"
    h.debug_wait_limit(DEFAULT_WAIT, -1)


@pytest.mark.parametrize("T,withhold", [(4, 5), (1, 0), (16, 131)])
def test_withheld_arrival_times_out_then_tiny_layer_is_correct(torch_cuda, T, withhold):
    wl = WORKLOADS["tiny"]
    L = make_layer_host(wl)
    import bit_expert_ffn_gemv_b200 as moe
    h = moe.MoeLayer(wl.shape.d, wl.shape.f, wl.shape.E, wl.shape.k, wl.shape.n_shared, 1, wl.shape.bits, 16)
    try:
        h.load_layer(0, *upload_layer(L))
        x_bits = synth.x_host(wl.shape, wl.master, 700 + T, T)
        x = x_to_device(x_bits)
        _timeout_then_recover(torch_cuda, h, x, withhold)
        for rep in range(2):  # the counters were reset: later launches hand off normally
            y = h.forward(0, x)
            torch_cuda.cuda.synchronize()
            assert h.check_status() == 0, f"launch {rep} after the timeout"
            y_ref, _, _ = oracle.layer(wl.shape, x_bits, L["router_w"], L["bias"], L["codes"], L["scales"])
            g = y_to_f64(y)
            assert rel_l2(g, y_ref) <= REL_L2 and max_abs(g, y_ref) <= MAX_ABS
    finally:
        h.close()


def test_withheld_arrival_full_shape_recovers_bit_for_bit(torch_cuda):
    """Full-shape layer: the output after the timeout equals the output before it, bit for bit."""
    import bit_expert_ffn_gemv_b200 as moe
    from synth import gpu
    wl = WORKLOADS["decode"]
    sh = wl.shape
    h = moe.MoeLayer(sh.d, sh.f, sh.E, sh.k, sh.n_shared, 1, sh.bits, 16)
    try:
        h.load_layer(0, *gpu.layer_device(sh, wl.master, 0, wl.zipf))
        x = gpu.x_device(sh, wl.master, 710, 4)
        y_before = h.forward(0, x).clone()
        torch_cuda.cuda.synchronize()
        assert h.check_status() == 0
        _timeout_then_recover(torch_cuda, h, x, 73)
        y_after = h.forward(0, x)
        torch_cuda.cuda.synchronize()
        assert h.check_status() == 0
        assert torch_cuda.equal(y_before.view(torch_cuda.int16), y_after.view(torch_cuda.int16))
    finally:
        h.close()


def test_wait_limit_hook_rejects_bad_arguments(torch_cuda):
    import bit_expert_ffn_gemv_b200 as moe
    wl = WORKLOADS["tiny"]
    sh = wl.shape
    h = moe.MoeLayer(sh.d, sh.f, sh.E, sh.k, sh.n_shared, 1, sh.bits, 4)
    try:
        for spins, cta in [(0, -1), (100, -2)]:
            with pytest.raises(moe.MoeError):
                h.debug_wait_limit(spins, cta)
    finally:
        h.close()
