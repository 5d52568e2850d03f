"""The device generator writes exactly the host generator's bytes."""
import numpy as np
import pytest

import synth
from synth import WORKLOADS, MoeShape

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("bits,bits_down", [(2, 0), (3, 0), (4, 0), (2, 3), (2, 4), (3, 2), (4, 2)])
def test_experts_match_host(bits, bits_down):
    """Uniform and mixed code widths (gate/up at `bits`, down at `bits_down`)."""
    import torch
    from synth import gpu
    sh = MoeShape(d=256, f=128, E=16, k=2, n_shared=1, bits=bits, bits_down=bits_down)
    cb, sb = synth.expert_bytes(sh)
    codes = torch.empty(17 * cb, dtype=torch.uint8, device="cuda")
    scales = torch.empty(17 * sb // 2, dtype=torch.int16, device="cuda")
    gpu.experts_into(codes, scales, sh, 99, 3, 0, 17)
    c, s = codes.cpu().numpy(), scales.cpu().numpy().view(np.uint16)
    for e in range(17):
        hc, hs = synth.expert_host(sh, 99, 3, e)
        assert np.array_equal(c[e * cb:(e + 1) * cb], hc), e
        assert np.array_equal(s[e * sb // 2:(e + 1) * sb // 2], hs), e


def test_full_shape_experts_match_host():
    import torch
    from synth import gpu
    wl = WORKLOADS["decode"]
    sh = wl.shape
    cb, sb = synth.expert_bytes(sh)
    for e in (0, 311, sh.E):
        codes = torch.empty(cb, dtype=torch.uint8, device="cuda")
        scales = torch.empty(sb // 2, dtype=torch.int16, device="cuda")
        gpu.experts_into(codes, scales, sh, wl.master, 0, e, 1)
        hc, hs = synth.expert_host(sh, wl.master, 0, e)
        assert np.array_equal(codes.cpu().numpy(), hc), e
        assert np.array_equal(scales.cpu().numpy().view(np.uint16), hs), e


def test_normals_match_host():
    from synth import gpu
    k = synth.key(5, 1, 0)
    got = gpu.normal_bf16(k, 100001, 1.0).view(__import__("torch").int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got, synth.normal_bf16(k, 100001, 1.0))
