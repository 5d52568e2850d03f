"""Checks of the seeded input generator (host side)."""
import math

import numpy as np
import pytest

import synth
from synth import WORKLOADS, MoeShape


def test_f16_rounding_matches_ieee():
    rng = np.random.default_rng(1)
    vals = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * np.float32(0.05),
        (rng.standard_normal(5000) * 1e-6).astype(np.float32),  # fp16 subnormal range
        (rng.standard_normal(2000) * 3e4).astype(np.float32),
        np.array([0.0, -0.0, 65504.0, 65519.99, 65520.0, 1e9, 2 ** -24, 2 ** -25, 1.5 * 2 ** -25, 2 ** -14,
                  2 ** -14 - 2 ** -30, 6e-8, 3e-8], np.float32),
    ])
    L = synth.lib()
    got = np.array([L.synth_f32_to_f16(float(v)) for v in vals], np.uint16)
    want = vals.astype(np.float16).view(np.uint16)
    assert np.array_equal(got, want)


def test_bf16_rounding_ties_to_even():
    L = synth.lib()
    # 1 + 2^-8 is exactly half-way between bf16 1.0 and 1 + 2^-7: ties to even 1.0
    assert L.synth_f32_to_bf16(1.0 + 2 ** -8) == 0x3F80
    # 1 + 3*2^-8 is half-way between 1+2^-7 (odd) and 1+2^-6 (even)
    assert L.synth_f32_to_bf16(1.0 + 3 * 2 ** -8) == 0x3F82
    assert L.synth_f32_to_bf16(1.0 + 2 ** -8 + 2 ** -20) == 0x3F81
    assert L.synth_f32_to_bf16(-2.0) == 0xC000


def test_normals_are_standard_normal():
    z = np.array([synth.lib().synth_normal(synth.key(7, 0, 0), i) for i in range(4000)])
    big = synth.normal_f32(synth.key(7, 1, 0), 2_000_000, 1.0).astype(np.float64)
    assert abs(big.mean()) < 4 / math.sqrt(big.size)
    assert abs(big.std() - 1) < 3e-3
    kurt = ((big - big.mean()) ** 4).mean() / big.var() ** 2
    assert abs(kurt - 3) < 0.03
    # Kolmogorov-Smirnov distance against the normal CDF
    from scipy.stats import kstest
    assert kstest(big[:200000], "norm").pvalue > 1e-3
    # scalar path equals the bulk path (same counter definition)
    bulk = synth.normal_f32(synth.key(7, 0, 0), 4000, 1.0)
    assert np.array_equal(bulk, z.astype(np.float32))


def test_keys_are_independent_and_deterministic():
    a = synth.normal_f32(synth.key(1, 0, 3, 0), 1000)
    b = synth.normal_f32(synth.key(1, 0, 3, 1), 1000)
    c = synth.normal_f32(synth.key(1, 0, 3, 0), 1000)
    assert np.array_equal(a, c)
    assert abs(np.corrcoef(a, b)[0, 1]) < 0.15


def _quant_ref(w, bits):
    """Reference block quantiser written from the format definition with numpy."""
    N, K = w.shape
    half = 2 ** (bits - 1)
    blocks = w.reshape(N, K // 32, 32)
    amax = np.abs(blocks).max(axis=2)
    s16 = (amax / np.float32(half)).astype(np.float16)
    sf = s16.astype(np.float32)[:, :, None]
    with np.errstate(divide="ignore", invalid="ignore"):
        t = np.where(sf != 0, blocks / np.where(sf != 0, sf, 1), 0).astype(np.float32)
    q = np.clip(np.rint(t), -half, half - 1).astype(np.int8)
    return q.reshape(N, K), s16.view(np.uint16)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_quantiser_matches_definition(bits):
    w = synth.normal_f32(synth.key(3, 0, 3, bits), 64 * 256, 0.02).reshape(64, 256)
    w[5, 32:64] = 0.0  # an all-zero block: scale 0, codes 0
    _, _, q, s = synth.quantize(w, bits)
    qr, sr = _quant_ref(w, bits)
    assert np.array_equal(s, sr)
    assert np.array_equal(q, qr)
    assert (q[5, 32:64] == 0).all() and (s[5, 1] == 0)
    # the clamp: a positive block maximum maps to 2^(b-1)-1
    assert q.max() == 2 ** (bits - 1) - 1 and q.min() == -(2 ** (bits - 1))


def test_zipf_bias_is_a_permuted_log_prior():
    E = 512
    b = synth.zipf_bias(synth.key(5, 0, 2), E, 1.1).astype(np.float64)
    assert abs(np.exp(b).sum() - 1) < 1e-5
    ranks = np.argsort(-b)
    p = np.exp(b[ranks])
    r = np.arange(1, E + 1, dtype=np.float64)
    want = r ** -1.1 / (r ** -1.1).sum()
    assert np.allclose(p, want, rtol=1e-5)
    b2 = synth.zipf_bias(synth.key(5, 1, 2), E, 1.1)
    assert not np.array_equal(np.argsort(b2), np.argsort(b))


def test_layer_builder_sizes():
    sh = WORKLOADS["tiny"].shape
    L = synth.layer_host(sh, 11, 0, zipf=False)
    cb, sb = synth.expert_bytes(sh)
    assert all(c.nbytes == cb for c in L["codes"]) and all(s.nbytes == sb for s in L["scales"])
    assert L["router_w"].shape == (sh.E, sh.d) and L["bias"] is None
    full = MoeShape(2048, 768, 512, 10, 1, 2)
    assert sum(synth.expert_bytes(full)) == 1_474_560
