"""Pins of the fp64 oracle against facts fixed outside it.

- a hand-worked quantisation block (tests/golden/dequant_block.txt)
- every code x a set of fp16 scales against q*s computed here
- the packed positions against a numpy quantiser (random weights)
- closed forms: uniform routing, one-hot bias, -I expert weights
- brute force: a dense formulation with k-subset enumeration on tiny layers
- invariants: weights sum to 1, token permutation, k = E dense mixture,
  unselected experts do not matter, logit shift invariance
"""
import itertools
import os

import numpy as np
import pytest

import oracle
import synth
from synth import MoeShape

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "dequant_block.txt")


def _f16(bits_u16):
    return np.asarray(bits_u16, np.uint16).view(np.float16).astype(np.float64)


def _bf16(bits_u16):
    return (np.asarray(bits_u16, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _golden_cases():
    cases, cur = [], None
    for line in open(GOLDEN):
        line = line.split("#")[0].strip()
        if not line:
            continue
        tok = line.split()
        if tok[0] == "bits":
            cur = dict(bits=int(tok[1]), scale=int(tok[3], 16), q=[int(v) for v in tok[5:]], fill=[], bytes=[])
        elif tok[0] == "fill":
            cur["fill"].append((int(tok[1]), int(tok[2]), int(tok[3], 16)))
        elif tok[0] == "bytes":
            cur["bytes"].append((int(tok[1]), [int(v, 16) for v in tok[2:]]))
        elif tok[0] == "end":
            cases.append(cur)
    return cases


W_BLOCK = np.array([0.0625, -0.03125, 0.015625, 0.046875, -0.0625, 0.0234375], np.float32)


@pytest.mark.parametrize("case", _golden_cases(), ids=lambda c: f"b{c['bits']}")
def test_hand_worked_block(case):
    bits = case["bits"]
    want = np.zeros(256 * bits, np.uint8)
    for off, n, val in case["fill"]:
        want[off:off + n] = val
    for off, bs in case["bytes"]:
        want[off:off + len(bs)] = bs
    w = np.zeros((16, 128), np.float32)
    w[0, :6] = W_BLOCK
    # the generator's quantiser + packer produce exactly the hand-worked bytes
    codes, scales, q, s = synth.quantize(w, bits)
    assert s[0, 0] == case["scale"] and (s.ravel()[1:] == 0).all()
    assert list(q[0, :6]) == case["q"]
    assert np.array_equal(codes, want)
    assert scales[0] == case["scale"] and (scales[1:] == 0).all()
    # the oracle's decoder reads the hand-worked bytes back as q * s
    sc = np.zeros(64, np.uint16)
    sc[0] = case["scale"]
    deq = oracle.dequant(want, sc, 16, 128, bits)
    expect = np.zeros((16, 128))
    expect[0, :6] = np.array(case["q"], np.float64) * _f16([case["scale"]])[0]
    assert np.array_equal(deq, expect)


SCALES = [0x3C00, 0x2800, 0x0001, 0x03FF, 0x0400, 0x7BFF, 0x0000, 0x8000 | 0x3555, 0x1234]


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_exhaustive_codes_times_scales(bits):
    half = 2 ** (bits - 1)
    for code in range(-half, half):
        for sb in SCALES:
            q = np.full((16, 128), code, np.int8)
            s = np.full((16, 4), sb, np.uint16)
            codes, scales = synth.pack(q, s, bits)
            deq = oracle.dequant(codes, scales, 16, 128, bits)
            assert np.array_equal(deq, np.full((16, 128), code * _f16([sb])[0])), (code, hex(sb))


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_positions_random_matrix(bits):
    rng = np.random.default_rng(bits)
    N, K = 48, 384
    half = 2 ** (bits - 1)
    q = rng.integers(-half, half, size=(N, K)).astype(np.int8)
    s = (rng.standard_normal((N, K // 32)) * 0.01).astype(np.float16).view(np.uint16)
    codes, scales = synth.pack(q, s, bits)
    deq = oracle.dequant(codes, scales, N, K, bits)
    expect = q.astype(np.float64) * np.repeat(_f16(s), 32, axis=1)
    assert np.array_equal(deq, expect)
    # the single-element decoder agrees at a few spots
    L = oracle.lib()
    for n, k in [(0, 0), (17, 129), (N - 1, K - 1), (8, 40)]:
        assert L.oracle_code(codes.ctypes.data, N, K, bits, n, k) == q[n, k]


# ---------------------------------------------------------------- layers
def _layer_from_q(shape, qs, ss, wr, bias):
    """Pack per-expert (q, s) triples [gate, up, down] into oracle inputs."""
    codes, scales = [], []
    for e in range(shape.E + shape.n_shared):
        cs, ssc = [], []
        for m in range(3):
            c, sc = synth.pack(qs[e][m], ss[e][m], synth.mat_bits(shape, m))
            cs.append(c)
            ssc.append(sc)
        codes.append(np.concatenate(cs))
        scales.append(np.concatenate(ssc))
    return codes, scales


def _random_layer(shape, seed, wr_scale=0.02, bias_scale=0.0):
    rng = np.random.default_rng(seed)
    qs, ss, deq = [], [], []
    for e in range(shape.E + shape.n_shared):
        qe, se, de = [], [], []
        for m in range(3):
            N, K = synth.mat_dims(shape, m)
            w = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
            _, _, q, s = synth.quantize(w, synth.mat_bits(shape, m))
            qe.append(q)
            se.append(s)
            de.append(q.astype(np.float64) * np.repeat(_f16(s), 32, axis=1))
        qs.append(qe)
        ss.append(se)
        deq.append(de)
    wr = (rng.standard_normal((shape.E, shape.d)) * wr_scale).astype(np.float32)
    wr_b = np.array([synth.lib().synth_f32_to_bf16(float(v)) for v in wr.ravel()], np.uint16).reshape(wr.shape)
    bias = (rng.standard_normal(shape.E) * bias_scale).astype(np.float32) if bias_scale else None
    codes, scales = _layer_from_q(shape, qs, ss, wr_b, bias)
    return dict(codes=codes, scales=scales, router_w=wr_b, bias=bias, deq=deq)


def _x(shape, T, seed):
    return synth.normal_bf16(synth.key(seed, 0, 0), T * shape.d, 1.0).reshape(T, shape.d)


def _dense(shape, L, x):
    """Dense formulation: every expert evaluated, top-k by k-subset enumeration."""
    X = _bf16(x)
    W = _bf16(L["router_w"])
    logits = X @ W.T + (0 if L["bias"] is None else L["bias"].astype(np.float64))
    outs = []
    for e in range(shape.E + shape.n_shared):
        g = X @ L["deq"][e][0].T
        u = X @ L["deq"][e][1].T
        h = g / (1 + np.exp(-g)) * u
        outs.append(h @ L["deq"][e][2].T)
    T = X.shape[0]
    y = np.zeros((T, shape.d))
    ids = np.zeros((T, shape.k), np.int64)
    for t in range(T):
        best, best_sum = None, None
        for S in itertools.combinations(range(shape.E), shape.k):
            sc = sum(logits[t, e] for e in S)
            if best is None or sc > best_sum:  # first max in lexicographic order
                best, best_sum = S, sc
        order = sorted(best, key=lambda e: (-logits[t, e], e))
        ids[t] = order
        lg = logits[t, order]
        w = np.exp(lg - lg.max())
        w /= w.sum()
        y[t] = (outs[shape.E][t] if shape.n_shared else 0) + sum(w[r] * outs[order[r]][t] for r in range(shape.k))
    return y, ids


@pytest.mark.parametrize("E,k,bits,shared,d,f", [(4, 2, 2, 1, 128, 128), (6, 3, 3, 1, 256, 128),
                                                 (5, 1, 4, 0, 128, 256), (6, 2, 2, 1, 128, 256)])
def test_brute_force_dense(E, k, bits, shared, d, f):
    shape = MoeShape(d=d, f=f, E=E, k=k, n_shared=shared, bits=bits)
    L = _random_layer(shape, seed=E * 10 + k, bias_scale=0.3)
    x = _x(shape, 5, seed=E + k)
    y, ids, w = oracle.layer(shape, x, L["router_w"], L["bias"], L["codes"], L["scales"])
    yd, idsd = _dense(shape, L, x)
    assert np.array_equal(ids, idsd)
    assert np.allclose(w.sum(1), 1, atol=1e-15, rtol=0)
    assert np.allclose(y, yd, rtol=1e-11, atol=1e-14)


def test_closed_form_uniform_routing():
    shape = MoeShape(d=128, f=128, E=16, k=4, n_shared=1, bits=2)
    wr = np.zeros((16, 128), np.uint16)
    x = _x(shape, 6, 3)
    ids, w = oracle.route(shape, x, wr, None)
    assert (ids == np.arange(4)).all()
    assert (w == 0.25).all()


@pytest.mark.parametrize("j", [0, 5, 15])
def test_closed_form_one_hot_bias(j):
    shape = MoeShape(d=128, f=128, E=16, k=2, n_shared=1, bits=2)
    wr = np.zeros((16, 128), np.uint16)
    Lb = 30.0
    bias = np.zeros(16, np.float32)
    bias[j] = Lb
    ids, w = oracle.route(shape, _x(shape, 3, 4), wr, bias)
    other = 0 if j != 0 else 1
    assert (ids[:, 0] == j).all() and (ids[:, 1] == other).all()
    assert np.allclose(w[:, 0], 1 / (1 + np.exp(-Lb)), rtol=1e-15)
    assert np.allclose(w[:, 1], np.exp(-Lb) / (1 + np.exp(-Lb)), rtol=1e-12)


@pytest.mark.parametrize("bits,d,f", [(2, 256, 128), (3, 128, 256), (4, 256, 256)])
def test_closed_form_minus_identity(bits, d, f):
    """W_g = W_u = W_d = -I: o_i = -x_i^2 sigmoid(-x_i) (i < min(f,d)), y = 2 o."""
    shape = MoeShape(d=d, f=f, E=8, k=3, n_shared=1, bits=bits)
    half = 2 ** (bits - 1)
    sbit = int(np.float16(1.0 / half).view(np.uint16))  # code -half times 1/half = -1 exactly
    qs, ss = [], []
    for _ in range(shape.E + 1):
        qe, se = [], []
        for m in range(3):
            N, K = synth.mat_dims(shape, m)
            q = np.zeros((N, K), np.int8)
            s = np.zeros((N, K // 32), np.uint16)
            for i in range(min(N, K)):
                q[i, i] = -half
                s[i, i // 32] = sbit
            qe.append(q)
            se.append(s)
        qs.append(qe)
        ss.append(se)
    rng = np.random.default_rng(9)
    wr = np.array([synth.lib().synth_f32_to_bf16(float(v)) for v in rng.standard_normal(8 * d) * 0.02],
                  np.uint16).reshape(8, d)
    codes, scales = _layer_from_q(shape, qs, ss, wr, None)
    x = _x(shape, 4, 21)
    y, ids, w = oracle.layer(shape, x, wr, None, codes, scales)
    X = _bf16(x)
    m = min(d, f)
    o = np.zeros_like(X)
    o[:, :m] = -X[:, :m] ** 2 / (1 + np.exp(X[:, :m]))
    assert np.allclose(y, 2 * o, rtol=1e-13, atol=1e-300)


@pytest.fixture(scope="module")
def tiny():
    shape = MoeShape(d=128, f=128, E=8, k=3, n_shared=1, bits=2)
    L = _random_layer(shape, seed=77, bias_scale=0.5)
    return shape, L


def test_weights_sum_to_one_and_permutation(tiny):
    shape, L = tiny
    x = _x(shape, 7, 5)
    y, ids, w = oracle.layer(shape, x, L["router_w"], L["bias"], L["codes"], L["scales"])
    assert np.abs(w.sum(1) - 1).max() <= 1e-15
    perm = np.array([3, 0, 6, 1, 5, 2, 4])
    yp, idsp, wp = oracle.layer(shape, x[perm], L["router_w"], L["bias"], L["codes"], L["scales"])
    assert np.array_equal(yp, y[perm]) and np.array_equal(idsp, ids[perm]) and np.array_equal(wp, w[perm])


def test_k_equals_E_is_dense_softmax_mixture(tiny):
    shape, L = tiny
    full = MoeShape(d=shape.d, f=shape.f, E=shape.E, k=shape.E, n_shared=1, bits=shape.bits)
    x = _x(shape, 4, 6)
    y, ids, w = oracle.layer(full, x, L["router_w"], L["bias"], L["codes"], L["scales"])
    X = _bf16(x)
    logits = X @ _bf16(L["router_w"]).T + L["bias"].astype(np.float64)
    p = np.exp(logits - logits.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)
    yd = np.zeros_like(X)
    for e in range(shape.E + 1):
        g = X @ L["deq"][e][0].T
        u = X @ L["deq"][e][1].T
        o = (g / (1 + np.exp(-g)) * u) @ L["deq"][e][2].T
        yd += o if e == shape.E else p[:, e:e + 1] * o
    assert np.allclose(y, yd, rtol=1e-11, atol=1e-15)


def test_unselected_experts_do_not_matter(tiny):
    shape, L = tiny
    x = _x(shape, 5, 8)
    y, ids, _ = oracle.layer(shape, x, L["router_w"], L["bias"], L["codes"], L["scales"])
    unused = sorted(set(range(shape.E)) - set(ids.ravel().tolist()))
    assert unused, "test needs at least one unselected expert"
    codes = list(L["codes"])
    for e in unused:
        codes[e] = np.random.default_rng(e).integers(0, 256, codes[e].size).astype(np.uint8)
    y2, _, _ = oracle.layer(shape, x, L["router_w"], L["bias"], codes, L["scales"])
    assert np.array_equal(y, y2)
    # and they may be absent altogether
    for e in unused:
        codes[e] = None
    y3, _, _ = oracle.layer(shape, x, L["router_w"], L["bias"], codes, L["scales"])
    assert np.array_equal(y, y3)


def test_logit_shift_invariance(tiny):
    shape, L = tiny
    x = _x(shape, 6, 9)
    b0 = (np.round(L["bias"].astype(np.float64) * 1024) / 1024).astype(np.float32)  # coarse grid: shifts are exact
    b2 = (b0.astype(np.float64) + 3.0).astype(np.float32)
    assert np.array_equal(b2.astype(np.float64) - 3.0, b0.astype(np.float64))
    y, ids, w = oracle.layer(shape, x, L["router_w"], b0, L["codes"], L["scales"])
    y2, ids2, w2 = oracle.layer(shape, x, L["router_w"], b2, L["codes"], L["scales"])
    assert np.array_equal(ids, ids2)
    assert np.allclose(w, w2, rtol=1e-13)
    assert np.allclose(y, y2, rtol=1e-12, atol=1e-15)


def test_route_matches_layer_routing(tiny):
    shape, L = tiny
    x = _x(shape, 9, 10)
    ids, w, lg = oracle.route(shape, x, L["router_w"], L["bias"], with_logits=True)
    _, ids2, w2 = oracle.layer(shape, x, L["router_w"], L["bias"], L["codes"], L["scales"])
    assert np.array_equal(ids, ids2) and np.array_equal(w, w2)
    X = _bf16(x)
    assert np.allclose(lg, X @ _bf16(L["router_w"]).T + L["bias"], rtol=1e-13, atol=1e-13)


def test_bad_arguments():
    shape = MoeShape(d=100, f=128, E=8, k=2, n_shared=1, bits=2)
    with pytest.raises(ValueError):
        oracle.route(shape, np.zeros((1, 100), np.uint16), np.zeros((8, 100), np.uint16), None)
    shape = MoeShape(d=128, f=128, E=8, k=9, n_shared=1, bits=2)
    with pytest.raises(ValueError):
        oracle.route(shape, np.zeros((1, 128), np.uint16), np.zeros((8, 128), np.uint16), None)


# ------------------------------------------------------------------ route-tail skip
def test_tail_skip_hand_worked_batch():
    """Two tokens of a top-10 over 16 experts, worked by hand: best ranks 5:0 9:0 2:2 6:2 7:3 12:3 11:4
    3:5 10:5 4:6 13:6 0:7 8:7 1:8 14:8 15:9, so rank 6 drops {0, 1, 4, 8, 13, 14, 15} -- expert 0 is
    7th for one token and 10th for the other, expert 2 stays because token 0 ranks it 3rd."""
    ids = np.array([[5, 9, 2, 7, 11, 3, 4, 8, 1, 0],
                    [9, 5, 6, 12, 2, 10, 13, 0, 14, 15]], np.int32)
    drop = oracle.tail_skip(ids, 16, 6)
    assert sorted(np.flatnonzero(drop).tolist()) == [0, 1, 4, 8, 13, 14, 15]
    # each token alone: its own ranks 6..9
    assert sorted(np.flatnonzero(oracle.tail_skip(ids[:1], 16, 6)).tolist()) == sorted([4, 8, 1, 0])
    assert sorted(np.flatnonzero(oracle.tail_skip(ids[1:], 16, 6)).tolist()) == sorted([13, 0, 14, 15])


def test_tail_skip_limits(tiny):
    """rank >= k drops nothing (the layer is unchanged bit for bit); rank 0 drops every selected expert
    (only the shared expert is left)."""
    shape, L = tiny
    x = _x(shape, 8, 11)
    ids, _ = oracle.route(shape, x, L["router_w"], L["bias"])
    assert not oracle.tail_skip(ids, shape.E, shape.k).any()
    y, _, _ = oracle.layer(shape, x, L["router_w"], L["bias"], L["codes"], L["scales"])
    y0, _, _ = oracle.layer(shape, x, L["router_w"], L["bias"], L["codes"], L["scales"],
                            drop=oracle.tail_skip(ids, shape.E, shape.k))
    assert np.array_equal(y, y0)
    all_drop = oracle.tail_skip(ids, shape.E, 0)
    assert np.array_equal(np.flatnonzero(all_drop), np.unique(ids))
    ys, _, _ = oracle.layer(shape, x, L["router_w"], L["bias"], L["codes"], L["scales"], drop=all_drop)
    g = _bf16(x) @ L["deq"][shape.E][0].T
    u = _bf16(x) @ L["deq"][shape.E][1].T
    o = (g / (1 + np.exp(-g)) * u) @ L["deq"][shape.E][2].T
    assert np.allclose(ys, o, rtol=1e-12, atol=1e-15)


def test_tail_skip_equals_zeroed_experts():
    """Dropping an expert's terms equals giving that expert all-zero scales (its output is then exactly
    0, and routing depends on the router alone): a different mechanism for the same sum."""
    shape = MoeShape(d=128, f=128, E=24, k=8, n_shared=1, bits=3)
    L = _random_layer(shape, seed=91, bias_scale=0.8)
    x = _x(shape, 6, 12)
    ids, _ = oracle.route(shape, x, L["router_w"], L["bias"])
    drop = oracle.tail_skip(ids, shape.E, 6)
    assert drop.any() and (np.unique(ids).size > drop.sum()), "test needs some dropped and some kept experts"
    ys, ids_s, w_s = oracle.layer(shape, x, L["router_w"], L["bias"], L["codes"], L["scales"], drop=drop)
    scales = [np.zeros_like(s) if e < shape.E and drop[e] else s for e, s in enumerate(L["scales"])]
    yz, ids_z, w_z = oracle.layer(shape, x, L["router_w"], L["bias"], L["codes"], scales)
    assert np.array_equal(ids_s, ids) and np.array_equal(ids_z, ids) and np.array_equal(w_s, w_z)
    assert np.array_equal(ys, yz)
    # and the single-token batch drops exactly that token's ranks 6.. (nothing else can save them)
    for t in range(x.shape[0]):
        d1 = oracle.tail_skip(ids[t:t + 1], shape.E, 6)
        assert sorted(np.flatnonzero(d1).tolist()) == sorted(ids[t, 6:].tolist())


# ------------------------------------------------------------------ per-tensor mixed precision
@pytest.mark.parametrize("bits,bits_down", [(2, 3), (2, 4), (3, 2), (4, 2)])
def test_mixed_widths_match_dense_formulation(bits, bits_down):
    """Gate/up at one code width and down at another: the oracle equals the dense formulation built from
    numpy-quantised matrices of those widths (k-subset enumeration for the selection)."""
    shape = MoeShape(d=128, f=128, E=6, k=2, n_shared=1, bits=bits, bits_down=bits_down)
    L = _random_layer(shape, seed=400 + 10 * bits + bits_down, bias_scale=0.3)
    x = _x(shape, 5, 41)
    y, ids, w = oracle.layer(shape, x, L["router_w"], L["bias"], L["codes"], L["scales"])
    yd, idsd = _dense(shape, L, x)[:2]
    assert np.array_equal(ids, idsd)
    assert np.allclose(y, yd, rtol=1e-11, atol=1e-14)
    # each expert's block really holds three matrices of those widths
    assert L["codes"][0].size == 128 * 128 * (2 * bits + bits_down) // 8


def test_mixed_widths_differ_from_uniform_reading():
    """Reading a mixed layer as uniform width gives a different output: the down width is used."""
    mixed = MoeShape(d=128, f=128, E=6, k=2, n_shared=1, bits=2, bits_down=4)
    L = _random_layer(mixed, seed=77)
    x = _x(mixed, 3, 5)
    y, _, _ = oracle.layer(mixed, x, L["router_w"], L["bias"], L["codes"], L["scales"])
    same = MoeShape(d=128, f=128, E=6, k=2, n_shared=1, bits=2, bits_down=2)
    short = [c[:128 * 128 * 6 // 8] for c in L["codes"]]
    y2, _, _ = oracle.layer(same, x, L["router_w"], L["bias"], short, L["scales"])
    assert not np.allclose(y, y2)


def test_tail_skip_depends_on_the_batch():
    """An expert that one token ranks 7th or lower is dropped when that token is alone, and kept when a
    token that ranks it among its first six shares the batch; the first token's output then gains that
    expert's term."""
    shape = MoeShape(d=128, f=128, E=24, k=8, n_shared=1, bits=2)
    L = _random_layer(shape, seed=515, bias_scale=0.3)
    xs = _x(shape, 40, 77)
    ids, _ = oracle.route(shape, xs, L["router_w"], L["bias"])
    found = None
    for a in range(40):
        for r in range(6, shape.k):
            e = int(ids[a, r])
            b = next((b for b in range(40) if e in ids[b, :6].tolist()), None)
            if b is not None:
                found = (a, b, e)
                break
        if found:
            break
    assert found is not None, "test needs such a pair of tokens"
    a, b, e = found
    alone = oracle.tail_skip(ids[[a]], shape.E, 6)
    both = oracle.tail_skip(ids[[a, b]], shape.E, 6)
    assert alone[e] == 1 and both[e] == 0
    ya, _, _ = oracle.layer(shape, xs[[a]], L["router_w"], L["bias"], L["codes"], L["scales"], drop=alone)
    yab, _, _ = oracle.layer(shape, xs[[a, b]], L["router_w"], L["bias"], L["codes"], L["scales"], drop=both)
    assert not np.allclose(ya[0], yab[0])
