"""Expert parallelism on the device: a handle restricted to an expert range (moe_set_expert_range)
computes that range's partial output on every path.

The ranks of a W-way split run here one after another on the one GPU, each an
independent call (nothing waits on another rank): every partial output is
checked against the oracle's partial sum (the other experts' terms dropped,
the shared expert only on rank 0), and the sum of the partials against the
full layer.  The all-reduce itself is covered on CPU (test_expert_parallel.py).
"""
import numpy as np
import pytest

import oracle
import synth
from synth import WORKLOADS, MoeShape
from bit_expert_ffn_gemv_b200.expert_parallel import expert_shard
from tests.gpu_util import REL_L2_FP32, upload_layer, x_to_device, y_to_f64

pytestmark = pytest.mark.gpu

REL_L2_FP32_TC = 8e-4
SMALL = MoeShape(d=256, f=128, E=64, k=10, n_shared=1, bits=2)


@pytest.fixture(scope="module")
def torch_cuda():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import bit_expert_ffn_gemv_b200.build as b
    b.build()
    return torch


def _oracle_partial(shape, L, xb, begin, end, with_shared, drop_extra=None):
    drop = np.ones(shape.E, np.uint8)
    drop[begin:end] = 0
    if drop_extra is not None:
        drop |= drop_extra
    if with_shared:
        y, _, _ = oracle.layer(shape, xb, L["router_w"], L["bias"], L["codes"], L["scales"], drop=drop)
    else:
        sh0 = MoeShape(shape.d, shape.f, shape.E, shape.k, 0, shape.bits)
        y, _, _ = oracle.layer(sh0, xb, L["router_w"], L["bias"], L["codes"][:shape.E], L["scales"][:shape.E],
                               drop=drop)
    return y


def _run_split(torch, h, shape, L, xb, world, flags, tol, label, tail_skip=False):
    import bit_expert_ffn_gemv_b200 as moe
    x = x_to_device(xb)
    fl = flags | moe.MOE_OUT_FP32 | (moe.MOE_ROUTE_TAIL_SKIP if tail_skip else 0)
    extra = None
    if tail_skip:
        ids, _ = oracle.route(shape, xb, L["router_w"], L["bias"])
        extra = oracle.tail_skip(ids, shape.E, moe.MOE_TAIL_SKIP_RANK)
    full, _, _ = oracle.layer(shape, xb, L["router_w"], L["bias"], L["codes"], L["scales"], drop=extra)
    norm = np.linalg.norm(full)
    total = None
    try:
        for r in range(world):
            b, e, sh_on = expert_shard(shape.E, r, world)
            h.set_expert_range(b, e, sh_on)
            y = h.forward(0, x, flags=fl)
            torch.cuda.synchronize()
            assert h.check_status() == 0, (label, r)
            ref = _oracle_partial(shape, L, xb, b, e, sh_on, extra)
            err = np.linalg.norm(y_to_f64(y) - ref) / norm
            assert err <= tol, f"{label}: rank {r}/{world} partial off by {err:.3e} of the layer"
            total = y.clone() if total is None else total + y
    finally:
        h.set_expert_range(0, shape.E, True)
    err = np.linalg.norm(y_to_f64(total) - full) / norm
    print(f"{label} world={world} T={xb.shape[0]}: sum of partials vs layer rel_l2 {err:.3e}")
    assert err <= tol, label
    # the handle computes the whole layer again once the range is reset
    y = h.forward(0, x, flags=fl)
    torch.cuda.synchronize()
    assert np.linalg.norm(y_to_f64(y) - full) / norm <= tol, label


@pytest.fixture(scope="module")
def small(torch_cuda):
    import bit_expert_ffn_gemv_b200 as moe
    L = synth.layer_host(SMALL, 4243, 0, True)
    h = moe.MoeLayer(SMALL.d, SMALL.f, SMALL.E, SMALL.k, SMALL.n_shared, 1, SMALL.bits, 256)
    h.load_layer(0, *upload_layer(L))
    yield L, h
    h.close()


@pytest.mark.parametrize("T,path,world", [(1, "fused", 2), (4, "fused", 3), (16, "fused", 8), (4, "unfused", 2),
                                          (64, "gemv", 3), (200, "gemv", 2), (40, "gemm", 2), (200, "gemm", 3)])
def test_expert_split_small(torch_cuda, small, T, path, world):
    """E = 64, k = 10: with 3 or 8 ranks some tokens have no expert on a rank without the shared
    expert, whose partial output is then exactly 0."""
    import bit_expert_ffn_gemv_b200 as moe
    L, h = small
    flags = {"fused": 0, "unfused": moe.MOE_FORCE_UNFUSED, "gemv": moe.MOE_FORCE_GEMV,
             "gemm": moe.MOE_FORCE_GEMM}[path]
    xb = synth.x_host(SMALL, 4243, 10 + T, T)
    _run_split(torch_cuda, h, SMALL, L, xb, world, flags, REL_L2_FP32_TC if path == "gemm" else REL_L2_FP32,
               f"ep {path}")


def test_expert_split_with_tail_skip(torch_cuda, small):
    """The expert range and the route-tail skip drop experts together."""
    L, h = small
    xb = synth.x_host(SMALL, 4243, 99, 4)
    _run_split(torch_cuda, h, SMALL, L, xb, 2, 0, REL_L2_FP32, "ep fused + tail skip", tail_skip=True)


def test_expert_range_rejects_bad_arguments(torch_cuda, small):
    import bit_expert_ffn_gemv_b200 as moe
    _, h = small
    for args in [(-1, 4, 1), (5, 4, 1), (0, SMALL.E + 1, 1), (0, 4, 2)]:
        with pytest.raises(moe.MoeError):
            moe.moe_set_expert_range(h.handle, *args)
    h.set_expert_range(0, SMALL.E, True)


@pytest.mark.parametrize("T", [1, 4])
def test_expert_split_full_shape_decode(torch_cuda, T):
    """The full-shape layer split 8 ways (64 experts per rank) at decode batch sizes."""
    import bit_expert_ffn_gemv_b200 as moe
    from synth import gpu as sgpu
    wl = WORKLOADS["decode"]
    sh = wl.shape
    h = moe.MoeLayer(sh.d, sh.f, sh.E, sh.k, sh.n_shared, 1, sh.bits, 16)
    try:
        h.load_layer(0, *sgpu.layer_device(sh, wl.master, 0, wl.zipf))
        xb = synth.x_host(sh, wl.master, 3, T)
        wr, bias = synth.router_host(sh, wl.master, 0, wl.zipf)
        ids, _ = oracle.route(sh, xb, wr, bias)
        L = synth.layer_host(sh, wl.master, 0, wl.zipf, experts=set(ids.ravel().tolist()) | {sh.E})
        _run_split(torch_cuda, h, sh, L, xb, 8, 0, REL_L2_FP32, "ep full-shape")
    finally:
        h.close()


# ---------------------------------------------------------------- all-to-all dispatch and combine
def _segments(rows, counts):
    out, off = [], 0
    for n in counts:
        out.append(rows[off:off + n])
        off += n
    return out


@pytest.mark.parametrize("world,tokens", [(2, (3, 20)), (4, (1, 9, 40, 5))])
def test_all_to_all_virtual_ranks(torch_cuda, small, world, tokens):
    """Tokens data-parallel over `world` virtual ranks on the one GPU, experts split: each rank's tokens
    are dispatched to the ranks holding their experts, the library computes each rank's partial outputs on
    the rows it received (its expert range, no shared expert), and the partials return and are combined
    with the shared expert's output.  Run phase by phase in one process (the exchange is a list
    transposition; the gloo test covers torch.distributed's); every rank's layer output must match the
    oracle."""
    import bit_expert_ffn_gemv_b200 as moe
    from bit_expert_ffn_gemv_b200.expert_parallel import combine_rows, dispatch_plan, pack_rows
    torch = torch_cuda
    L, h = small
    sh = SMALL
    xbs = [synth.x_host(sh, 4243, 500 + r, tokens[r]) for r in range(world)]
    xs = [x_to_device(xb) for xb in xbs]
    try:
        plans, sends = [], []
        for r in range(world):
            ids, _ = h.route(0, xs[r])
            plan = dispatch_plan(ids, sh.E, world)
            plans.append(plan)
            sends.append(pack_rows(xs[r], plan))
        # exchange: rank R receives, source by source, the rows each rank packed for it
        recv = [torch.cat([_segments(*sends[r])[R] for r in range(world)]) for R in range(world)]
        recv_counts = [[sends[r][1][R] for r in range(world)] for R in range(world)]
        parts = []
        for R in range(world):
            b, e, _ = expert_shard(sh.E, R, world)
            h.set_expert_range(b, e, False)
            parts.append(h.forward(0, recv[R], flags=moe.MOE_OUT_FP32))
        back = [torch.cat([_segments(parts[R], recv_counts[R])[r] for R in range(world)]) for r in range(world)]
        h.set_expert_range(0, 0, True)
        for r in range(world):
            y = h.forward(0, xs[r], flags=moe.MOE_OUT_FP32)
            combine_rows(y, plans[r], back[r])
            torch.cuda.synchronize()
            assert h.check_status() == 0
            full, _, _ = oracle.layer(sh, xbs[r], L["router_w"], L["bias"], L["codes"], L["scales"])
            err = np.linalg.norm(y_to_f64(y) - full) / np.linalg.norm(full)
            print(f"a2a world={world} rank {r} T={tokens[r]}: rel_l2 {err:.3e}")
            assert err <= REL_L2_FP32_TC, (world, r, err)
    finally:
        h.set_expert_range(0, sh.E, True)


def test_all_to_all_layer_single_rank(torch_cuda, small):
    """a2a_layer without a process group (one rank) is the layer."""
    from bit_expert_ffn_gemv_b200.expert_parallel import a2a_layer
    L, h = small
    xb = synth.x_host(SMALL, 4243, 77, 33)
    y = a2a_layer(h, 0, x_to_device(xb))
    torch_cuda.cuda.synchronize()
    full, _, _ = oracle.layer(SMALL, xb, L["router_w"], L["bias"], L["codes"], L["scales"])
    assert np.linalg.norm(y_to_f64(y) - full) / np.linalg.norm(full) <= REL_L2_FP32_TC
