"""Expert parallelism, host side: the expert split and the all-reduce of partial outputs, as gloo ranks
on CPU whose partial outputs come from the oracle (the kernels' expert-range filter is checked on the
GPU in test_gpu_tail_skip.py)."""
import multiprocessing as mp
import os
import socket

import numpy as np
import pytest

from bit_expert_ffn_gemv_b200.expert_parallel import expert_shard


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("E,world", [(512, 2), (512, 8), (16, 3), (256, 5), (7, 7), (3, 4)])
def test_shards_partition_the_experts(E, world):
    shards = [expert_shard(E, r, world) for r in range(world)]
    cover = np.zeros(E, int)
    for b, e, _ in shards:
        assert 0 <= b <= e <= E
        cover[b:e] += 1
    assert (cover == 1).all()
    sizes = [e - b for b, e, _ in shards]
    assert max(sizes) - min(sizes) <= 1
    assert [s for _, _, s in shards] == [True] + [False] * (world - 1)
    with pytest.raises(ValueError):
        expert_shard(E, world, world)


def _rank(rank, world, port, out):
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        import synth
        from synth import MoeShape
        from bit_expert_ffn_gemv_b200.expert_parallel import expert_shard, reduce_partial
        sh = MoeShape(d=128, f=128, E=12, k=4, n_shared=1, bits=2)
        L = synth.layer_host(sh, 31337, 0, True)
        x = synth.x_host(sh, 31337, 1, 5)
        b, e, with_shared = expert_shard(sh.E, rank, world)
        drop = np.ones(sh.E, np.uint8)
        drop[b:e] = 0
        if with_shared:
            y, _, _ = oracle.layer(sh, x, L["router_w"], L["bias"], L["codes"], L["scales"], drop=drop)
        else:  # no shared expert on this rank
            sh0 = MoeShape(sh.d, sh.f, sh.E, sh.k, 0, sh.bits)
            y, _, _ = oracle.layer(sh0, x, L["router_w"], L["bias"], L["codes"][:sh.E], L["scales"][:sh.E],
                                   drop=drop)
        yt = torch.from_numpy(y.copy())
        reduce_partial(yt)
        full, _, _ = oracle.layer(sh, x, L["router_w"], L["bias"], L["codes"], L["scales"])
        out.put((rank, float(np.abs(yt.numpy() - full).max()), float(np.abs(full).max())))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_partial_outputs_sum_to_the_layer(world):
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, err, scale in res:
        assert err <= 1e-12 * max(scale, 1.0), (rank, err)


def test_single_process_reduce_is_identity():
    import torch
    from bit_expert_ffn_gemv_b200.expert_parallel import reduce_partial
    y = torch.arange(6.0).reshape(2, 3)
    assert torch.equal(reduce_partial(y.clone()), y)


def test_forward_refuses_accumulate():
    """Every rank would add the residual once: the expert-parallel forward refuses MOE_ACCUMULATE before
    touching the handle."""
    import bit_expert_ffn_gemv_b200 as moe
    from bit_expert_ffn_gemv_b200.expert_parallel import forward

    class NoHandle:
        def forward(self, *a, **k):
            raise AssertionError("must not be reached")

    with pytest.raises(ValueError):
        forward(NoHandle(), 0, None, flags=moe.MOE_ACCUMULATE)


# ---------------------------------------------------------------- all-to-all dispatch and combine
def test_expert_owner_matches_the_shards():
    import torch
    from bit_expert_ffn_gemv_b200.expert_parallel import expert_owner
    for E, world in [(512, 8), (16, 3), (3, 4), (7, 7), (10, 1)]:
        own = expert_owner(torch.arange(E), E, world)
        for e in range(E):
            b, en, _ = expert_shard(E, int(own[e]), world)
            assert b <= e < en, (E, world, e)


def test_dispatch_plan_and_combine_on_a_worked_case():
    """3 tokens, k = 2, E = 4 over 2 ranks (experts 0-1 on rank 0, 2-3 on rank 1)."""
    import torch
    from bit_expert_ffn_gemv_b200.expert_parallel import combine_rows, dispatch_plan, pack_rows
    ids = torch.tensor([[2, 0], [3, 2], [1, 0]])
    plan = dispatch_plan(ids, 4, 2)
    assert [p.tolist() for p in plan] == [[0, 2], [0, 1]]
    x = torch.arange(6.).view(3, 2)
    rows, counts = pack_rows(x, plan)
    assert counts == [2, 2] and rows.tolist() == [[0, 1], [4, 5], [0, 1], [2, 3]]
    y = torch.full((3, 2), 0.5, dtype=torch.float64)
    back = torch.tensor([[1., 1.], [2., 2.], [10., 10.], [20., 20.]])
    combine_rows(y, plan, back)
    assert y.tolist() == [[11.5, 11.5], [20.5, 20.5], [2.5, 2.5]]


def _a2a_rank(rank, world, port, out):
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        import synth
        from synth import MoeShape
        from bit_expert_ffn_gemv_b200.expert_parallel import a2a_forward, dist_exchange, expert_shard
        sh = MoeShape(d=128, f=128, E=12, k=4, n_shared=1, bits=2)
        L = synth.layer_host(sh, 4242, 0, True)
        sh0 = MoeShape(sh.d, sh.f, sh.E, sh.k, 0, sh.bits)
        b, e, _ = expert_shard(sh.E, rank, world)
        xb = synth.x_host(sh, 4242, 10 + rank, 3 + 2 * rank)  # every rank its own tokens, ragged counts
        x = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16)

        def bits(t):
            return t.view(torch.int16).numpy().view(np.uint16)

        def route(xx):
            return torch.from_numpy(oracle.route(sh, bits(xx), L["router_w"], L["bias"])[0].astype(np.int64))

        def partial(rows):  # this rank's routed experts only, no shared expert
            if rows.shape[0] == 0:
                return torch.zeros(0, sh.d, dtype=torch.float64)
            drop = np.ones(sh.E, np.uint8)
            drop[b:e] = 0
            y, _, _ = oracle.layer(sh0, bits(rows), L["router_w"], L["bias"], L["codes"][:sh.E], L["scales"][:sh.E],
                                   drop=drop)
            return torch.from_numpy(y.copy())

        def shared(xx):  # the shared expert alone
            y, _, _ = oracle.layer(sh, bits(xx), L["router_w"], L["bias"], L["codes"], L["scales"],
                                   drop=np.ones(sh.E, np.uint8))
            return torch.from_numpy(y.copy())

        y = a2a_forward(x, route, partial, shared, sh.E, world, dist_exchange())
        full, _, _ = oracle.layer(sh, xb, L["router_w"], L["bias"], L["codes"], L["scales"])
        out.put((rank, float(np.abs(y.numpy() - full).max()), float(np.abs(full).max())))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_all_to_all_layer_equals_the_layer(world):
    """Tokens data-parallel, experts split: dispatch, partial outputs (oracle), combine over gloo ranks."""
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_a2a_rank, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, err, scale in res:
        assert err <= 1e-12 * max(scale, 1.0), (rank, err)
