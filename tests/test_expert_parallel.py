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
