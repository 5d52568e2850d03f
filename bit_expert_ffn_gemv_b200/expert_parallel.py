"""Expert parallelism over torch.distributed (one process per GPU).

Each rank holds a contiguous range of the routed experts (rank 0 also the
shared expert) and computes, for all tokens, the fp32 partial output of its
experts (``moe_set_expert_range``).  Every rank routes over all experts with
the replicated router, so the ranks agree on the selection and the weights.
An all-reduce of the partial outputs then gives the layer on every rank (NCCL
over NVLink on GPUs; gloo on CPU for the host-side tests).

The Strata pages split a model over two GPUs by layers (24 + 24 layers with
pipelining: kangdaejong.com video summary, "pick-ups" section); that split
needs nothing from this library beyond one handle per GPU holding its
layers.  Splitting one layer's experts is the finer-grained alternative: a
rank reads only its experts' weights, at the price of one all-reduce of
[T x d] fp32 per layer.
"""
from __future__ import annotations

from . import MOE_ACCUMULATE, MOE_OUT_FP32


def expert_shard(n_experts: int, rank: int, world: int):
    """(begin, end, with_shared) of `rank`: [0, n_experts) split into `world` contiguous ranges whose sizes
    differ by at most one; the shared expert goes to rank 0."""
    if world < 1 or not 0 <= rank < world or n_experts < 0:
        raise ValueError("bad rank / world / expert count")
    return rank * n_experts // world, (rank + 1) * n_experts // world, rank == 0


def shard_handle(h, rank: int, world: int) -> None:
    """Restrict a MoeLayer handle to this rank's experts."""
    h.set_expert_range(*expert_shard(h.cfg.n_experts, rank, world))


def reduce_partial(y, group=None, stream=None):
    """Sum the ranks' fp32 partial outputs in place: afterwards y holds the layer on every rank.

    With a CUDA stream, the all-reduce is ordered on that stream (the one the partial output was computed
    on); without one, on the current stream.
    """
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        if stream is None:
            dist.all_reduce(y, op=dist.ReduceOp.SUM, group=group)
        else:
            import torch
            with torch.cuda.stream(stream):
                dist.all_reduce(y, op=dist.ReduceOp.SUM, group=group)
    return y


def forward(h, layer: int, x, y=None, flags: int = 0, group=None, stream=None):
    """This rank's partial output of `layer` for x (fp32 [T x d]), then the all-reduce.

    flags may add path or approximation flags; MOE_ACCUMULATE is refused, since every rank would add
    the residual once.  Add the residual after the call instead.
    """
    if flags & MOE_ACCUMULATE:
        raise ValueError("expert-parallel forward sums partial outputs: add the residual after the call")
    y = h.forward(layer, x, y, flags=flags | MOE_OUT_FP32, stream=stream)
    return reduce_partial(y, group, stream)
