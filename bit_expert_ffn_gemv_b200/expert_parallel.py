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


# ---------------------------------------------------------------- all-to-all dispatch and combine
# For prefill, where every rank holds its own tokens (data parallel) and
# moving [T x d] activations is cheaper than replicating every expert:
#   1. each rank routes its tokens with the replicated router;
#   2. dispatch: token t goes, once, to every rank that holds one of its
#      selected experts (all_to_all of bf16 rows);
#   3. each rank computes its experts' fp32 partial outputs for the rows it
#      received (the library re-routes them to the same selection -- routing
#      is per token -- and keeps only its expert range);
#   4. combine: the partials return to the tokens' home ranks (all_to_all of
#      fp32 rows), which add them to the shared expert's output in a fixed
#      rank order.
# The route-tail skip depends on which tokens share a batch, so it is refused.

def expert_owner(ids, n_experts: int, world: int):
    """Rank that holds each expert id under expert_shard's contiguous split (same shape as ids)."""
    import torch
    starts = torch.tensor([r * n_experts // world for r in range(world)], dtype=torch.int64, device=ids.device)
    return torch.searchsorted(starts, ids.to(torch.int64).contiguous(), right=True) - 1


def dispatch_plan(ids, n_experts: int, world: int):
    """Per destination rank, the ascending indices of the tokens (rows of ids [T x k]) that select one of
    its experts."""
    import torch
    own = expert_owner(ids, n_experts, world)
    dest = torch.zeros(ids.shape[0], world, dtype=torch.bool, device=ids.device)
    if ids.numel():
        dest.scatter_(1, own, True)
    return [dest[:, r].nonzero().flatten() for r in range(world)]


def pack_rows(x, plan):
    """The rows of x to send, destination by destination, and their counts."""
    import torch
    counts = [int(i.numel()) for i in plan]
    rows = torch.cat([x.index_select(0, i) for i in plan]) if x.shape[0] else x[:0]
    return rows, counts


def combine_rows(y, plan, returned):
    """y += the partial rows that came back, source rank by source rank (a fixed order: deterministic)."""
    off = 0
    for idx in plan:
        n = int(idx.numel())
        if n:
            y.index_add_(0, idx, returned[off:off + n].to(y.dtype))
        off += n
    return y


def dist_exchange(group=None):
    """exchange(rows, send_counts) -> (received rows, receive counts) over torch.distributed
    all_to_all_single; 16-bit rows travel as bytes so every backend (gloo has no bf16) carries them bit
    for bit."""
    import torch
    import torch.distributed as dist

    def exchange(rows, counts):
        world = dist.get_world_size(group)
        sc = torch.tensor(counts, dtype=torch.int64, device=rows.device)
        rc = torch.empty(world, dtype=torch.int64, device=rows.device)
        dist.all_to_all_single(rc, sc, group=group)
        recv_counts = [int(v) for v in rc.tolist()]
        as_bytes = rows.element_size() == 2
        wire = rows.contiguous().view(torch.uint8) if as_bytes else rows.contiguous()
        out = wire.new_empty((sum(recv_counts),) + tuple(wire.shape[1:]))
        dist.all_to_all_single(out, wire, output_split_sizes=recv_counts, input_split_sizes=counts, group=group)
        return (out.view(rows.dtype) if as_bytes else out), recv_counts

    return exchange


def a2a_forward(x, route, partial, shared, n_experts: int, world: int, exchange):
    """One layer for this rank's tokens x [T x d] with the experts spread over `world` ranks.

    route(x) -> ids [T x k] (replicated router); partial(rows) -> this rank's experts' fp32 partial
    outputs for received rows; shared(x) -> the shared expert's output for x, or None; exchange as
    dist_exchange.  Returns y [T x d] (the dtype of shared's output, fp32 without one).
    """
    import torch
    ids = route(x)
    plan = dispatch_plan(ids, n_experts, world)
    rows, counts = pack_rows(x, plan)
    recv, recv_counts = exchange(rows, counts)
    part = partial(recv)
    back, _ = exchange(part, recv_counts)
    y = shared(x)
    if y is None:
        y = torch.zeros(x.shape[0], x.shape[1], dtype=torch.float32, device=x.device)
    return combine_rows(y, plan, back)


def a2a_layer(h, layer: int, x, group=None, flags: int = 0, stream=None):
    """a2a_forward through the library on a MoeLayer handle holding all experts' weights of `layer` (only
    this rank's experts are read): this rank's experts are those of expert_shard; the shared expert runs
    on every rank for its own tokens.  The handle's max_tokens must cover the rows a rank can receive
    (at most the sum of all ranks' T).  The handle's expert range is left at the full layer."""
    import torch.distributed as dist

    from . import MOE_ROUTE_TAIL_SKIP
    if flags & (MOE_ACCUMULATE | MOE_ROUTE_TAIL_SKIP):
        raise ValueError("all-to-all forward: add the residual after the call; the route-tail skip depends on "
                         "the batch and is refused")
    world = dist.get_world_size(group) if dist.is_available() and dist.is_initialized() else 1
    rank = dist.get_rank(group) if world > 1 else 0
    E = h.cfg.n_experts
    b, e, _ = expert_shard(E, rank, world)

    def partial(rows):
        h.set_expert_range(b, e, False)
        return h.forward(layer, rows, flags=flags | MOE_OUT_FP32, stream=stream)

    def shared(xx):
        if h.cfg.n_shared == 0:
            return None
        h.set_expert_range(0, 0, True)
        return h.forward(layer, xx, flags=flags | MOE_OUT_FP32, stream=stream)

    exchange = dist_exchange(group) if world > 1 else (lambda rows, counts: (rows, counts))
    try:
        return a2a_forward(x, lambda xx: h.route(layer, xx, stream=stream)[0], partial, shared, E, world, exchange)
    finally:
        h.set_expert_range(0, E, True)
