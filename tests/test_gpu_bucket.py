"""The grouping step alone (moe_debug_bucket) against a host counting sort.

The pages route each token to its top-k experts and run every selected expert
on the tokens that chose it (discuss.pytorch.kr post, "how it works"); the
unfused and tensor-core paths first group the T*k (token, rank) pairs by
expert.  The grouping must be a stable counting sort: per-expert counts and
offsets, pairs in ascending expert order and ascending token order inside a
group, the inverse permutation, and the list of non-empty experts.  A scatter
that loses stability would still give correct layer outputs (the combine sums
the same terms), so only a direct check like this one sees it.  Both variants
are covered: one CTA below 8192 pairs, three kernels over 128 CTAs from 8192
pairs on; with and without the route-tail skip and an expert range.
"""
import numpy as np
import pytest

SKIP_RANK = 6  # MOE_TAIL_SKIP_RANK in include/moe.h


def host_grouping(ids: np.ndarray, E: int, skip_rank: int = 0, e_begin: int = 0, e_end: int = 1 << 30):
    """Stable counting sort of the pairs p = t*k + r by expert ids[t, r], after dropping pairs whose
    expert is outside [e_begin, e_end) or (skip_rank > 0) never ranked below skip_rank."""
    T, k = ids.shape
    flat = ids.reshape(-1).astype(np.int64)
    keep = (flat >= e_begin) & (flat < e_end)
    if skip_rank > 0:
        best = np.full(E, k)
        ranks = np.tile(np.arange(k), T)
        np.minimum.at(best, flat, ranks)
        keep &= best[flat] < skip_rank
    p_kept = np.nonzero(keep)[0]
    order = p_kept[np.argsort(flat[p_kept], kind="stable")]
    counts = np.bincount(flat[p_kept], minlength=E)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    inv = np.full(T * k, -1, np.int32)
    inv[order] = np.arange(order.size, dtype=np.int32)
    active = np.nonzero(counts)[0].astype(np.int32)
    return offsets, order.astype(np.int32), inv, active


def draw_ids(rng, T: int, E: int, k: int, skew: float = 1.1) -> np.ndarray:
    """k distinct experts per token, drawn from a Zipf-like prior (a few experts in most tokens)."""
    p = 1.0 / np.arange(1, E + 1) ** skew
    p = p[rng.permutation(E)]
    p /= p.sum()
    return np.stack([rng.choice(E, k, replace=False, p=p) for _ in range(T)]).astype(np.int32)


def test_host_grouping_on_a_worked_case():
    """Hand-checked: 3 tokens, k = 2, E = 4."""
    ids = np.array([[2, 0], [0, 3], [2, 1]], np.int32)
    off, pairs, inv, act = host_grouping(ids, 4)
    assert off.tolist() == [0, 2, 3, 5, 6]
    assert pairs.tolist() == [1, 2, 5, 0, 4, 3]  # expert 0: t0r1, t1r0; 1: t2r1; 2: t0r0, t2r0; 3: t1r1
    assert inv.tolist() == [3, 0, 1, 5, 4, 2]
    assert act.tolist() == [0, 1, 2, 3]
    # the skip rank 1 keeps only experts that some token ranked first (2 and 0)
    off, pairs, inv, act = host_grouping(ids, 4, skip_rank=1)
    assert off.tolist() == [0, 2, 2, 4, 4] and pairs.tolist() == [1, 2, 0, 4] and act.tolist() == [0, 2]
    assert inv.tolist() == [2, 0, 1, -1, 3, -1]


@pytest.fixture(scope="module")
def torch_cuda():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import bit_expert_ffn_gemv_b200.build as b
    b.build()
    return torch


CASES = [
    # (E, k, T): one CTA below 8192 pairs, three kernels from 8192 on
    (16, 2, 37),
    (512, 10, 64),
    (512, 10, 819),   # 8190 pairs: the one-CTA kernel's largest case here
    (512, 10, 820),   # 8200 pairs: the three-kernel variant
    (512, 10, 8192),
    (1024, 10, 100),
    (1024, 10, 900),
]


@pytest.mark.gpu
@pytest.mark.parametrize("E,k,T", CASES)
@pytest.mark.parametrize("mode", ["plain", "skip", "range", "range+skip"])
def test_grouping_matches_host_counting_sort(torch_cuda, E, k, T, mode):
    import bit_expert_ffn_gemv_b200 as moe
    torch = torch_cuda
    rng = np.random.default_rng(E * 100003 + T)
    ids_h = draw_ids(rng, T, E, k)
    w_h = rng.random((T, k), dtype=np.float32)
    h = moe.MoeLayer(256, 128, E, k, 1, 1, 2, max(T, 16))
    try:
        e_begin, e_end = (E // 5, E // 5 + E // 3) if "range" in mode else (0, 1 << 30)
        if "range" in mode:
            h.set_expert_range(e_begin, e_end)
        flags = moe.MOE_ROUTE_TAIL_SKIP if "skip" in mode else 0
        ids = torch.from_numpy(ids_h).cuda()
        w = torch.from_numpy(w_h).cuda()
        off, pairs, inv, act, ws = h.bucket(ids, w, flags=flags)
        torch.cuda.synchronize()
        assert h.check_status() == 0
        r_off, r_pairs, r_inv, r_act = host_grouping(ids_h, E, SKIP_RANK if "skip" in mode else 0, e_begin, e_end)
        n = int(r_off[-1])
        assert np.array_equal(off.cpu().numpy(), r_off), "offsets"
        assert np.array_equal(pairs.cpu().numpy()[:n], r_pairs), "pairs (stable order)"
        assert np.array_equal(inv.cpu().numpy(), r_inv), "inverse positions"
        assert np.array_equal(act.cpu().numpy()[:r_act.size], r_act), "active experts"
        assert np.array_equal(ws.cpu().numpy()[:n], w_h.reshape(-1)[r_pairs]), "weights in group order"
    finally:
        h.close()


@pytest.mark.gpu
def test_out_of_range_id_sets_bounds_status(torch_cuda):
    """An id outside [0, E) is skipped and reported as MOE_ERR_BOUNDS (host-made input, no device fault)."""
    import bit_expert_ffn_gemv_b200 as moe
    torch = torch_cuda
    E, k, T = 16, 2, 8
    ids_h = draw_ids(np.random.default_rng(5), T, E, k)
    ids_h[3, 1] = E + 4
    h = moe.MoeLayer(256, 128, E, k, 1, 1, 2, T)
    try:
        off, pairs, inv, act, _ = h.bucket(torch.from_numpy(ids_h).cuda())
        torch.cuda.synchronize()
        assert moe.STATUS[h.check_status()] == "MOE_ERR_BOUNDS"
        assert int(off[-1]) == T * k - 1 and int(inv[3 * k + 1]) == -1
    finally:
        h.close()
