"""Helpers shared by the GPU tests: upload synthetic layers, compare outputs."""
from __future__ import annotations

import numpy as np

import synth

# Output tolerance of the layer (bf16 activations, fp32 accumulation):
# relative L2 over the whole output and the largest absolute error.
REL_L2 = 2e-3
MAX_ABS = 1e-2
# fp32 output: no bf16 rounding of y; h is held in fp16 (2^-11 relative) and
# sums are fp32, so the error is far below the bf16 bar.
REL_L2_FP32 = 5e-4


def upload_layer(L: dict, device="cuda"):
    """Host layer dict (synth.layer_host) -> contiguous CUDA tensors."""
    import torch
    codes = torch.from_numpy(np.concatenate(L["codes"])).to(device)
    scales = torch.from_numpy(np.concatenate(L["scales"]).view(np.int16)).to(device)
    wr = torch.from_numpy(L["router_w"].view(np.int16)).to(device)
    bias = None if L["bias"] is None else torch.from_numpy(L["bias"]).to(device)
    return codes, scales, wr, bias


def x_to_device(x_bits: np.ndarray, device="cuda"):
    import torch
    return torch.from_numpy(x_bits.view(np.int16)).to(device).view(torch.bfloat16)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def rel_l2(got: np.ndarray, ref: np.ndarray) -> float:
    return float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))


def max_abs(got: np.ndarray, ref: np.ndarray) -> float:
    return float(np.abs(got - ref).max()) if got.size else 0.0


def y_to_f64(y) -> np.ndarray:
    import torch
    return y.float().cpu().numpy().astype(np.float64) if y.dtype != torch.float32 else y.cpu().numpy().astype(
        np.float64)


def make_layer_host(wl, layer=0, experts=None, shape=None):
    shape = shape or wl.shape
    return synth.layer_host(shape, wl.master, layer, wl.zipf, experts)


# Tokens per expert tile of the tensor-core path, and rows of its small
# activation box (groups of at most 64 tokens load 32-row boxes).
TILE_TOKENS = 256
SMALL_BOX_ROWS = 32
SMALL_GROUP = 64


def tile_cover_rows(ids: np.ndarray, E: int, n_shared: int = 1) -> np.ndarray:
    """Tokens to check so that every tile the tensor-core path forms holds at least one of them.

    Each routed expert's group (the tokens that selected it, ascending) is cut
    into tiles of 256 tokens, and groups of at most 64 tokens are loaded in
    32-row boxes; the shared expert's group is every token.  Greedily, each
    tile or box that holds no chosen token adds its last token (the ragged
    edge); the first and last token of the batch are always in.
    """
    T = ids.shape[0]
    sets = []
    for e in range(E):
        g = np.nonzero((ids == e).any(1))[0]
        step = SMALL_BOX_ROWS if 0 < g.size <= SMALL_GROUP else TILE_TOKENS
        sets += [g[s:s + step] for s in range(0, g.size, step)]
    if n_shared:
        sets += [np.arange(s, min(T, s + TILE_TOKENS)) for s in range(0, T, TILE_TOKENS)]
    chosen = {0, T - 1}
    for st in sets:
        if not chosen.intersection(st.tolist()):
            chosen.add(int(st[-1]))
    return np.array(sorted(chosen))
