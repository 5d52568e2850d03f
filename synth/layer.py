"""Workload definitions and per-layer input builders (host side).

A layer's packed expert weights are laid out expert-major: expert e (the
shared expert is index E) holds three matrices in the order gate [f x d],
up [f x d], down [d x f], each in the tiled format described in synth.c.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

from . import (MASTER_BASE, MAT_TENSOR, T_PERM, T_WR, T_X, codes_bytes, expert_matrix, key, normal_bf16,
               scales_bytes, zipf_bias)

__all__ = ["MoeShape", "Workload", "WORKLOADS", "mat_dims", "mat_bits", "expert_bytes", "router_host", "expert_host",
           "layer_host", "x_host"]


@dataclass(frozen=True)
class MoeShape:
    d: int
    f: int
    E: int
    k: int
    n_shared: int = 1
    bits: int = 2
    bits_down: int = 0  # code width of the down matrices; 0: bits (per-tensor mixed precision otherwise)

    @property
    def n_experts_total(self) -> int:
        return self.E + self.n_shared

    @property
    def bd(self) -> int:
        return self.bits_down or self.bits


@dataclass(frozen=True)
class Workload:
    name: str
    shape: MoeShape
    tokens: tuple
    layers: int
    zipf: bool
    master: int
    chunks: int = 1
    bits_sweep: tuple = field(default=())


def _full(bits: int = 2) -> MoeShape:
    return MoeShape(d=2048, f=768, E=512, k=10, n_shared=1, bits=bits)


# The five synthetic workloads: a tiny layer; one full-shape decode layer; the
# 48-layer resident chain; 4 x 8192-token prefill chunks; the bit/batch sweep.
WORKLOADS = {
    "tiny": Workload("tiny", MoeShape(d=256, f=128, E=16, k=2, n_shared=1, bits=2), (8,), 1, False,
                     MASTER_BASE + 1),
    "decode": Workload("decode", _full(), (1, 4), 1, True, MASTER_BASE + 2),
    "chain48": Workload("chain48", _full(), (1, 4), 48, True, MASTER_BASE + 3),
    "prefill": Workload("prefill", _full(), (8192,), 1, True, MASTER_BASE + 4, chunks=4),
    "sweep": Workload("sweep", _full(), (1, 4, 16, 64, 512, 8192), 1, True, MASTER_BASE + 5, bits_sweep=(2, 3, 4)),
}


def mat_dims(shape: MoeShape, mat: int):
    """(N, K) of matrix mat: 0 gate [f x d], 1 up [f x d], 2 down [d x f]."""
    return (shape.f, shape.d) if mat < 2 else (shape.d, shape.f)


def mat_bits(shape: MoeShape, mat: int) -> int:
    """Code width of matrix mat: gate and up at `bits`, down at `bits_down` (when set)."""
    return shape.bd if mat == 2 else shape.bits


def expert_bytes(shape: MoeShape):
    """(codes bytes, scale bytes) of one expert's three matrices."""
    n = shape.f * shape.d
    return n * (2 * shape.bits + shape.bd) // 8, 3 * (n // 32) * 2


def router_host(shape: MoeShape, master: int, layer: int, zipf: bool):
    """Router weights (bf16 bits [E, d], std 0.02) and Zipf(1.1) log-prior bias (or None)."""
    wr = normal_bf16(key(master, layer, T_WR), shape.E * shape.d, 0.02).reshape(shape.E, shape.d)
    bias = zipf_bias(key(master, layer, T_PERM), shape.E, 1.1) if zipf else None
    return wr, bias


def expert_host(shape: MoeShape, master: int, layer: int, expert: int):
    """Packed codes (uint8) and scales (uint16) of one expert: gate, up, down back to back."""
    cb, sb = expert_bytes(shape)
    codes = np.empty(cb, np.uint8)
    scales = np.empty(sb // 2, np.uint16)
    co = so = 0
    for mat in range(3):
        N, K = mat_dims(shape, mat)
        c, s = expert_matrix(key(master, layer, MAT_TENSOR[mat], expert), N, K, mat_bits(shape, mat))
        codes[co:co + c.size] = c
        scales[so:so + s.size] = s
        co += c.size
        so += s.size
    assert co == cb and so * 2 == 3 * scales_bytes(shape.f, shape.d)
    return codes, scales


def layer_host(shape: MoeShape, master: int, layer: int, zipf: bool, experts=None):
    """Router + packed experts of one layer.

    experts: None for all E + n_shared experts, else an iterable of expert
    indices to materialise (the others are None in the returned lists).
    Returns dict(router_w, bias, codes=[...], scales=[...]).
    """
    wr, bias = router_host(shape, master, layer, zipf)
    n = shape.n_experts_total
    want = range(n) if experts is None else sorted(set(int(e) for e in experts))
    codes = [None] * n
    scales = [None] * n
    for e in want:
        codes[e], scales[e] = expert_host(shape, master, layer, e)
    return dict(router_w=wr, bias=bias, codes=codes, scales=scales)


def x_host(shape: MoeShape, master: int, stream: int, T: int) -> np.ndarray:
    """Activations x ~ N(0,1) as bf16 bits [T, d]; `stream` selects an independent draw."""
    return normal_bf16(key(master, stream, T_X), T * shape.d, 1.0).reshape(T, shape.d)
