"""fp64 CPU oracle of the routed-MoE layer -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg (and its ``--impl reference`` arm) may import this package.  The product
path (``bit_expert_ffn_gemv_b200``) never does and has no CPU fallback.

The arithmetic lives in ``oracle.c`` (plain C, fp64, OpenMP over tokens); this
module compiles it with gcc on first use and marshals numpy arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "_oracle.so")
_lock = threading.Lock()
_lib = None


class Shape(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int32), ("f", ctypes.c_int32), ("E", ctypes.c_int32), ("k", ctypes.c_int32),
                ("n_shared", ctypes.c_int32), ("bits", ctypes.c_int32), ("bits_down", ctypes.c_int32)]


def build(force: bool = False) -> str:
    """Compile oracle.c into _oracle.so."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-std=c11", "-Wall", "-o", tmp, _SRC,
                               "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = ctypes.CDLL(_LIB)
            vp, i32 = ctypes.c_void_p, ctypes.c_int
            L.oracle_fp16.restype = ctypes.c_double
            L.oracle_fp16.argtypes = [ctypes.c_uint16]
            L.oracle_bf16.restype = ctypes.c_double
            L.oracle_bf16.argtypes = [ctypes.c_uint16]
            L.oracle_code.restype = i32
            L.oracle_code.argtypes = [vp, i32, i32, i32, i32, i32]
            L.oracle_dequant.restype = i32
            L.oracle_dequant.argtypes = [i32, i32, i32, vp, vp, vp]
            L.oracle_route.restype = i32
            L.oracle_route.argtypes = [ctypes.POINTER(Shape), vp, i32, vp, vp, vp, vp, vp]
            L.oracle_layer.restype = i32
            L.oracle_layer.argtypes = [ctypes.POINTER(Shape), vp, i32, vp, vp, vp, vp, vp, vp, vp, vp]
            L.oracle_threads.restype = i32
            L.oracle_threads.argtypes = [i32]
            _lib = L
    return _lib


def _p(a):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _shape(shape) -> Shape:
    return Shape(shape.d, shape.f, shape.E, shape.k, shape.n_shared, shape.bits, getattr(shape, "bits_down", 0))


def threads(n: int = 0) -> int:
    """Threads the oracle uses (n > 0 sets the count first)."""
    return int(lib().oracle_threads(n))


def fp16(h: int) -> float:
    return float(lib().oracle_fp16(h))


def dequant(codes: np.ndarray, scales: np.ndarray, N: int, K: int, bits: int) -> np.ndarray:
    """fp64 What[N, K] = q * s of one packed matrix."""
    out = np.empty((N, K), np.float64)
    rc = lib().oracle_dequant(N, K, bits, _p(np.ascontiguousarray(codes)), _p(np.ascontiguousarray(scales)),
                              _p(out))
    if rc != 0:
        raise ValueError("oracle_dequant: bad arguments")
    return out


def route(shape, x: np.ndarray, router_w: np.ndarray, bias, with_logits: bool = False):
    """Routing of T tokens: (ids [T,k] int32, w [T,k] f64[, logits [T,E] f64])."""
    x = np.ascontiguousarray(x, np.uint16)
    T = x.shape[0]
    ids = np.empty((T, shape.k), np.int32)
    w = np.empty((T, shape.k), np.float64)
    lg = np.empty((T, shape.E), np.float64) if with_logits else None
    b = None if bias is None else np.ascontiguousarray(bias, np.float32)
    rc = lib().oracle_route(ctypes.byref(_shape(shape)), _p(x), T, _p(np.ascontiguousarray(router_w, np.uint16)),
                            _p(b), _p(ids), _p(w), _p(lg))
    if rc != 0:
        raise ValueError("oracle_route: bad arguments")
    return (ids, w, lg) if with_logits else (ids, w)


def tail_skip(ids: np.ndarray, E: int, rank: int) -> np.ndarray:
    """Route-tail skip of one batch: drop[e] = 1 for every expert that some
    token of the batch selects and that every token selecting it ranks at
    position `rank` or later (0-based; 6 = "7th or lower" of a top-10).

    The rule of the discuss.pytorch.kr post, section "Strata's operating
    principle / experts split across VRAM, RAM and SSD": an expert that all
    the tokens processed together picked only at ranks 7 to 10 is skipped.
    Written as its definition: the best (lowest) rank of each expert over the
    batch, then the comparison.
    """
    T, k = ids.shape
    best = {}
    for t in range(T):
        for r in range(k):
            e = int(ids[t, r])
            best[e] = min(best.get(e, k), r)
    drop = np.zeros(E, np.uint8)
    for e, b in best.items():
        if b >= rank:
            drop[e] = 1
    return drop


def layer(shape, x: np.ndarray, router_w: np.ndarray, bias, codes: list, scales: list, drop=None):
    """Full layer: (y [T,d] f64, ids [T,k], w [T,k]).

    codes/scales: per-expert packed arrays (index E = shared expert); None for
    experts that no token selects.  drop: optional uint8 [E] mask (see
    tail_skip); the terms of dropped experts leave the routed sum and the
    other weights keep their values.
    """
    x = np.ascontiguousarray(x, np.uint16)
    T = x.shape[0]
    n = shape.E + shape.n_shared
    assert len(codes) == n and len(scales) == n
    cptr = (ctypes.c_void_p * n)(*[None if c is None else _p(c) for c in codes])
    sptr = (ctypes.c_void_p * n)(*[None if s is None else _p(s) for s in scales])
    y = np.empty((T, shape.d), np.float64)
    ids = np.empty((T, shape.k), np.int32)
    w = np.empty((T, shape.k), np.float64)
    b = None if bias is None else np.ascontiguousarray(bias, np.float32)
    dm = None if drop is None else np.ascontiguousarray(drop, np.uint8)
    assert dm is None or dm.shape == (shape.E,)
    rc = lib().oracle_layer(ctypes.byref(_shape(shape)), _p(x), T, _p(np.ascontiguousarray(router_w, np.uint16)),
                            _p(b), ctypes.cast(cptr, ctypes.c_void_p), ctypes.cast(sptr, ctypes.c_void_p), _p(dm),
                            _p(y), _p(ids), _p(w))
    if rc == -2:
        raise KeyError("oracle_layer: a selected expert was not materialised")
    if rc != 0:
        raise ValueError("oracle_layer: bad arguments")
    return y, ids, w
