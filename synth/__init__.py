"""Seeded synthetic inputs for the routed-MoE layer.

This package generates inputs only (activations, router weights, the Zipf
log-prior bias and quantised expert weights in the packed tiled format).  It
holds none of the layer's arithmetic.  The oracle (``oracle/``) and the CUDA
path (``bit_expert_ffn_gemv_b200``) both consume what it writes; neither is
imported here.

The host generator is ``synth.c`` (built on first use with gcc).  The device
generator ``synth_gpu.cu`` reproduces the same packed bytes on a GPU for the
multi-gigabyte workloads; ``tests/test_synth_gpu.py`` checks the two agree.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB = os.path.join(_HERE, "_synth.so")
_lock = threading.Lock()
_lib = None

# tensor ids inside one layer's key space
T_X, T_WR, T_PERM, T_WG, T_WU, T_WD = 0, 1, 2, 3, 4, 5
MAT_TENSOR = (T_WG, T_WU, T_WD)
MASTER_BASE = 0x5EED0000


def build(force: bool = False) -> str:
    """Compile synth.c into _synth.so (gcc, OpenMP, no FP contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off", "-std=c11",
             "-Wall", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = ctypes.CDLL(_LIB)
            u64, i64, i32, vp, d = ctypes.c_uint64, ctypes.c_int64, ctypes.c_int, ctypes.c_void_p, ctypes.c_double
            L.synth_key.restype = u64
            L.synth_key.argtypes = [u64, ctypes.c_uint32, ctypes.c_uint32, ctypes.c_uint32]
            L.synth_normal.restype = d
            L.synth_normal.argtypes = [u64, u64]
            L.synth_f32_to_bf16.restype = ctypes.c_uint16
            L.synth_f32_to_bf16.argtypes = [ctypes.c_float]
            L.synth_f32_to_f16.restype = ctypes.c_uint16
            L.synth_f32_to_f16.argtypes = [ctypes.c_float]
            L.synth_pack.restype = i32
            L.synth_pack.argtypes = [i32, i32, i32, vp, vp, vp, vp]
            L.synth_quantize.restype = i32
            L.synth_quantize.argtypes = [i32, i32, i32, vp, vp, vp, vp, vp]
            L.synth_normal_f32.restype = None
            L.synth_normal_f32.argtypes = [u64, i64, d, vp]
            L.synth_normal_bf16.restype = None
            L.synth_normal_bf16.argtypes = [u64, i64, d, vp]
            L.synth_expert_matrix.restype = i32
            L.synth_expert_matrix.argtypes = [u64, i32, i32, i32, vp, vp]
            L.synth_zipf_bias.restype = None
            L.synth_zipf_bias.argtypes = [u64, i32, d, vp]
            _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def key(master: int, layer: int, tensor: int, expert: int = 0) -> int:
    return int(lib().synth_key(master, layer, tensor, expert))


def normal_f32(k: int, n: int, std: float = 1.0) -> np.ndarray:
    out = np.empty(n, np.float32)
    lib().synth_normal_f32(k, n, std, _p(out))
    return out


def normal_bf16(k: int, n: int, std: float = 1.0) -> np.ndarray:
    """bf16 bit patterns (uint16) of round-to-nearest-even((float)(std*z))."""
    out = np.empty(n, np.uint16)
    lib().synth_normal_bf16(k, n, std, _p(out))
    return out


def codes_bytes(N: int, K: int, bits: int) -> int:
    return N * K * bits // 8


def scales_bytes(N: int, K: int) -> int:
    return N * (K // 32) * 2


def pack(q: np.ndarray, s: np.ndarray, bits: int):
    """Pack signed codes q[N,K] (int8) and fp16 scale bits s[N,K/32] (uint16)."""
    N, K = q.shape
    q = np.ascontiguousarray(q, np.int8)
    s = np.ascontiguousarray(s, np.uint16)
    assert s.shape == (N, K // 32)
    codes = np.empty(codes_bytes(N, K, bits), np.uint8)
    scales = np.empty(N * (K // 32), np.uint16)
    rc = lib().synth_pack(N, K, bits, _p(q), _p(s), _p(codes), _p(scales))
    if rc != 0:
        raise ValueError(f"synth_pack: bad shape {N}x{K} or bits {bits}")
    return codes, scales


def quantize(w: np.ndarray, bits: int):
    """Quantise fp32 w[N,K]; returns (codes, scales, q[N,K] int8, s[N,K/32] uint16)."""
    N, K = w.shape
    w = np.ascontiguousarray(w, np.float32)
    codes = np.empty(codes_bytes(N, K, bits), np.uint8)
    scales = np.empty(N * (K // 32), np.uint16)
    q = np.empty((N, K), np.int8)
    s = np.empty((N, K // 32), np.uint16)
    rc = lib().synth_quantize(N, K, bits, _p(w), _p(codes), _p(scales), _p(q), _p(s))
    if rc != 0:
        raise ValueError(f"synth_quantize: bad shape {N}x{K} or bits {bits}")
    return codes, scales, q, s


def expert_matrix(k: int, N: int, K: int, bits: int):
    codes = np.empty(codes_bytes(N, K, bits), np.uint8)
    scales = np.empty(N * (K // 32), np.uint16)
    rc = lib().synth_expert_matrix(k, N, K, bits, _p(codes), _p(scales))
    if rc != 0:
        raise ValueError("synth_expert_matrix failed")
    return codes, scales


def zipf_bias(k: int, E: int, s: float = 1.1) -> np.ndarray:
    out = np.empty(E, np.float32)
    lib().synth_zipf_bias(k, E, s, _p(out))
    return out


from .layer import *  # noqa: E402,F401,F403
