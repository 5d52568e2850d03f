"""Device generator (synth_gpu.cu): the same packed inputs as synth.c, written to GPU memory.

Used for workloads whose weights are too large to generate on the host (a
full-shape layer is 2.4e9 weights).  tests/test_synth_gpu.py checks the bytes
equal the host generator's.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

from . import MAT_TENSOR, T_PERM, T_WR, T_X, key, zipf_bias
from .layer import MoeShape, expert_bytes

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth_gpu.cu")
_LIB = os.path.join(_HERE, "_synth_gpu.so")
_lock = threading.Lock()
_lib = None
assert MAT_TENSOR == (3, 4, 5)  # synth_gpu.cu uses tensor id 3 + matrix


def build(force: bool = False) -> str:
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call([os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc"), "-gencode",
                               "arch=compute_100a,code=sm_100a", "-O3", "-fmad=false", "-std=c++17", "-Xcompiler",
                               "-fPIC", "-shared", "-o", tmp, _SRC])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = ctypes.CDLL(_LIB)
            u64, i32, vp = ctypes.c_uint64, ctypes.c_int, ctypes.c_void_p
            L.synth_gpu_experts.restype = i32
            L.synth_gpu_experts.argtypes = [u64, ctypes.c_uint32, i32, i32, i32, i32, i32, i32, vp, vp, vp]
            L.synth_gpu_normal_bf16.restype = i32
            L.synth_gpu_normal_bf16.argtypes = [u64, ctypes.c_int64, ctypes.c_double, vp, vp]
            L.synth_gpu_key.restype = u64
            L.synth_gpu_key.argtypes = [u64, ctypes.c_uint32, ctypes.c_uint32, ctypes.c_uint32]
            _lib = L
    return _lib


def _stream():
    import torch
    return torch.cuda.current_stream().cuda_stream


def experts_into(codes, scales, shape: MoeShape, master: int, layer: int, expert0: int, n: int):
    """Generate experts expert0..expert0+n-1 of a layer into CUDA tensors (uint8 / int16)."""
    cb, sb = expert_bytes(shape)
    assert codes.numel() >= n * cb and scales.numel() * 2 >= n * sb
    rc = lib().synth_gpu_experts(master, layer, shape.d, shape.f, expert0, n, shape.bits, shape.bd, codes.data_ptr(),
                                 scales.data_ptr(), _stream())
    if rc != 0:
        raise RuntimeError(f"synth_gpu_experts failed ({rc})")


def normal_bf16(k: int, n: int, std: float, device="cuda"):
    """bf16 tensor of n normals (same bits as synth.normal_bf16)."""
    import torch
    out = torch.empty(n, dtype=torch.bfloat16, device=device)
    rc = lib().synth_gpu_normal_bf16(k, n, std, out.data_ptr(), _stream())
    if rc != 0:
        raise RuntimeError("synth_gpu_normal_bf16 failed")
    return out


def layer_device(shape: MoeShape, master: int, layer: int, zipf: bool, device="cuda"):
    """(codes uint8, scales int16, router_w bf16 [E,d], bias fp32 or None) of one layer on the GPU."""
    import torch
    cb, sb = expert_bytes(shape)
    n = shape.n_experts_total
    codes = torch.empty(n * cb, dtype=torch.uint8, device=device)
    scales = torch.empty(n * sb // 2, dtype=torch.int16, device=device)
    experts_into(codes, scales, shape, master, layer, 0, n)
    wr = normal_bf16(key(master, layer, T_WR), shape.E * shape.d, 0.02, device).view(shape.E, shape.d)
    bias = torch.from_numpy(zipf_bias(key(master, layer, T_PERM), shape.E, 1.1)).to(device) if zipf else None
    return codes, scales, wr, bias


def x_device(shape: MoeShape, master: int, stream_id: int, T: int, device="cuda"):
    return normal_bf16(key(master, stream_id, T_X), T * shape.d, 1.0, device).view(T, shape.d)
