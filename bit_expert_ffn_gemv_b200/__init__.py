"""Thin Python binding of libmoe.so, the B200 routed-MoE layer (C ABI in include/moe.h).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  PyTorch supplies device memory and the CUDA stream.  There is no
CPU fallback: if the library is missing, importing the binding's functions
raises.

Module-level functions carry the C names (moe_layer_init, moe_load_layer,
moe_route, moe_forward, moe_forward_host, moe_destroy, moe_debug_dequant,
moe_check_status, moe_get_stats, moe_status_string); ``MoeLayer`` wraps a
handle for torch tensors.
"""
from __future__ import annotations

import ctypes
import os
import threading

__all__ = ["MoeError", "MoeConfig", "MoeLayerWeights", "MoeLayer", "lib", "library_path", "MOE_OUT_FP32",
           "MOE_ACCUMULATE", "MOE_FORCE_GEMV", "MOE_FORCE_GEMM", "MOE_FORCE_UNFUSED", "MOE_ROUTE_TAIL_SKIP",
           "MOE_TAIL_SKIP_RANK", "MOE_NORM_INPUT", "STATUS", "moe_layer_init", "moe_load_layer",
           "moe_route", "moe_route_noalloc", "moe_forward", "moe_forward_host", "moe_destroy", "moe_debug_dequant", "moe_debug_last_routing", "moe_debug_bucket", "moe_check_status",
           "moe_get_stats", "moe_status_string", "moe_profile", "moe_profile_read", "moe_kernel_name", "MoeStats",
           "moe_debug_router_logits", "moe_router_error_depth", "moe_rms_normalize", "rms_normalize",
           "moe_set_expert_range", "moe_debug_wait_limit"]

_HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_HERE, "libmoe.so")

MOE_OUT_FP32 = 0x1
MOE_ACCUMULATE = 0x2
MOE_FORCE_GEMV = 0x4
MOE_FORCE_GEMM = 0x8
MOE_FORCE_UNFUSED = 0x10
MOE_ROUTE_TAIL_SKIP = 0x20  # drop experts that every selecting token ranks >= MOE_TAIL_SKIP_RANK
MOE_TAIL_SKIP_RANK = 6
MOE_NORM_INPUT = 0x40  # the layer reads rmsnorm(x); with MOE_ACCUMULATE and y == x: x += layer(rmsnorm(x))
STATUS = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_CUDA", 3: "MOE_ERR_OOM", 4: "MOE_ERR_NOT_LOADED",
          5: "MOE_ERR_TIMEOUT", 6: "MOE_ERR_BOUNDS", 7: "MOE_ERR_RANGE"}


class MoeError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)} ({_status_text(status)})")


class MoeConfig(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int32), ("f", ctypes.c_int32), ("n_experts", ctypes.c_int32),
                ("top_k", ctypes.c_int32), ("n_shared", ctypes.c_int32), ("n_layers", ctypes.c_int32),
                ("bits", ctypes.c_int32), ("max_tokens", ctypes.c_int32), ("bits_down", ctypes.c_int32)]


class MoeStats(ctypes.Structure):
    _fields_ = [("fixup_tokens", ctypes.c_int64), ("active_experts", ctypes.c_int64), ("max_group", ctypes.c_int64),
                ("launches", ctypes.c_int64), ("cuda_error", ctypes.c_int64)]


MOE_KERNEL_COUNT = 13


class MoeLayerWeights(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("router_w", ctypes.c_void_p),
                ("router_bias", ctypes.c_void_p)]


_lock = threading.Lock()
_lib = None


def lib() -> ctypes.CDLL:
    """Load libmoe.so (built by bit_expert_ffn_gemv_b200.build); raise if it is absent."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(library_path):
                raise ImportError(f"{library_path} is missing: build it with `python -m bit_expert_ffn_gemv_b200.build`"
                                  " (there is no CPU fallback)")
            L = ctypes.CDLL(library_path)
            vp, i32, u32, st = ctypes.c_void_p, ctypes.c_int32, ctypes.c_uint32, ctypes.c_int
            L.moe_layer_init.restype = st
            L.moe_layer_init.argtypes = [ctypes.POINTER(MoeConfig), ctypes.POINTER(vp)]
            L.moe_load_layer.restype = st
            L.moe_load_layer.argtypes = [vp, i32, ctypes.POINTER(MoeLayerWeights)]
            L.moe_route.restype = st
            L.moe_route.argtypes = [vp, i32, vp, i32, vp, vp, vp]
            L.moe_forward.restype = st
            L.moe_forward.argtypes = [vp, i32, vp, i32, vp, u32, vp]
            L.moe_forward_host.restype = st
            L.moe_forward_host.argtypes = [vp, i32, vp, i32, vp, u32, vp]
            L.moe_destroy.restype = st
            L.moe_destroy.argtypes = [vp]
            L.moe_debug_dequant.restype = st
            L.moe_debug_dequant.argtypes = [vp, i32, i32, i32, vp, vp]
            L.moe_debug_last_routing.restype = st
            L.moe_debug_last_routing.argtypes = [vp, i32, vp, vp, vp]
            L.moe_debug_bucket.restype = st
            L.moe_debug_bucket.argtypes = [vp, vp, i32, vp, vp, vp, vp, vp, vp, u32, vp]
            L.moe_check_status.restype = st
            L.moe_check_status.argtypes = [vp]
            L.moe_get_stats.restype = st
            L.moe_get_stats.argtypes = [vp, ctypes.POINTER(MoeStats)]
            L.moe_profile.restype = st
            L.moe_profile.argtypes = [vp, i32]
            L.moe_profile_read.restype = st
            L.moe_profile_read.argtypes = [vp, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int64)]
            L.moe_kernel_name.restype = ctypes.c_char_p
            L.moe_kernel_name.argtypes = [i32]
            L.moe_route_noalloc.restype = st
            L.moe_route_noalloc.argtypes = [vp, i32, i32, i32, i32, vp, vp, vp, vp, vp]
            L.moe_debug_router_logits.restype = st
            L.moe_debug_router_logits.argtypes = [vp, i32, vp, i32, vp, i32, vp]
            L.moe_router_error_depth.restype = ctypes.c_float
            L.moe_router_error_depth.argtypes = [i32, i32, i32]
            L.moe_rms_normalize.restype = st
            L.moe_rms_normalize.argtypes = [vp, i32, i32, vp, vp]
            L.moe_set_expert_range.restype = st
            L.moe_set_expert_range.argtypes = [vp, i32, i32, i32]
            L.moe_debug_wait_limit.restype = st
            L.moe_debug_wait_limit.argtypes = [vp, u32, i32]
            L.moe_status_string.restype = ctypes.c_char_p
            L.moe_status_string.argtypes = [st]
            _lib = L
    return _lib


def _status_text(s: int) -> str:
    try:
        return lib().moe_status_string(s).decode()
    except Exception:  # pragma: no cover - library not loadable
        return "?"


def _check(s: int, what: str):
    if s != 0:
        raise MoeError(s, what)


# ---------------------------------------------------------------- C-named wrappers
def moe_layer_init(cfg: MoeConfig) -> int:
    h = ctypes.c_void_p()
    _check(lib().moe_layer_init(ctypes.byref(cfg), ctypes.byref(h)), "moe_layer_init")
    return h.value


def moe_load_layer(handle: int, layer: int, w: MoeLayerWeights) -> None:
    _check(lib().moe_load_layer(handle, layer, ctypes.byref(w)), "moe_load_layer")


def moe_route(handle: int, layer: int, x_ptr: int, T: int, ids_ptr: int, w_ptr: int, stream: int) -> None:
    _check(lib().moe_route(handle, layer, x_ptr, T, ids_ptr, w_ptr, stream), "moe_route")


def moe_forward(handle: int, layer: int, x_ptr: int, T: int, y_ptr: int, flags: int, stream: int) -> None:
    _check(lib().moe_forward(handle, layer, x_ptr, T, y_ptr, flags, stream), "moe_forward")


def moe_forward_host(handle: int, layer: int, x_host: int, T: int, y_host: int, flags: int, stream: int) -> None:
    _check(lib().moe_forward_host(handle, layer, x_host, T, y_host, flags, stream), "moe_forward_host")


def moe_route_noalloc(x_ptr: int, T: int, d: int, n_experts: int, top_k: int, router_w_ptr: int, bias_ptr,
                      ids_ptr: int, w_ptr: int, stream: int) -> None:
    """Routing for callers that cannot allocate device memory (no handle; fixed in-library scratch)."""
    _check(lib().moe_route_noalloc(x_ptr, T, d, n_experts, top_k, router_w_ptr, bias_ptr, ids_ptr, w_ptr, stream),
           "moe_route_noalloc")


def moe_set_expert_range(handle: int, begin: int, end: int, with_shared: int) -> None:
    _check(lib().moe_set_expert_range(handle, begin, end, with_shared), "moe_set_expert_range")


def moe_debug_wait_limit(handle: int, spins: int, withhold_cta: int = -1) -> None:
    """Test hook: device-side waits give up after `spins` polls; CTA withhold_cta withholds its router rows."""
    _check(lib().moe_debug_wait_limit(handle, spins, withhold_cta), "moe_debug_wait_limit")


def moe_destroy(handle: int) -> None:
    _check(lib().moe_destroy(handle), "moe_destroy")


def moe_debug_dequant(handle: int, layer: int, expert: int, mat: int, out_ptr: int, stream: int) -> None:
    _check(lib().moe_debug_dequant(handle, layer, expert, mat, out_ptr, stream), "moe_debug_dequant")


def moe_debug_bucket(handle: int, ids_ptr: int, T: int, w_ptr, offsets_ptr: int, pairs_ptr: int, inv_ptr: int,
                     active_ptr: int, wsorted_ptr, flags: int, stream: int) -> None:
    _check(lib().moe_debug_bucket(handle, ids_ptr, T, w_ptr, offsets_ptr, pairs_ptr, inv_ptr, active_ptr, wsorted_ptr,
                                  flags, stream), "moe_debug_bucket")


def moe_debug_last_routing(handle: int, T: int, ids_ptr: int, w_ptr: int, stream: int) -> None:
    _check(lib().moe_debug_last_routing(handle, T, ids_ptr, w_ptr, stream), "moe_debug_last_routing")


def moe_debug_router_logits(handle: int, layer: int, x_ptr: int, T: int, logits_ptr: int, tensor_cores: bool,
                            stream: int) -> None:
    _check(lib().moe_debug_router_logits(handle, layer, x_ptr, T, logits_ptr, 1 if tensor_cores else 0, stream),
           "moe_debug_router_logits")


def moe_router_error_depth(d: int, tensor_cores: bool, T: int = 0) -> float:
    return float(lib().moe_router_error_depth(d, T, 1 if tensor_cores else 0))


def moe_rms_normalize(x_ptr: int, T: int, d: int, out_ptr: int, stream: int) -> None:
    _check(lib().moe_rms_normalize(x_ptr, T, d, out_ptr, stream), "moe_rms_normalize")


def moe_check_status(handle: int) -> int:
    return int(lib().moe_check_status(handle))


def moe_get_stats(handle: int):
    st = MoeStats()
    _check(lib().moe_get_stats(handle, ctypes.byref(st)), "moe_get_stats")
    return {f: int(getattr(st, f)) for f, _ in MoeStats._fields_}


def moe_profile(handle: int, enable: bool) -> None:
    _check(lib().moe_profile(handle, 1 if enable else 0), "moe_profile")


def moe_profile_read(handle: int):
    """{kernel name: (total ms, launches)} of kernels launched since moe_profile(h, True)."""
    ms = (ctypes.c_double * MOE_KERNEL_COUNT)()
    n = (ctypes.c_int64 * MOE_KERNEL_COUNT)()
    _check(lib().moe_profile_read(handle, ms, n), "moe_profile_read")
    return {moe_kernel_name(i): (ms[i], n[i]) for i in range(MOE_KERNEL_COUNT) if n[i]}


def moe_kernel_name(i: int) -> str:
    return lib().moe_kernel_name(i).decode()


def moe_status_string(s: int) -> str:
    return lib().moe_status_string(s).decode()


# ---------------------------------------------------------------- torch convenience
def _stream_ptr(stream) -> int:
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(s.cuda_stream)


def rms_normalize(x, out=None, stream=None):
    """bf16 [T, d] -> bf16 x / rms(x) per row (the residual-stream pre-norm of a layer chain)."""
    import torch
    if out is None:
        out = torch.empty_like(x)
    moe_rms_normalize(x.data_ptr(), x.shape[0], x.shape[1], out.data_ptr(), _stream_ptr(stream))
    return out


class MoeLayer:
    """A handle holding up to n_layers routed-MoE layers (weights borrowed from torch tensors)."""

    def __init__(self, d, f, n_experts, top_k, n_shared=1, n_layers=1, bits=2, max_tokens=64, bits_down=0):
        self.cfg = MoeConfig(d, f, n_experts, top_k, n_shared, n_layers, bits, max_tokens, bits_down)
        self.handle = moe_layer_init(self.cfg)
        self._keep = {}

    def load_layer(self, layer, codes, scales, router_w, router_bias=None):
        """codes (uint8), scales (fp16 bits as int16/uint16/float16), router_w (bf16 bits or bf16), bias fp32."""
        for t in (codes, scales, router_w) + ((router_bias,) if router_bias is not None else ()):
            if not t.is_cuda or not t.is_contiguous():
                raise ValueError("weights must be contiguous CUDA tensors")
        w = MoeLayerWeights(codes.data_ptr(), scales.data_ptr(), router_w.data_ptr(),
                            router_bias.data_ptr() if router_bias is not None else None)
        moe_load_layer(self.handle, layer, w)
        self._keep[layer] = (codes, scales, router_w, router_bias)

    def route(self, layer, x, ids=None, w=None, stream=None):
        import torch
        T = x.shape[0]
        if ids is None:
            ids = torch.empty((T, self.cfg.top_k), dtype=torch.int32, device=x.device)
        if w is None:
            w = torch.empty((T, self.cfg.top_k), dtype=torch.float32, device=x.device)
        moe_route(self.handle, layer, x.data_ptr(), T, ids.data_ptr(), w.data_ptr(), _stream_ptr(stream))
        return ids, w

    def forward(self, layer, x, y=None, flags=0, stream=None):
        import torch
        T = x.shape[0]
        if y is None:
            dt = torch.float32 if flags & MOE_OUT_FP32 else torch.bfloat16
            y = torch.empty((T, self.cfg.d), dtype=dt, device=x.device)
        moe_forward(self.handle, layer, x.data_ptr(), T, y.data_ptr(), flags, _stream_ptr(stream))
        return y

    def forward_host(self, layer, x_host, y_host, flags=0, stream=None):
        moe_forward_host(self.handle, layer, x_host.data_ptr(), x_host.shape[0], y_host.data_ptr(), flags,
                         _stream_ptr(stream))
        return y_host

    def debug_dequant(self, layer, expert, mat, out=None, stream=None):
        import torch
        N, K = (self.cfg.f, self.cfg.d) if mat < 2 else (self.cfg.d, self.cfg.f)
        if out is None:
            out = torch.empty((N, K), dtype=torch.float32, device="cuda")
        moe_debug_dequant(self.handle, layer, expert, mat, out.data_ptr(), _stream_ptr(stream))
        return out

    def last_routing(self, T, stream=None):
        """(ids, w) the last forward computed internally for its T tokens."""
        import torch
        ids = torch.empty((T, self.cfg.top_k), dtype=torch.int32, device="cuda")
        w = torch.empty((T, self.cfg.top_k), dtype=torch.float32, device="cuda")
        moe_debug_last_routing(self.handle, T, ids.data_ptr(), w.data_ptr(), _stream_ptr(stream))
        return ids, w

    def bucket(self, ids, w=None, flags=0, stream=None):
        """The grouping step alone on ids [T x k]: (offsets, pairs, inv, active, wsorted or None)."""
        import torch
        T = ids.shape[0]
        n = T * self.cfg.top_k
        offsets = torch.full((self.cfg.n_experts + 1,), -7, dtype=torch.int32, device="cuda")
        pairs = torch.full((max(n, 4),), -7, dtype=torch.int32, device="cuda")
        inv = torch.full((max(n, 4),), -7, dtype=torch.int32, device="cuda")
        active = torch.full((self.cfg.n_experts,), -7, dtype=torch.int32, device="cuda")
        wsorted = torch.full((max(n, 4),), -7.0, dtype=torch.float32, device="cuda") if w is not None else None
        moe_debug_bucket(self.handle, ids.data_ptr(), T, w.data_ptr() if w is not None else None, offsets.data_ptr(),
                         pairs.data_ptr(), inv.data_ptr(), active.data_ptr(),
                         wsorted.data_ptr() if wsorted is not None else None, flags, _stream_ptr(stream))
        return offsets, pairs[:n], inv[:n], active, (wsorted[:n] if wsorted is not None else None)

    def router_logits(self, layer, x, tensor_cores=True, stream=None):
        """fp32 logits [T x E] from one of the two router kernels (for bound checks)."""
        import torch
        out = torch.empty((x.shape[0], self.cfg.n_experts), dtype=torch.float32, device=x.device)
        moe_debug_router_logits(self.handle, layer, x.data_ptr(), x.shape[0], out.data_ptr(), tensor_cores,
                                _stream_ptr(stream))
        return out

    def check_status(self) -> int:
        return moe_check_status(self.handle)

    def stats(self):
        return moe_get_stats(self.handle)

    def profile(self, enable: bool):
        moe_profile(self.handle, enable)

    def profile_read(self):
        return moe_profile_read(self.handle)

    def set_expert_range(self, begin, end, with_shared=True):
        """Compute only routed experts [begin, end) (and the shared one if with_shared) from now on."""
        moe_set_expert_range(self.handle, begin, end, 1 if with_shared else 0)

    def debug_wait_limit(self, spins: int, withhold_cta: int = -1):
        """Test hook of the device watchdog (see moe_debug_wait_limit in include/moe.h)."""
        moe_debug_wait_limit(self.handle, spins, withhold_cta)

    def close(self):
        if self.handle:
            moe_destroy(self.handle)
            self.handle = None
            self._keep = {}

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
