"""The C-ABI library loads and exports what include/moe.h declares (no GPU needed)."""
import ctypes
import os
import re

import pytest

import bit_expert_ffn_gemv_b200 as moe
from bit_expert_ffn_gemv_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(moe_[a-z_0-9]+)\s*\(", src))
    return names


@pytest.fixture(scope="module")
def L():
    build.build()
    return moe.lib()


def test_every_declared_symbol_is_exported(L):
    names = _declared()
    assert {"moe_layer_init", "moe_load_layer", "moe_route", "moe_forward", "moe_destroy"} <= names
    for n in names:
        assert hasattr(L, n), n


def test_status_strings(L):
    for s, name in moe.STATUS.items():
        assert moe.moe_status_string(s)
    assert moe.moe_status_string(99) == "unknown status"


def _cfg(**kw):
    base = dict(d=256, f=128, n_experts=16, top_k=2, n_shared=1, n_layers=1, bits=2, max_tokens=8)
    base.update(kw)
    return moe.MoeConfig(**base)


@pytest.mark.parametrize("bad", [dict(d=200), dict(f=100), dict(n_experts=0), dict(n_experts=2000),
                                 dict(top_k=0), dict(top_k=17), dict(n_shared=2), dict(bits=1), dict(bits=5),
                                 dict(max_tokens=0), dict(n_layers=0), dict(top_k=33, n_experts=64),
                                 dict(bits_down=1), dict(bits_down=5)])
def test_init_rejects_bad_config_before_touching_the_gpu(L, bad):
    h = ctypes.c_void_p(1234)
    s = L.moe_layer_init(ctypes.byref(_cfg(**bad)), ctypes.byref(h))
    assert s == 1 and h.value is None  # MOE_ERR_INVALID_ARG, *out cleared


def test_null_arguments(L):
    assert L.moe_layer_init(None, None) == 1
    assert L.moe_set_expert_range(None, 0, 1, 1) == 1
    assert L.moe_destroy(None) == 0
    assert L.moe_route(None, 0, None, 1, None, None, None) == 1
    assert L.moe_forward(None, 0, None, 1, None, 0, None) == 1
    assert L.moe_forward_host(None, 0, None, 1, None, 0, None) == 1
    assert L.moe_load_layer(None, 0, None) == 1
    assert L.moe_debug_dequant(None, 0, 0, 0, None, None) == 1
    assert L.moe_check_status(None) == 1
    assert L.moe_debug_last_routing(None, 1, None, None, None) == 1
    assert L.moe_get_stats(None, None) == 1
    assert L.moe_profile(None, 1) == 1
    assert L.moe_profile_read(None, None, None) == 1
    assert moe.moe_kernel_name(0) == "router_logits" and moe.moe_kernel_name(99) == "unknown"


def test_flag_constants_match_the_header():
    """Every #define MOE_* value of the header equals the binding's constant of the same name."""
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    defs = dict(re.findall(r"#define\s+(MOE_[A-Z0-9_]+)\s+(0x[0-9a-fA-F]+|\d+)u?\b", src))
    assert {"MOE_OUT_FP32", "MOE_ROUTE_TAIL_SKIP", "MOE_TAIL_SKIP_RANK"} <= set(defs)
    for name, v in defs.items():
        assert getattr(moe, name) == int(v, 0), name


@pytest.mark.parametrize("bad", [dict(d=200), dict(d=8320), dict(T=129), dict(E=1025, T=1), dict(k=0), dict(k=33),
                                 dict(E=8, k=9), dict(T=-1), dict(x=0), dict(x=8), dict(w=0)])
def test_noalloc_route_rejects_bad_arguments_before_touching_the_gpu(L, bad):
    """Every limit moe_route_noalloc states is checked before any CUDA call (so this runs without a GPU)."""
    a = dict(x=256, T=4, d=256, E=512, k=10, wr=512, bias=None, ids=768, w=1024)
    a.update(bad)
    s = L.moe_route_noalloc(a["x"], a["T"], a["d"], a["E"], a["k"], a["wr"], a["bias"], a["ids"], a["w"], None)
    assert s == 1  # MOE_ERR_INVALID_ARG


@pytest.mark.parametrize("d,T,expect", [
    # split router GEMM (T <= 128): one K chunk per 64-wide step, at most 32 chunks
    (2048, 1, 34 * (2048 // 16 // 32) + 31 + 2), (2048, 16, 169.0), (2048, 64, 169.0), (2048, 128, 169.0),
    # 128-token tiles: four chunks fill the 512 tensor-memory columns
    (2048, 129, 34 * (2048 // 16 // 4) + 3 + 2), (2048, 8192, 1093.0), (2048, 0, 1093.0),
    # few K steps cap the chunk count (a power of two dividing d / 64)
    (128, 16, 34 * (128 // 16 // 2) + 1 + 2), (384, 16, 34 * (384 // 16 // 2) + 1 + 2),
    (384, 8192, 34 * (384 // 16 // 2) + 1 + 2), (256, 8192, 34 * (256 // 16 // 4) + 3 + 2),
])
def test_router_error_depth_follows_the_chunk_count(L, d, T, expect):
    """The tensor-core logits' depth is 34 per 16-wide step of one K chunk, plus one per chunk add and
    two for the bias: the chunk count is what the GEMM uses at that batch size (host logic only)."""
    import bit_expert_ffn_gemv_b200 as moe
    assert moe.moe_router_error_depth(d, True, T) == pytest.approx(expect)
    assert moe.moe_router_error_depth(d, True, T) <= moe.moe_router_error_depth(d, True)
    assert moe.moe_router_error_depth(d, False, T) == pytest.approx(d // 32 + 6)
    assert moe.moe_router_error_depth(0, True, T) == 0.0
