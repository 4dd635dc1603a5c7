"""CPU checks of the C ABI: the library loads, exports every entry point that
include/moe.h declares, and its host-side argument checks answer without a GPU."""
import ctypes
import os
import re

import pytest

import moe_inputs as mi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", text)) - {"MOE_ROUTER_SUM_DEPTH"})


def test_library_exports_every_declared_entry_point():
    import expert_ffn_layer_route_b200 as m
    L = m.lib()
    names = _declared()
    assert len(names) >= 18
    missing = [n for n in names if not hasattr(L, n)]
    assert missing == []
    assert sorted(m._native.EXPORTS) == names


def test_status_strings():
    import expert_ffn_layer_route_b200 as m
    assert m.moe_status_string(0) == "ok"
    assert "workspace" in m.moe_status_string(8)


def test_router_sum_depth_matches_header():
    import expert_ffn_layer_route_b200 as m
    for d in (256, 2048, 2049, 2880, 7168):
        assert m.router_sum_depth(d) == 8 * ((d + 2047) // 2048) + 12


@pytest.mark.parametrize("shape", [mi.TINY, mi.GPTOSS, mi.MIXTRAL, mi.KIMI, mi.BANK])
def test_workspace_size_and_layout(shape):
    import expert_ffn_layer_route_b200 as m
    for T in mi.CONFIG_TOKENS[shape.name]:
        d = m.make_desc(shape, T)
        n = m.moe_workspace_size(d)
        lay = m.moe_workspace_layout_of(d)
        assert lay.total == n
        offs = [lay.topk_idx, lay.topk_w, lay.offsets, lay.row_token, lay.inv]
        assert offs == sorted(offs) and all(o % 256 == 0 for o in offs)
        R = T * shape.top_k
        # at least: h, y and the routing arrays
        assert n >= R * shape.d_ff * 2 + R * shape.d_model * 2


def _status(fn, *args):
    return fn(*args)


def test_host_argument_checks_without_gpu():
    import expert_ffn_layer_route_b200 as m
    L = m.lib()
    good = m.make_desc(mi.TINY, 16)
    n = ctypes.c_size_t()
    bad_cases = [
        dict(d_model=100),            # not a multiple of 32
        dict(top_k=9),                # k > E
        dict(top_k=0),
        dict(wdtype=7),
        dict(T=-1),
        dict(router_fp32=2),
    ]
    for kw in bad_cases:
        d = m.make_desc(mi.TINY, 16)
        for k, v in kw.items():
            setattr(d, k, v)
        assert L.moe_workspace_size(ctypes.byref(d), ctypes.byref(n)) == 1, kw
    d = m.make_desc(mi.TINY.replace(wdtype="int4", d_model=192), 4)
    assert L.moe_workspace_size(ctypes.byref(d), ctypes.byref(n)) == 1  # INT4 needs multiples of 128
    d = m.make_desc(mi.TINY.replace(n_experts=2048), 4)
    assert L.moe_workspace_size(ctypes.byref(d), ctypes.byref(n)) == 2  # unsupported
    assert L.moe_workspace_size(None, ctypes.byref(n)) == 1
    # T = 0 is a no-op that returns OK before touching any pointer or the GPU
    z = m.make_desc(mi.TINY, 0)
    assert L.moe_layer_forward(ctypes.byref(z), None, None, None, None, None, None, None, 0, None) == 0
    assert L.moe_route_topk(ctypes.byref(z), None, None, None, None, None, None, 0, None) == 0
    # null / misaligned pointers are rejected synchronously
    assert L.moe_route_topk(ctypes.byref(good), None, None, None, None, None, None, 0, None) == 1
    assert L.moe_route_topk(ctypes.byref(good), 16, 32, None, 64, 128, 3, 1 << 20, None) == 1  # misaligned ws
    assert L.moe_route_topk(ctypes.byref(good), 16, 32, None, 64, 128, 256, 16, None) == 8   # workspace too small
    w = m.Weights()
    assert L.moe_layer_forward(ctypes.byref(good), 16, 32, None, ctypes.byref(w), None, 48, 256, 1 << 30, None) == 1
    w.w13, w.w2 = 4096, 8192
    w.stride_w13 = 8  # not a multiple of 16
    assert L.moe_layer_forward(ctypes.byref(good), 16, 32, None, ctypes.byref(w), None, 48, 256, 1 << 30, None) == 1


def test_cache_argument_checks_without_gpu():
    import expert_ffn_layer_route_b200 as m
    L = m.lib()
    h = ctypes.c_void_p()
    for bad in [m.CacheDesc(0, 8, 2, 1024, None, 0), m.CacheDesc(2, 8, 9, 1024, None, 0),
                m.CacheDesc(2, 8, 2, 1000, None, 0), m.CacheDesc(2, 2048, 2, 1024, None, 0)]:
        assert L.moe_cache_init(ctypes.byref(h), ctypes.byref(bad)) == 1
    assert L.moe_cache_destroy(None) == 1
