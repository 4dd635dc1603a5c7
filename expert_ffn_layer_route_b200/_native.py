"""ctypes declarations of ``include/moe.h`` and thin wrappers over torch tensors."""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional, Sequence

_HERE = os.path.dirname(os.path.abspath(__file__))
lib_path = os.path.join(_HERE, "libmoe_b200.so")

WDTYPE = {"bf16": 0, "mxfp4": 1, "nvfp4": 2, "int4": 3}
_BLOCK = {"bf16": 1, "mxfp4": 32, "nvfp4": 16, "int4": 128}

MOE_OK = 0


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: status {status} ({moe_status_string(status)})")


class LayerDesc(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("d_model", ctypes.c_int32), ("n_experts", ctypes.c_int32),
                ("top_k", ctypes.c_int32), ("d_ff", ctypes.c_int32), ("n_shared", ctypes.c_int32),
                ("wdtype", ctypes.c_int32), ("router_fp32", ctypes.c_int32)]


class Weights(ctypes.Structure):
    _fields_ = [("w13", ctypes.c_void_p), ("s13", ctypes.c_void_p), ("w2", ctypes.c_void_p),
                ("s2", ctypes.c_void_p), ("g13", ctypes.c_void_p), ("g2", ctypes.c_void_p),
                ("stride_w13", ctypes.c_int64), ("stride_s13", ctypes.c_int64),
                ("stride_w2", ctypes.c_int64), ("stride_s2", ctypes.c_int64),
                ("slot_map", ctypes.c_void_p), ("n_physical", ctypes.c_int32)]


class WorkspaceLayout(ctypes.Structure):
    _fields_ = [("topk_idx", ctypes.c_size_t), ("topk_w", ctypes.c_size_t), ("offsets", ctypes.c_size_t),
                ("row_token", ctypes.c_size_t), ("inv", ctypes.c_size_t), ("total", ctypes.c_size_t)]


class CacheDesc(ctypes.Structure):
    _fields_ = [("n_layers", ctypes.c_int32), ("n_experts", ctypes.c_int32),
                ("slots_per_layer", ctypes.c_int32), ("expert_bytes", ctypes.c_int64),
                ("host_bank", ctypes.c_void_p), ("device", ctypes.c_int32)]


class ProfileEntry(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 32), ("launches", ctypes.c_int64), ("total_ms", ctypes.c_double)]


class CacheStats(ctypes.Structure):
    _fields_ = [("lookups", ctypes.c_int64), ("hits", ctypes.c_int64), ("misses", ctypes.c_int64),
                ("evictions", ctypes.c_int64), ("prefetch_issued", ctypes.c_int64),
                ("prefetch_used", ctypes.c_int64), ("bytes_h2d", ctypes.c_int64), ("copy_ms", ctypes.c_double)]

    def as_dict(self):
        return {f: getattr(self, f) for f, _ in self._fields_}


_LIB = None

_P = ctypes.c_void_p
_DP = ctypes.POINTER(LayerDesc)
_WP = ctypes.POINTER(Weights)

_SIGS = {
    "moe_workspace_size": [_DP, ctypes.POINTER(ctypes.c_size_t)],
    "moe_workspace_layout_of": [_DP, ctypes.POINTER(WorkspaceLayout)],
    "moe_route_topk": [_DP, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P],
    "moe_route_topk_noalloc": [_DP, _P, _P, _P, _P, _P, _P],
    "moe_permute": [_DP, _P, _P, _P, _P, _P, _P, _P],
    "moe_grouped_ffn": [_DP, _WP, _WP, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P],
    "moe_combine": [_DP, _P, _P, _P, _P, _P, _P],
    "moe_layer_forward": [_DP, _P, _P, _P, _WP, _WP, _P, _P, ctypes.c_size_t, _P],
    "moe_cache_init": [ctypes.POINTER(_P), ctypes.POINTER(CacheDesc)],
    "moe_cache_prefetch": [_P, ctypes.c_int32, ctypes.POINTER(ctypes.c_int32), ctypes.c_int32],
    "moe_cache_lookup": [_P, ctypes.c_int32, ctypes.POINTER(ctypes.c_int32), ctypes.c_int32, _P, _P],
    "moe_cache_release": [_P, ctypes.c_int32, _P],
    "moe_cache_slot_map": [_P, ctypes.c_int32, ctypes.POINTER(ctypes.c_int32)],
    "moe_cache_stats": [_P, ctypes.POINTER(CacheStats)],
    "moe_cache_destroy": [_P],
    "moe_get_last_error": [],
    "moe_profile_enable": [ctypes.c_int],
    "moe_diag_wait_timeout": [ctypes.c_uint64, _P, _P],
    "moe_profile_collect": [ctypes.POINTER(ProfileEntry), ctypes.c_int32, ctypes.POINTER(ctypes.c_int32)],
}
_PTR_RET = {"moe_cache_host_expert": [_P, ctypes.c_int32, ctypes.c_int32],
            "moe_cache_slot_base": [_P, ctypes.c_int32]}

EXPORTS = sorted(list(_SIGS) + list(_PTR_RET) + ["moe_status_string"])


def lib() -> ctypes.CDLL:
    """The loaded CUDA library; raises if it has not been built."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(lib_path):
            raise ImportError(f"{lib_path} is missing: build it with `python -m expert_ffn_layer_route_b200.build`")
        L = ctypes.CDLL(lib_path)
        for name, args in _SIGS.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = ctypes.c_int
        for name, args in _PTR_RET.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = ctypes.c_void_p
        L.moe_status_string.argtypes = [ctypes.c_int]
        L.moe_status_string.restype = ctypes.c_char_p
        _LIB = L
    return _LIB


def moe_status_string(status: int) -> str:
    try:
        return lib().moe_status_string(status).decode()
    except ImportError:
        return "?"


def _check(status: int, where: str):
    if status != MOE_OK:
        raise MoeError(status, where)


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is not None:
        return stream if isinstance(stream, int) else stream.cuda_stream
    import torch

    return torch.cuda.current_stream().cuda_stream


def router_sum_depth(d: int) -> int:
    """MOE_ROUTER_SUM_DEPTH(d) of the header."""
    return 8 * ((d + 2047) // 2048) + 12


def make_desc(shape, T: int) -> LayerDesc:
    """LayerDesc from a ``moe_inputs.LayerShape``-like object."""
    return LayerDesc(int(T), shape.d_model, shape.n_experts, shape.top_k, shape.d_ff, shape.n_shared,
                     WDTYPE[shape.wdtype], 1 if shape.router_fp32 else 0)


def make_weights(experts: Dict[str, object], slot_map=None, n_physical: int = 0,
                 strides: Optional[Sequence[int]] = None) -> Weights:
    """Weights from a dict of device tensors w13/s13/w2/s2/g13/g2 (missing = NULL)."""
    w = Weights()
    for key in ("w13", "s13", "w2", "s2", "g13", "g2"):
        setattr(w, key, _ptr(experts.get(key)))
    if strides is not None:
        w.stride_w13, w.stride_s13, w.stride_w2, w.stride_s2 = strides
    w.slot_map = _ptr(slot_map)
    w.n_physical = n_physical
    return w


def moe_workspace_size(desc: LayerDesc) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().moe_workspace_size(ctypes.byref(desc), ctypes.byref(n)), "moe_workspace_size")
    return n.value


def moe_workspace_layout_of(desc: LayerDesc) -> WorkspaceLayout:
    out = WorkspaceLayout()
    _check(lib().moe_workspace_layout_of(ctypes.byref(desc), ctypes.byref(out)), "moe_workspace_layout_of")
    return out


def moe_route_topk(desc, x, w_router, logit_bias, topk_idx, topk_w, workspace, stream=None):
    _check(lib().moe_route_topk(ctypes.byref(desc), _ptr(x), _ptr(w_router), _ptr(logit_bias), _ptr(topk_idx),
                                _ptr(topk_w), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                _stream(stream)), "moe_route_topk")


def moe_route_topk_noalloc(desc, x, w_router, logit_bias, topk_idx, topk_w, stream=None):
    """moe_route_topk with the library's fixed scratch (for callers that cannot allocate)."""
    _check(lib().moe_route_topk_noalloc(ctypes.byref(desc), _ptr(x), _ptr(w_router), _ptr(logit_bias),
                                        _ptr(topk_idx), _ptr(topk_w), _stream(stream)), "moe_route_topk_noalloc")


def moe_permute(desc, topk_idx, offsets, row_token, inv, stream=None, x=None, x_perm=None):
    """Grouping; with ``x`` also gathers x_perm[r] = x[row_token[r]]."""
    _check(lib().moe_permute(ctypes.byref(desc), _ptr(topk_idx), _ptr(x), _ptr(offsets), _ptr(row_token),
                             _ptr(inv), _ptr(x_perm), _stream(stream)), "moe_permute")


def moe_grouped_ffn(desc, routed: Weights, shared: Optional[Weights], offsets, row_token, x, y_perm, y_shared,
                    workspace, stream=None):
    _check(lib().moe_grouped_ffn(ctypes.byref(desc), ctypes.byref(routed),
                                 ctypes.byref(shared) if shared is not None else None, _ptr(offsets),
                                 _ptr(row_token), _ptr(x), _ptr(y_perm), _ptr(y_shared), _ptr(workspace),
                                 workspace.numel() * workspace.element_size(), _stream(stream)),
           "moe_grouped_ffn")


def moe_combine(desc, y_perm, inv, topk_w, y_shared, out, stream=None):
    _check(lib().moe_combine(ctypes.byref(desc), _ptr(y_perm), _ptr(inv), _ptr(topk_w), _ptr(y_shared), _ptr(out),
                             _stream(stream)), "moe_combine")


def moe_layer_forward(desc, x, w_router, logit_bias, routed: Weights, shared: Optional[Weights], out, workspace,
                      stream=None):
    _check(lib().moe_layer_forward(ctypes.byref(desc), _ptr(x), _ptr(w_router), _ptr(logit_bias),
                                   ctypes.byref(routed), ctypes.byref(shared) if shared is not None else None,
                                   _ptr(out), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                   _stream(stream)), "moe_layer_forward")


def moe_get_last_error() -> int:
    return lib().moe_get_last_error()


def moe_diag_wait_timeout(limit_ns: int, finished, stream=None):
    _check(lib().moe_diag_wait_timeout(int(limit_ns), _ptr(finished), _stream(stream)), "moe_diag_wait_timeout")


def moe_profile_enable(on: bool = True):
    _check(lib().moe_profile_enable(1 if on else 0), "moe_profile_enable")


def moe_profile_collect() -> dict:
    """{kernel name: (launches, total ms)} recorded since the last collect."""
    cap = 64
    arr = (ProfileEntry * cap)()
    n = ctypes.c_int32()
    _check(lib().moe_profile_collect(arr, cap, ctypes.byref(n)), "moe_profile_collect")
    return {arr[i].name.decode(): (arr[i].launches, arr[i].total_ms) for i in range(min(n.value, cap))}


class ExpertCache:
    """Owner of one ``moe_cache`` (per-layer LRU over HBM slots + pinned host bank)."""

    def __init__(self, n_layers: int, n_experts: int, slots_per_layer: int, expert_bytes: int, device: int = 0,
                 host_bank: Optional[int] = None):
        self.desc = CacheDesc(n_layers, n_experts, slots_per_layer, expert_bytes, host_bank, device)
        h = ctypes.c_void_p()
        _check(lib().moe_cache_init(ctypes.byref(h), ctypes.byref(self.desc)), "moe_cache_init")
        self.handle = h
        self.n_experts = n_experts

    def host_expert(self, layer: int, e: int) -> int:
        return lib().moe_cache_host_expert(self.handle, layer, e)

    def slot_base(self, layer: int) -> int:
        return lib().moe_cache_slot_base(self.handle, layer)

    @staticmethod
    def _ints(xs):
        xs = [int(v) for v in xs]
        return (ctypes.c_int32 * max(len(xs), 1))(*xs), len(xs)

    def prefetch(self, layer: int, experts):
        arr, n = self._ints(experts)
        _check(lib().moe_cache_prefetch(self.handle, layer, arr, n), "moe_cache_prefetch")

    def lookup(self, layer: int, experts, slot_map_dev, stream=None):
        """slot_map_dev may be None for a policy-only cache (device < 0)."""
        arr, n = self._ints(experts)
        st = _stream(stream) if self.desc.device >= 0 else None
        _check(lib().moe_cache_lookup(self.handle, layer, arr, n, _ptr(slot_map_dev), st), "moe_cache_lookup")

    def release(self, layer: int, stream=None):
        st = _stream(stream) if self.desc.device >= 0 else None
        _check(lib().moe_cache_release(self.handle, layer, st), "moe_cache_release")

    def slot_map(self, layer: int):
        out = (ctypes.c_int32 * self.n_experts)()
        _check(lib().moe_cache_slot_map(self.handle, layer, out), "moe_cache_slot_map")
        return list(out)

    def stats(self) -> dict:
        s = CacheStats()
        _check(lib().moe_cache_stats(self.handle, ctypes.byref(s)), "moe_cache_stats")
        return s.as_dict()

    def close(self):
        if self.handle:
            _check(lib().moe_cache_destroy(self.handle), "moe_cache_destroy")
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
