"""Python binding of the B200 MoE layer library (``libmoe_b200.so``).

Argument marshalling only: every function here passes device pointers,
sizes and the current CUDA stream to the C entry point of the same name and
raises ``MoeError`` on a non-OK status.  All arithmetic runs in the CUDA
kernels; there is no CPU or PyTorch fallback.  Importing this package on a
machine without the built library raises immediately.
"""
from __future__ import annotations

from ._native import (  # noqa: F401
    MoeError,
    LayerDesc,
    Weights,
    WorkspaceLayout,
    CacheDesc,
    CacheStats,
    WDTYPE,
    lib,
    lib_path,
    make_desc,
    make_weights,
    moe_workspace_size,
    moe_workspace_layout_of,
    moe_route_topk,
    moe_route_topk_noalloc,
    moe_permute,
    moe_grouped_ffn,
    moe_combine,
    moe_layer_forward,
    moe_status_string,
    moe_get_last_error,
    ExpertCache,
    router_sum_depth,
    moe_profile_enable,
    moe_profile_collect,
    moe_diag_wait_timeout,
)
