"""The allocation-free router/top-k entry point against the workspace one.

moe_route_topk_noalloc serves callers that cannot allocate device memory
(their host framework owns every allocation, or their device memory is fixed
at start-up): it keeps the logits scratch in a fixed device array inside the
library.  Its results must match moe_route_topk's on the same inputs, call
after call, since every call shares that array.  This file is collected last
so that a run stopping at the first failure has run every other test first.
"""
import numpy as np
import pytest
import torch

import expert_ffn_layer_route_b200 as moe
import moe_inputs as mi

pytestmark = pytest.mark.gpu

GATE_TOL = 1e-5  # the gate tolerance of the parity tests


def _inputs(shape, T, seed):
    x = mi.draw_tokens(T, shape.d_model, seed, "cuda")
    router = mi.draw_router(shape, seed, "cuda")
    bias = mi.zipf_offsets(shape.n_experts, shape.zipf_s, seed, "cuda") if shape.zipf_s else None
    return x, router, bias


def _both(shape, T, seed):
    desc = moe.make_desc(shape, T)
    x, router, bias = _inputs(shape, T, seed)
    ws = torch.empty(moe.moe_workspace_size(desc), dtype=torch.uint8, device="cuda")
    i_ref = torch.empty(T, shape.top_k, dtype=torch.int32, device="cuda")
    g_ref = torch.empty(T, shape.top_k, dtype=torch.float32, device="cuda")
    moe.moe_route_topk(desc, x, router, bias, i_ref, g_ref, ws)
    i_na = torch.full((T, shape.top_k), -7, dtype=torch.int32, device="cuda")
    g_na = torch.full((T, shape.top_k), -7.0, dtype=torch.float32, device="cuda")
    moe.moe_route_topk_noalloc(desc, x, router, bias, i_na, g_na)
    torch.cuda.synchronize()
    return i_ref, g_ref, i_na, g_na


def test_noalloc_matches_workspace_entry_point_on_consecutive_calls():
    # two calls in a row of different sizes, then the first again: the shared
    # scratch keeps the previous call's contents, which must not leak through
    for shape, T, seed in [(mi.GPTOSS, 64, 21), (mi.KIMI, 128, 22), (mi.GPTOSS, 64, 21), (mi.TINY, 16, 23)]:
        i_ref, g_ref, i_na, g_na = _both(shape, T, seed)
        assert torch.equal(i_na, i_ref), shape.name
        assert torch.allclose(g_na, g_ref, rtol=0, atol=GATE_TOL), shape.name
    assert moe.moe_get_last_error() == 0


def test_noalloc_at_its_size_limit_matches_both_references():
    """The largest call the scratch holds (T * n_experts = 261888 of 262144
    logits) twice in a row: indices bit-exact and gates within GATE_TOL of the
    workspace entry point, and the expert choice against the fp64 oracle."""
    from oracle import layer as OL
    shape = mi.KIMI
    T = 262144 // shape.n_experts
    for rep in range(2):
        i_ref, g_ref, i_na, g_na = _both(shape, T, 25)
        assert torch.equal(i_na, i_ref)
        assert torch.allclose(g_na, g_ref, rtol=0, atol=GATE_TOL)
    x, router, bias = _inputs(shape, T, 25)
    xs, wr, b = OL.to_f64(x.cpu()), OL.to_f64(router.cpu()), OL.to_f64(bias.cpu())
    logits = OL.router_logits(xs, wr, b)
    ridx, rg, margin = OL.topk_select(logits, shape.top_k)
    beta = OL.logit_error_bound(xs, wr, b, moe.router_sum_depth(shape.d_model))
    uniq = margin > 2 * beta
    assert np.array_equal(i_na.cpu().numpy()[uniq], ridx[uniq])
    g = g_na.cpu().double().numpy()
    assert np.all(np.abs(g[uniq] - rg[uniq]) <= GATE_TOL + 2 * rg[uniq] * beta[uniq, None])
    assert moe.moe_get_last_error() == 0


def test_noalloc_rejects_sizes_beyond_its_scratch():
    shape = mi.KIMI  # 384 experts
    T = 262144 // shape.n_experts + 1
    desc = moe.make_desc(shape, T)
    x, router, bias = _inputs(shape, 4, 24)
    idx = torch.empty(4, shape.top_k, dtype=torch.int32, device="cuda")
    gw = torch.empty(4, shape.top_k, dtype=torch.float32, device="cuda")
    with pytest.raises(moe.MoeError) as err:
        moe.moe_route_topk_noalloc(desc, x, router, bias, idx, gw)
    assert err.value.status == 8  # MOE_ERR_WORKSPACE, returned before any GPU work
