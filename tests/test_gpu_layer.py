"""GPU parity: the CUDA library (through its C ABI) against the fp64 oracle.

Shapes span several row tiles and K chunks with ragged tails (d, d_ff = 2880
leave 64-row and 64-column remainders), multiple activation passes (experts
with more than 32 rows), shared experts, every weight format, empty and
degenerate cases.  Full-size configurations are checked on sampled tokens.
"""
import numpy as np
import pytest
import torch

import moe_inputs as mi
import gpu_harness as H

pytestmark = pytest.mark.gpu


def _layer(shape, T, seed, device="cpu", **kw):
    """(layer for the oracle, the same layer on the GPU).  Full-size layers are
    drawn on the GPU; the oracle then reads the experts it needs from there."""
    hl = mi.draw_layer(shape, T, seed, device=device, **kw)
    return hl, H.to_device(hl)


CASES = [
    # name, shape, T
    ("tiny", mi.TINY, 16),
    ("mxfp4_gptoss_dims", mi.GPTOSS.replace(n_experts=16), 8),
    ("mxfp4_gptoss_dims_T1", mi.GPTOSS.replace(n_experts=16), 1),
    ("mxfp4_gptoss_dims_T3", mi.GPTOSS.replace(n_experts=16), 3),
    ("mxfp4_many_rows", mi.GPTOSS.replace(n_experts=4, top_k=2, d_model=576, d_ff=832), 150),
    ("int4_shared", mi.KIMI.replace(d_model=896, d_ff=384, n_experts=48), 40),
    ("int4_shared_T1", mi.KIMI.replace(d_model=896, d_ff=384, n_experts=48), 1),
    ("nvfp4_zipf", mi.BANK.replace(d_model=1024, d_ff=384, n_experts=32), 16),
    ("bf16_passes", mi.MIXTRAL.replace(d_model=512, d_ff=1024), 100),
    ("bf16_router_fp32_odd", mi.TINY.replace(d_model=320, d_ff=96, n_experts=7, top_k=3), 33),
]


@pytest.mark.parametrize("name,shape,T", CASES, ids=[c[0] for c in CASES])
@pytest.mark.parametrize("seed", [0, 1])
def test_layer_matches_oracle(name, shape, T, seed):
    hl, dl = _layer(shape, T, seed)
    res = H.run_layer(dl)
    rel, n_amb = H.full_check(hl, res)
    print(f"{name} seed={seed}: rel err {rel:.2e}, ambiguous tokens {n_amb}")


def test_int4_offset_decode_with_positive_activations():
    """The INT4 decode removes, per 128-wide scale group, a constant
    proportional to the group's activation sum.  All-positive activation rows
    make that constant largest relative to the result (no cancellation inside
    the sum), the hardest case for the fp32 accumulation."""
    shape = mi.KIMI.replace(d_model=896, d_ff=384, n_experts=48)
    hl = mi.draw_layer(shape, 24, 5)
    hl["x"] = (hl["x"].float().abs() + 1.0).to(hl["x"].dtype)
    rel, n_amb = H.full_check(hl, H.run_layer(H.to_device(hl)))
    print(f"int4 positive activations: rel err {rel:.2e}, ambiguous tokens {n_amb}")


@pytest.mark.parametrize("half", ["0", "1"])
def test_half_items_forced_in_both_stages(half, monkeypatch):
    """The streaming FFN's half-height items (64 + 64 rows in stage 1, 128 in
    stage 2; by default only stage 2 of small batches uses them) forced on and
    off for every format, against the oracle."""
    monkeypatch.setenv("MOE_FFN_HALF", half)
    for shape, T in [(mi.GPTOSS.replace(n_experts=16), 3),
                     (mi.KIMI.replace(d_model=896, d_ff=384, n_experts=48), 5),
                     (mi.BANK.replace(d_model=1024, d_ff=384, n_experts=32), 4),
                     (mi.TINY.replace(n_experts=16, top_k=2), 6)]:
        hl, dl = _layer(shape, T, 21)
        rel, n_amb = H.full_check(hl, H.run_layer(dl))
        print(f"half={half} {shape.name} T={T}: rel err {rel:.2e}, ambiguous {n_amb}")


FUSED_CASES = [
    # every token-tile width (1, 2, 4, 8) and activation-row format, fp32 and
    # bf16 routers, shared experts, 384 experts (a cluster of 16 CTAs where the
    # device can co-schedule it), 64 (token, slot) pairs, and 7 experts (CTAs
    # with no router slice)
    ("mxfp4_T1", mi.GPTOSS.replace(n_experts=16), 1),
    ("mxfp4_T3", mi.GPTOSS.replace(n_experts=16), 3),
    ("mxfp4_T8", mi.GPTOSS.replace(n_experts=16), 8),
    ("int4_shared_T2", mi.KIMI.replace(d_model=896, d_ff=384, n_experts=48), 2),
    ("int4_shared_T5", mi.KIMI.replace(d_model=896, d_ff=384, n_experts=48), 5),
    ("int4_E384_T1", mi.KIMI.replace(d_model=1024, d_ff=256, n_experts=384), 1),
    ("int4_E384_T8_64pairs", mi.KIMI.replace(d_model=1024, d_ff=256, n_experts=384), 8),
    ("nvfp4_T4", mi.BANK.replace(d_model=1024, d_ff=384, n_experts=32), 4),
    ("bf16_fp32router_T6", mi.TINY.replace(n_experts=16, top_k=2), 6),
    ("bf16_E7_T7", mi.TINY.replace(d_model=320, d_ff=96, n_experts=7, top_k=3), 7),
]


@pytest.mark.parametrize("name,shape,T", FUSED_CASES, ids=[c[0] for c in FUSED_CASES])
def test_fused_small_batch_routing_matches_unfused(name, shape, T, monkeypatch):
    """The one-launch routing kernel for small batches (router, top-k,
    permutation, activation rows) forced on and off: the same router tile,
    top-k and row-prep routines give bit-identical routing, permutation and
    layer output, and the fused run matches the oracle."""
    hl, dl = _layer(shape, T, 31)
    monkeypatch.setenv("MOE_FUSED_ROUTE", "1")
    a = H.run_layer(dl)
    rel, n_amb = H.full_check(hl, a)
    monkeypatch.setenv("MOE_FUSED_ROUTE", "0")
    b = H.run_layer(dl)
    for key in ("out", "idx", "gates", "offsets", "row_token", "inv"):
        assert torch.equal(a[key], b[key]), key
    print(f"fused {name}: rel err {rel:.2e}, ambiguous {n_amb}")


@pytest.mark.parametrize("split", ["1", "2", "3", "4"])
def test_split_k_forced(split, monkeypatch):
    """The streaming FFN's split-K items (each item's K chunks in S slices,
    the slice partials summed by the last-arriving warp; by default used when
    a batch of at most 8 tokens would leave most block slots idle) forced to
    1-4 slices for every format, against the oracle, and bit-identical on a
    second run (the slice sums are taken in slice order whichever warp
    arrives last)."""
    monkeypatch.setenv("MOE_FFN_SPLIT", split)
    for shape, T in [(mi.GPTOSS.replace(n_experts=16), 1),
                     (mi.GPTOSS.replace(n_experts=16), 7),
                     (mi.KIMI.replace(d_model=2048, d_ff=384, n_experts=48), 2),
                     (mi.BANK.replace(d_model=1024, d_ff=512, n_experts=32), 4),
                     (mi.TINY.replace(d_model=512, d_ff=640, n_experts=16, top_k=2), 3)]:
        hl, dl = _layer(shape, T, 23)
        a = H.run_layer(dl)
        rel, n_amb = H.full_check(hl, a)
        out = a["out"].clone()
        assert torch.equal(H.run_layer(dl)["out"], out)
        print(f"split={split} {shape.name} T={T}: rel err {rel:.2e}, ambiguous {n_amb}")


@pytest.mark.parametrize("seed", [2])
def test_tiny_seed2(seed):
    hl, dl = _layer(mi.TINY, 16, seed)
    H.full_check(hl, H.run_layer(dl))


def test_stepwise_entry_points_equal_layer_forward():
    for shape, T in [(mi.KIMI.replace(d_model=896, d_ff=384, n_experts=48), 12),
                     (mi.GPTOSS.replace(n_experts=16), 5), (mi.TINY, 16)]:
        hl, dl = _layer(shape, T, 3)
        a = H.run_layer(dl)
        b = H.run_steps(dl)
        for key in ("out", "idx", "gates", "offsets", "row_token", "inv"):
            assert torch.equal(a[key], b[key]), key


@pytest.mark.parametrize("shape,T", [(mi.GPTOSS.replace(n_experts=32), 24),
                                     (mi.GPTOSS.replace(n_experts=16), 1),
                                     (mi.KIMI.replace(d_model=896, d_ff=384, n_experts=48), 2)],
                         ids=["mxfp4_T24", "mxfp4_T1", "int4_T2"])
def test_deterministic_across_runs(shape, T):
    """Bit-identical outputs run to run, from single-token batches up."""
    hl, dl = _layer(shape, T, 4)
    a = H.run_layer(dl)["out"].clone()
    for _ in range(3):
        assert torch.equal(a, H.run_layer(dl)["out"])


def test_empty_batch_is_noop():
    hl, dl = _layer(mi.TINY, 0, 0)
    res = H.run_layer(dl)
    assert res["out"].shape == (0, 256)


def test_single_expert_dense_mlp():
    shape = mi.TINY.replace(n_experts=1, top_k=1, router_fp32=False)
    hl, dl = _layer(shape, 9, 5)
    H.full_check(hl, H.run_layer(dl))


def test_k_equals_E_with_zero_router_is_uniform_average():
    shape = mi.GPTOSS.replace(n_experts=4, top_k=4, d_model=256, d_ff=256)
    hl, dl = _layer(shape, 6, 6)
    hl["router"] = torch.zeros_like(hl["router"])
    dl["router"] = hl["router"].cuda()
    res = H.run_layer(dl)
    assert torch.allclose(res["gates"], torch.full_like(res["gates"], 0.25), atol=0, rtol=0)
    assert res["idx"].cpu().tolist() == [[0, 1, 2, 3]] * 6  # ties: lower index first
    H.full_check(hl, res)


def test_identical_router_rows_tie_to_lower_index():
    shape = mi.GPTOSS.replace(n_experts=8, top_k=2, d_model=256, d_ff=256)
    hl, dl = _layer(shape, 20, 7)
    r = hl["router"].clone()
    r[5] = r[2]  # experts 2 and 5 always tie exactly
    r[6] = r[1]
    hl["router"] = r
    dl["router"] = r.cuda()
    res = H.run_layer(dl)
    idx = res["idx"].cpu().numpy()
    assert not np.any((idx == 5).any(1) & ~(idx == 2).any(1))  # 5 only ever chosen together with 2
    H.full_check(hl, res)


def test_identical_experts_reduce_to_one_ffn():
    shape = mi.BANK.replace(d_model=512, d_ff=256, n_experts=16)
    hl, dl = _layer(shape, 11, 8, identical_experts=True)
    H.full_check(hl, H.run_layer(dl))


def test_out_of_range_expert_index_sets_status():
    import expert_ffn_layer_route_b200 as moe
    moe.moe_get_last_error()
    shape = mi.TINY
    desc = moe.make_desc(shape, 4)
    idx = torch.tensor([[0, 1], [2, 99], [3, 4], [5, 6]], dtype=torch.int32, device="cuda")
    offs = torch.empty(shape.n_experts + 1, dtype=torch.int32, device="cuda")
    rtok = torch.empty(8, dtype=torch.int32, device="cuda")
    inv = torch.empty(8, dtype=torch.int32, device="cuda")
    x = mi.draw_tokens(4, shape.d_model, 3, "cuda")
    xp = torch.full((8, shape.d_model), 7.0, dtype=torch.bfloat16, device="cuda")
    moe.moe_permute(desc, idx, offs, rtok, inv, x=x, x_perm=xp)
    assert moe.moe_get_last_error() == 9
    assert inv.cpu().tolist()[3] == -1
    assert offs.cpu().tolist()[-1] == 7
    assert moe.moe_get_last_error() == 0  # cleared
    # the seven grouped rows are gathered; the dropped pair's row has no source and is zero
    assert torch.equal(xp[:7], x[rtok[:7].long()])


@pytest.mark.parametrize("shape,T", [(mi.GPTOSS.replace(n_experts=16), 13), (mi.KIMI, 40), (mi.TINY, 0)],
                         ids=["mxfp4_E16_T13", "kimi_T40", "empty"])
def test_permute_gathers_rows_in_expert_order(shape, T):
    """moe_permute with x: offsets / row_token / inv bit-exact against the
    oracle's stable counting sort, and x_perm[r] = x[row_token[r]] bit for bit."""
    import expert_ffn_layer_route_b200 as moe
    from oracle import layer as OL
    desc = moe.make_desc(shape, T)
    k, E = shape.top_k, shape.n_experts
    gen = torch.Generator().manual_seed(T + 5)
    idx = torch.stack([torch.randperm(E, generator=gen)[:k] for _ in range(T)]).to(torch.int32) if T else \
        torch.zeros(0, k, dtype=torch.int32)
    x = mi.draw_tokens(T, shape.d_model, 9, "cuda")
    offs = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    rtok = torch.empty(max(T * k, 1), dtype=torch.int32, device="cuda")
    inv = torch.empty(max(T * k, 1), dtype=torch.int32, device="cuda")
    xp = torch.empty(max(T * k, 1), shape.d_model, dtype=torch.bfloat16, device="cuda")
    moe.moe_permute(desc, idx.cuda(), offs, rtok, inv, x=x, x_perm=xp)
    torch.cuda.synchronize()
    assert moe.moe_get_last_error() == 0
    c, o, rt, iv = OL.permute(idx.numpy(), E)
    assert np.array_equal(offs.cpu().numpy(), o)
    if T == 0:
        return
    assert np.array_equal(rtok.cpu().numpy(), rt)
    assert np.array_equal(inv.cpu().numpy(), iv)
    assert torch.equal(xp.cpu(), x.cpu()[torch.from_numpy(rt).long()])


# ------------------------------------------------------------ full sizes ----

@pytest.mark.parametrize("shape,T", [(mi.GPTOSS, 64), (mi.GPTOSS, 1), (mi.KIMI, 128), (mi.BANK, 16),
                                     (mi.MIXTRAL, 4096)])
def test_full_size_routing_exact(shape, T):
    """Router + top-k + permutation at the measured sizes, every token."""
    import expert_ffn_layer_route_b200 as moe
    from oracle import layer as OL
    gen_dev = "cuda"
    x = mi.draw_tokens(T, shape.d_model, 11, gen_dev)
    router = mi.draw_router(shape, 11, gen_dev)
    bias = mi.zipf_offsets(shape.n_experts, shape.zipf_s, 11, gen_dev) if shape.zipf_s else None
    desc = moe.make_desc(shape, T)
    ws = torch.empty(moe.moe_workspace_size(desc), dtype=torch.uint8, device="cuda")
    idx = torch.empty(T, shape.top_k, dtype=torch.int32, device="cuda")
    gw = torch.empty(T, shape.top_k, dtype=torch.float32, device="cuda")
    moe.moe_route_topk(desc, x, router, bias, idx, gw, ws)
    offs = torch.empty(shape.n_experts + 1, dtype=torch.int32, device="cuda")
    rtok = torch.empty(T * shape.top_k, dtype=torch.int32, device="cuda")
    inv = torch.empty(T * shape.top_k, dtype=torch.int32, device="cuda")
    moe.moe_permute(desc, idx, offs, rtok, inv)
    torch.cuda.synchronize()
    hl = {"shape": shape, "x": x.cpu(), "router": router.cpu(), "bias": bias.cpu() if bias is not None else None}
    xs, wr = OL.to_f64(hl["x"]), OL.to_f64(hl["router"])
    b = OL.to_f64(hl["bias"]) if bias is not None else None
    logits = OL.router_logits(xs, wr, b)
    ridx, rg, margin = OL.topk_select(logits, shape.top_k)
    beta = OL.logit_error_bound(xs, wr, b, moe.router_sum_depth(shape.d_model))
    uniq = margin > 2 * beta
    g_idx = idx.cpu().numpy()
    assert np.array_equal(g_idx[uniq], ridx[uniq])
    print(f"{shape.name} T={T}: ambiguous tokens {int((~uniq).sum())}")
    c, o, rt, iv = OL.permute(g_idx, shape.n_experts)
    assert np.array_equal(offs.cpu().numpy(), o)
    assert np.array_equal(rtok.cpu().numpy(), rt)
    assert np.array_equal(inv.cpu().numpy(), iv)
    g = gw.cpu().double().numpy()
    assert np.all(np.abs(g[uniq] - rg[uniq]) <= 1e-5 + 2 * rg[uniq] * beta[uniq, None])


FULL_VALUE_CASES = [
    # shape, T, tokens compared (None: every token; n: a seeded subset of n)
    (mi.GPTOSS, 1, None), (mi.GPTOSS, 8, None), (mi.GPTOSS, 32, None), (mi.GPTOSS, 64, None),
    (mi.KIMI, 1, None), (mi.KIMI, 8, None), (mi.KIMI, 32, None), (mi.KIMI, 128, 64),
    (mi.BANK, 16, None),
]


def _tile_covering_subset(res, T, k, n, seed):
    """n tokens: one whose row lies in each 128-row m-tile of each expert's
    group (so that every tile the tensor-core kernel runs is checked), the rest
    a seeded random choice."""
    row_of = res["inv"].cpu().numpy().reshape(T, k)
    offs = res["offsets"].cpu().numpy()
    first = {}
    for t in range(T):
        for r in row_of[t]:
            e = int(np.searchsorted(offs, r, side="right") - 1)
            first.setdefault((e, (int(r) - int(offs[e])) // 128), t)
    tiles = {(e, m) for e in range(len(offs) - 1) for m in range((int(offs[e + 1] - offs[e]) + 127) // 128)}
    assert set(first) == tiles
    chosen = set(first.values())
    rest = [t for t in np.random.default_rng(seed).permutation(T).tolist() if t not in chosen]
    return sorted(chosen | set(rest[: max(0, n - len(chosen))]))


def _token_subset(T, n, seed):
    if n is None or n >= T:
        return None
    return sorted(np.random.default_rng(seed).choice(T, n, replace=False).tolist())


@pytest.mark.parametrize("shape,T,n_tok", FULL_VALUE_CASES,
                         ids=[f"{c[0].name}_T{c[1]}" for c in FULL_VALUE_CASES])
def test_full_size_layer_values(shape, T, n_tok):
    """Whole layer at the measured sizes, in the launch configurations the
    benchmark times (column groups per pass, blocks per SM, half-height items
    and dynamic item claiming all follow T): routing bit-exact on every token,
    outputs against the oracle on every token (a seeded subset of 64 at
    Kimi T=128)."""
    hl, dl = _layer(shape, T, 12, device="cuda")
    res = H.run_layer(dl)
    tokens = _token_subset(T, n_tok, T)
    ref, n_amb = H.check_routing(hl, res["idx"], res["gates"], tokens=tokens)
    H.check_permutation(res, shape)
    rel = H.check_output(res["out"], ref["out"], tokens=tokens)
    n = T if tokens is None else len(tokens)
    print(f"{shape.name} T={T}: rel err {rel:.2e} on {n} tokens, ambiguous {n_amb}")


@pytest.mark.parametrize("n_seq,depth", [(16, 3), (4, 2), (1, 4)])
def test_verification_block_values_and_expert_union(n_seq, depth):
    """A speculative verification block (n_seq sequences x (1 + depth)
    correlated positions in one call) on the full-size gpt-oss layer: every
    position against the oracle, and the experts the call reads (from the
    GPU's offsets) equal to the union of the positions' oracle choices."""
    from oracle import cost as OC
    shape = mi.GPTOSS
    T = n_seq * (depth + 1)
    hl, dl = _layer(shape, T, 14, device="cuda")
    x = mi.draw_verify_tokens(n_seq, depth, shape.d_model, 0.5, 15, "cuda")
    hl["x"], dl["x"] = x, x
    res = H.run_layer(dl)
    ref, n_amb = H.check_routing(hl, res["idx"], res["gates"])
    H.check_permutation(res, shape)
    rel = H.check_output(res["out"], ref["out"])
    offs = res["offsets"].cpu().numpy()
    assert int((np.diff(offs) > 0).sum()) == OC.expert_union(ref["idx"])
    print(f"verify n_seq={n_seq} depth={depth}: rel err {rel:.2e}, union {OC.expert_union(ref['idx'])} experts, "
          f"ambiguous {n_amb}")


# --------------------------------------------------- tensor-core GEMM path ----

GEMM_CASES = [
    ("bf16_gemm_ragged", mi.MIXTRAL.replace(d_model=512, d_ff=1024, n_experts=4), 300),
    ("bf16_gemm_shared", mi.MIXTRAL.replace(d_model=512, d_ff=512, n_experts=8, n_shared=1), 200),
    ("bf16_gemm_many_tiles", mi.MIXTRAL.replace(d_model=1024, d_ff=1536, n_experts=8), 1000),
]


@pytest.mark.parametrize("name,shape,T", GEMM_CASES, ids=[c[0] for c in GEMM_CASES])
def test_gemm_path_matches_oracle_and_stream_path(name, shape, T, monkeypatch):
    hl, dl = _layer(shape, T, 31)
    monkeypatch.setenv("MOE_FFN_PATH", "gemm")
    res = H.run_layer(dl)
    rel, n_amb = H.full_check(hl, res)
    monkeypatch.setenv("MOE_FFN_PATH", "stream")
    res_s = H.run_layer(dl)
    o1, o2 = res["out"].float(), res_s["out"].float()
    # both are fp32-accumulated roundings of the same sums
    assert (o1 - o2).abs().max().item() <= 1e-2 * o2.abs().max().item()
    import expert_ffn_layer_route_b200 as moe
    assert moe.moe_get_last_error() == 0
    print(f"{name}: rel err {rel:.2e}, ambiguous {n_amb}")


def test_gemm_path_full_size_prefill_sampled():
    """Mixtral-shaped prefill (T=4096) through the default path (tensor-core
    GEMM): routing and permutation bit-exact on every token, outputs against
    the oracle on a seeded subset of 512 tokens (which touches every m-tile of
    every expert)."""
    hl, dl = _layer(mi.MIXTRAL, 4096, 12, device="cuda")
    res = H.run_layer(dl)
    ref_all, n_amb_all = H.check_routing(hl, res["idx"], res["gates"], tokens=None, values=False)
    H.check_permutation(res, mi.MIXTRAL)
    tokens = _tile_covering_subset(res, 4096, 2, 512, 4096)
    ref, n_amb = H.check_routing(hl, res["idx"], res["gates"], tokens=tokens)
    rel = H.check_output(res["out"], ref["out"], tokens=tokens)
    print(f"mixtral T=4096: rel err {rel:.2e} on {len(tokens)} tokens, ambiguous {n_amb_all} of 4096")


# ------------------------------------------ 4-bit tensor-core GEMM path ----

Q4_GEMM_CASES = [
    # 4-bit layers with prefill-sized expert groups; K multiples of 512 (MXFP4),
    # 256 (NVFP4), 1024 (INT4); ragged groups (second 128-row half partly or
    # not at all filled), shared expert, several weight tiles and K steps
    ("mxfp4_gemm_ragged", mi.GPTOSS.replace(d_model=1024, d_ff=1536, n_experts=4, top_k=2), 300),
    ("mxfp4_gemm_small_groups", mi.GPTOSS.replace(d_model=512, d_ff=512, n_experts=8, top_k=2), 290),
    ("nvfp4_gemm", mi.BANK.replace(d_model=512, d_ff=768, n_experts=6, top_k=2), 400),
    ("int4_gemm_shared", mi.KIMI.replace(d_model=1024, d_ff=1024, n_experts=8, top_k=2), 260),
    ("mxfp4_gemm_shared", mi.GPTOSS.replace(d_model=512, d_ff=1024, n_experts=6, top_k=2, n_shared=1), 200),
    ("nvfp4_gemm_shared_zipf", mi.BANK.replace(d_model=768, d_ff=512, n_experts=10, top_k=3, n_shared=2), 230),
]


@pytest.mark.parametrize("name,shape,T", Q4_GEMM_CASES, ids=[c[0] for c in Q4_GEMM_CASES])
def test_q4_gemm_path_matches_oracle_and_stream_path(name, shape, T, monkeypatch):
    """4-bit experts through the tensor-core GEMM (weights decoded once per
    tile to 16-bit values in shared memory) against the fp64 oracle, and
    against the streaming path on the same inputs."""
    import expert_ffn_layer_route_b200 as moe
    hl, dl = _layer(shape, T, 33)
    monkeypatch.setenv("MOE_FFN_PATH", "gemm")
    moe.moe_profile_enable(True)
    moe.moe_profile_collect()
    res = H.run_layer(dl)
    prof = moe.moe_profile_collect()
    moe.moe_profile_enable(False)
    assert "ffn_gemm_q4_stage1_gate_up" in prof and "ffn_gemm_q4_stage2_down" in prof, sorted(prof)
    rel, n_amb = H.full_check(hl, res)
    monkeypatch.setenv("MOE_FFN_PATH", "stream")
    res_s = H.run_layer(dl)
    o1, o2 = res["out"].float(), res_s["out"].float()
    assert (o1 - o2).abs().max().item() <= 1e-2 * o2.abs().max().item()
    assert moe.moe_get_last_error() == 0
    print(f"{name}: rel err {rel:.2e}, ambiguous {n_amb}")


def test_q4_gemm_is_default_for_prefill_sized_groups():
    """Without an override a 4-bit batch averaging >= 64 rows per expert takes
    the tensor-core path; a decode-sized batch keeps the streaming kernel."""
    import expert_ffn_layer_route_b200 as moe
    shape = mi.GPTOSS.replace(d_model=512, d_ff=512, n_experts=4, top_k=2)
    for T, want in [(256, "ffn_gemm_q4_stage1_gate_up"), (8, "ffn_stage1_gate_up")]:
        hl, dl = _layer(shape, T, 34)
        moe.moe_profile_enable(True)
        moe.moe_profile_collect()
        res = H.run_layer(dl)
        prof = moe.moe_profile_collect()
        moe.moe_profile_enable(False)
        assert want in prof, (T, sorted(prof))
        H.full_check(hl, res)


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4", "int4"])
def test_q4_gemm_through_a_slot_map(fmt, monkeypatch):
    """The 4-bit tensor-core path addressing experts through a slot map (the
    expert cache's placement): experts stored in a permuted order give
    bit-identical outputs to the identity placement; an expert marked
    non-resident (-1) is skipped and its rows are left as they were."""
    import expert_ffn_layer_route_b200 as moe
    monkeypatch.setenv("MOE_FFN_PATH", "gemm")
    shape = mi.BANK.replace(d_model=1024, d_ff=1024, n_experts=6, top_k=2, wdtype=fmt, zipf_s=0.0)
    T = 160
    hl, dl = _layer(shape, T, 35)
    ref = H.run_steps(dl)
    perm = torch.tensor([3, 0, 5, 1, 4, 2], dtype=torch.int32)  # logical e -> physical slot perm[e]
    phys = {}
    for key, v in dl["experts"].items():
        if key in ("g13", "g2"):
            phys[key] = v  # global scales are indexed by the logical expert
            continue
        t = torch.empty_like(v)
        t[perm.long().cuda()] = v
        phys[key] = t
    desc = moe.make_desc(shape, T)
    ws = torch.empty(moe.moe_workspace_size(desc), dtype=torch.uint8, device="cuda")
    for missing in (None, 4):
        smap = perm.clone()
        if missing is not None:
            smap[missing] = -1
        smap_d = smap.cuda()  # kept alive until the kernel has run
        w = moe.make_weights(phys, slot_map=smap_d, n_physical=6)
        y = torch.full_like(ref["y"], 3.0)
        moe.moe_grouped_ffn(desc, w, None, ref["offsets"], ref["row_token"], dl["x"], y, None, ws)
        torch.cuda.synchronize()
        assert moe.moe_get_last_error() == 0
        if missing is None:
            assert torch.equal(y, ref["y"])
        else:
            offs = ref["offsets"].cpu().tolist()
            lo, hi = offs[missing], offs[missing + 1]
            keep = torch.ones(y.shape[0], dtype=torch.bool)
            keep[lo:hi] = False
            assert torch.equal(y[keep.cuda()], ref["y"][keep.cuda()])
            assert bool((y[lo:hi] == 3.0).all())


def test_q4_gemm_full_size_mixtral_mxfp4_prefill_sampled():
    """Mixtral-shaped prefill (T=4096) with MXFP4 experts on the tensor-core
    path: routing bit-exact on every token, outputs against the oracle on a
    seeded subset of 512 tokens."""
    hl, dl = _layer(mi.MIXTRAL_MXFP4, 4096, 13, device="cuda")
    res = H.run_layer(dl)
    H.check_routing(hl, res["idx"], res["gates"], tokens=None, values=False)
    H.check_permutation(res, mi.MIXTRAL_MXFP4)
    tokens = _tile_covering_subset(res, 4096, 2, 512, 4097)
    ref, n_amb = H.check_routing(hl, res["idx"], res["gates"], tokens=tokens)
    rel = H.check_output(res["out"], ref["out"], tokens=tokens)
    print(f"mixtral mxfp4 T=4096: rel err {rel:.2e} on {len(tokens)} tokens, ambiguous {n_amb}")


def test_bounded_wait_times_out_with_status_and_context_survives():
    """A pipeline wait that can never be satisfied gives up after its limit,
    reports MOE_ERR_TIMEOUT, and the GPU keeps working afterwards."""
    import time
    import expert_ffn_layer_route_b200 as moe
    moe.moe_get_last_error()
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    t0 = time.perf_counter()
    moe.moe_diag_wait_timeout(50_000_000, flag)  # 50 ms
    assert moe.moe_get_last_error() == 6  # MOE_ERR_TIMEOUT (synchronises)
    assert time.perf_counter() - t0 < 5.0
    assert flag.item() == 1
    hl, dl = _layer(mi.TINY, 16, 0)
    H.full_check(hl, H.run_layer(dl))  # the context is still usable
