"""Pins for the oracle's layer arithmetic (CPU only).

The oracle is checked against closed forms, brute force and library routines
that share nothing with it:

* a hand-worked 3-expert layer whose output is a closed form in e;
* top-k against brute force over every k-subset (with ties);
* gates against scipy's softmax over the selected logits, for the top-k and
  for forced selections (any subset, any order), plus a forced selection of the
  worked layer in closed form;
* the permutation against numpy's stable argsort;
* k = E with a zero router, E = 1, identical experts and a shared expert
  against a dense SwiGLU MLP written with torch.nn.functional in float64;
* the fp32 logit error bound against float32 evaluations in several orders.

The planted-mistake tests at the end show that each pin rejects a plausible
slip in the oracle (gate/up swapped, renormalisation dropped, tie rule
reversed, wrong permutation order, shared expert dropped; for forced
selections: renormalisation dropped, the wrong token's logits, sorted instead
of the given order, the selection or its gates ignored).
"""
import itertools
import math

import numpy as np
import pytest
import scipy.special
import torch
import torch.nn.functional as TF

import moe_inputs as mi
from oracle import layer as L
from oracle import formats as F


def _bf16(a):
    return torch.tensor(a, dtype=torch.float32).to(torch.bfloat16)


def _tiny_layer():
    """d=2, E=3, k=2, d_ff=1; every value exact in bf16."""
    shape = mi.LayerShape("worked", 2, 3, 2, 1, "bf16")
    w13 = [[[0, 0], [0, 0]],      # expert 0: gate, up
           [[1, 0], [0, 1]],      # expert 1
           [[0, 1], [1, 1]]]      # expert 2
    w2 = [[[0], [0]], [[1], [-1]], [[2], [0]]]
    return {"shape": shape, "x": _bf16([[1.0, 2.0]]), "router": _bf16([[1, 0], [0, 1], [1, 1]]),
            "bias": None, "experts": {"w13": _bf16(w13), "w2": _bf16(w2)}, "shared": None}


def test_worked_example_closed_form():
    # logits = [1, 2, 3] -> experts (2, 1); gates = softmax(3, 2)
    g2 = 1.0 / (1.0 + math.exp(-1.0))
    g1 = 1.0 - g2
    # expert 1: a = 1, b = 2 -> h = 2 silu(1); y = (h, -h)
    h1 = 2.0 * (1.0 / (1.0 + math.exp(-1.0)))
    # expert 2: a = 2, b = 3 -> h = 3 silu(2); y = (2h, 0)
    h2 = 3.0 * (2.0 / (1.0 + math.exp(-2.0)))
    expect = np.array([[g2 * 2.0 * h2 + g1 * h1, -g1 * h1]])
    r = L.moe_layer(_tiny_layer())
    assert r["idx"].tolist() == [[2, 1]]
    assert np.allclose(r["gates"], [[g2, g1]], rtol=0, atol=1e-15)
    assert np.allclose(r["out"], expect, rtol=1e-14, atol=0)
    assert r["counts"].tolist() == [0, 1, 1]
    assert r["offsets"].tolist() == [0, 0, 1, 2]
    assert r["inv"].tolist() == [1, 0]  # pair (t0, slot0) is expert 2 -> row 1


# ---------------------------------------------------------------- top-k ----

def brute_force_topk(lt, k):
    """The unique k-subset S with every member beating every non-member
    (larger logit, or equal logit and lower index), ordered the same way."""
    E = len(lt)
    beats = lambda i, j: lt[i] > lt[j] or (lt[i] == lt[j] and i < j)
    found = []
    for S in itertools.combinations(range(E), k):
        rest = [j for j in range(E) if j not in S]
        if all(beats(i, j) for i in S for j in rest):
            found.append(S)
    assert len(found) == 1
    S = list(found[0])
    # order inside the set: insertion sort with the same relation
    for a in range(len(S)):
        for b in range(a + 1, len(S)):
            if beats(S[b], S[a]):
                S[a], S[b] = S[b], S[a]
    return S


def pin_topk(topk_fn):
    rng = np.random.default_rng(5)
    for trial in range(300):
        E = int(rng.integers(1, 9))
        k = int(rng.integers(1, E + 1))
        lt = rng.integers(-3, 4, size=E).astype(np.float64)  # many ties
        idx, gates, margin = topk_fn(lt[None, :], k)
        if idx[0].tolist() != brute_force_topk(lt, k):
            return False
        ref = scipy.special.softmax(lt[idx[0]])
        if not np.allclose(gates[0], ref, rtol=1e-13, atol=1e-15):
            return False
        if abs(gates[0].sum() - 1.0) > 1e-12:
            return False
    return True


def test_topk_matches_brute_force_and_softmax():
    assert pin_topk(L.topk_select)


def pin_gates_for(gates_fn):
    """Gates of a given (forced) selection: the softmax of the selected logits
    (scipy), in the selection's own order, for selections that are not the
    top-k (any k-subset, any order, ties included), on logits large enough
    that a missing max-shift would overflow."""
    rng = np.random.default_rng(11)
    for trial in range(200):
        T = int(rng.integers(1, 6))
        E = int(rng.integers(1, 9))
        k = int(rng.integers(1, E + 1))
        logits = rng.integers(-3, 4, size=(T, E)).astype(np.float64)
        if trial % 3 == 0:
            logits = logits * 300.0  # exp overflows without the shift
        idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
        g = gates_fn(logits, idx)
        for t in range(T):
            ref = scipy.special.softmax(logits[t, idx[t]])
            if not np.allclose(g[t], ref, rtol=1e-13, atol=1e-15):
                return False
            if abs(g[t].sum() - 1.0) > 1e-12:
                return False
    return True


def test_gates_for_forced_selection_matches_softmax():
    assert pin_gates_for(L.gates_for)


def pin_forced_worked_example(layer_fn):
    """The worked 3-expert layer with its selection forced to (2, 0), which is
    not the top-2 (that is (2, 1)): gates = softmax(l2, l0) = softmax(3, 1) in
    that order; expert 0 has zero weights, so out = g2 * y2 with
    y2 = (2 h2, 0), h2 = 3 silu(2)."""
    g2 = 1.0 / (1.0 + math.exp(-2.0))
    h2 = 3.0 * (2.0 / (1.0 + math.exp(-2.0)))
    r = layer_fn(_tiny_layer(), forced_idx=np.array([[2, 0]], np.int32))
    return (r["idx"].tolist() == [[2, 0]] and np.allclose(r["gates"], [[g2, 1.0 - g2]], rtol=0, atol=1e-15)
            and np.allclose(r["out"], [[g2 * 2.0 * h2, 0.0]], rtol=1e-14, atol=1e-15)
            and r["inv"].tolist() == [1, 0] and r["counts"].tolist() == [1, 0, 1])


def test_forced_selection_worked_example_closed_form():
    assert pin_forced_worked_example(L.moe_layer)


def test_forced_selection_token_subset():
    """Forced routing with a token subset takes each listed token's own row."""
    lay = _small("mxfp4", E=8, k=2, d=64, f=64, T=9)
    rng = np.random.default_rng(3)
    forced = np.stack([rng.permutation(8)[:2] for _ in range(9)]).astype(np.int32)
    full = L.moe_layer(lay, forced_idx=forced)
    sub = L.moe_layer(lay, forced_idx=forced, tokens=[7, 2, 4])
    assert np.array_equal(sub["idx"], forced[[7, 2, 4]])
    assert np.allclose(sub["gates"], full["gates"][[7, 2, 4]], rtol=1e-15, atol=0)
    assert np.allclose(sub["out"], full["out"][[7, 2, 4]], rtol=1e-13, atol=1e-13 * np.abs(full["out"]).max())


def test_margin_definition():
    lt = np.array([[0.5, 3.0, 2.0, 2.5]])
    _, _, m = L.topk_select(lt, 2)
    assert m[0] == 2.5 - 2.0
    _, _, m = L.topk_select(lt, 4)
    assert m[0] == np.inf


# ----------------------------------------------------------- permutation ----

def pin_permute(perm_fn):
    rng = np.random.default_rng(7)
    for trial in range(50):
        E = int(rng.integers(1, 40))
        k = int(rng.integers(1, min(E, 8) + 1))
        T = int(rng.integers(0, 60))
        idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]) if T else np.zeros((0, k), np.int32)
        counts, offsets, row_token, inv = perm_fn(idx.astype(np.int32), E)
        flat = idx.reshape(-1)
        order = np.argsort(flat, kind="stable")  # library stable sort
        if not np.array_equal(row_token, order // k):
            return False
        ref_inv = np.empty_like(order)
        ref_inv[order] = np.arange(order.size)
        if not np.array_equal(inv, ref_inv):
            return False
        if not np.array_equal(counts, np.bincount(flat, minlength=E)):
            return False
        if not (offsets[0] == 0 and np.array_equal(np.diff(offsets), counts)):
            return False
    return True


def test_permute_matches_stable_sort():
    assert pin_permute(L.permute)


# ------------------------------------------------------------------ FFN ----

def torch_dense_swiglu(x, w13, w2):
    """Dense SwiGLU MLP from torch.nn.functional, float64."""
    x = torch.from_numpy(np.asarray(x, np.float64))
    w13 = torch.from_numpy(np.asarray(w13, np.float64))
    w2 = torch.from_numpy(np.asarray(w2, np.float64))
    f = w13.shape[0] // 2
    h = TF.silu(TF.linear(x, w13[:f])) * TF.linear(x, w13[f:])
    return TF.linear(h, w2).numpy()


def _small(wdtype, E=4, k=2, d=64, f=96, n_shared=0, T=5, seed=0, **kw):
    shape = mi.LayerShape("t", d, E, k, f, wdtype, n_shared=n_shared, **kw)
    return mi.draw_layer(shape, T, seed)


def pin_dense_single_expert(layer_fn=None, wdtype="bf16"):
    """E = 1, k = 1: the layer is a plain dense SwiGLU MLP."""
    layer_fn = layer_fn or L.moe_layer
    f = 128 if wdtype == "int4" else 96
    lay = _small(wdtype, E=1, k=1, d=128, f=f, T=6)
    w13, w2 = F.dequant_expert(wdtype, lay["experts"], 0)
    ref = torch_dense_swiglu(L.to_f64(lay["x"]), w13, w2)
    return np.allclose(layer_fn(lay)["out"], ref, rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("wdtype", ["bf16", "mxfp4", "nvfp4", "int4"])
def test_single_expert_is_dense_mlp(wdtype):
    assert pin_dense_single_expert(L.moe_layer, wdtype)


def pin_uniform_average(layer_fn):
    """k = E with a zero router: uniform gates 1/E; out = mean over all experts."""
    lay = _small("bf16", E=4, k=4, d=64, f=96, T=5)
    lay["router"] = torch.zeros_like(lay["router"])
    ref = np.mean([torch_dense_swiglu(L.to_f64(lay["x"]), *F.dequant_expert("bf16", lay["experts"], e))
                   for e in range(4)], axis=0)
    r = layer_fn(lay)
    return np.allclose(r["out"], ref, rtol=1e-12, atol=1e-14) and np.allclose(r["gates"], 0.25)


def test_k_equals_E_uniform_average():
    assert pin_uniform_average(L.moe_layer)


def pin_identical_experts(layer_fn):
    """Identical experts: out = FFN(x) whatever the routing (gates sum to 1)."""
    shape = mi.LayerShape("t", 64, 6, 3, 64, "mxfp4")
    lay = mi.draw_layer(shape, 7, seed=3, identical_experts=True)
    ref = torch_dense_swiglu(L.to_f64(lay["x"]), *F.dequant_expert("mxfp4", lay["experts"], 0))
    return np.allclose(layer_fn(lay)["out"], ref, rtol=1e-12, atol=1e-13)


def test_identical_experts_reduce_to_one_ffn():
    assert pin_identical_experts(L.moe_layer)


def pin_shared_only(layer_fn):
    """Routed experts with W_down = 0: out = shared expert's FFN alone."""
    lay = _small("int4", E=5, k=2, d=128, f=128, n_shared=1, T=4, zipf_s=1.1)
    lay["experts"] = dict(lay["experts"])
    lay["experts"]["s2"] = torch.zeros_like(lay["experts"]["s2"])
    ref = torch_dense_swiglu(L.to_f64(lay["x"]), *F.dequant_expert("int4", lay["shared"], 0))
    return np.allclose(layer_fn(lay)["out"], ref, rtol=1e-12, atol=1e-14)


def test_shared_expert_weight_one():
    assert pin_shared_only(L.moe_layer)


def test_routed_plus_shared_decomposes():
    """out = routed-only layer + shared FFN (shared added with weight 1)."""
    lay = _small("int4", E=5, k=2, d=128, f=128, n_shared=1, T=4, zipf_s=1.1)
    full = L.moe_layer(lay)["out"]
    routed = L.moe_layer(dict(lay, shared=None))["out"]
    shared = torch_dense_swiglu(L.to_f64(lay["x"]), *F.dequant_expert("int4", lay["shared"], 0))
    assert np.allclose(full, routed + shared, rtol=1e-12, atol=1e-14)


def test_token_subset_matches_full():
    lay = _small("mxfp4", E=8, k=2, d=64, f=64, T=9)
    full = L.moe_layer(lay)
    sub = L.moe_layer(lay, tokens=[7, 2, 4])
    assert np.array_equal(sub["idx"], full["idx"][[7, 2, 4]])
    assert np.allclose(sub["out"], full["out"][[7, 2, 4]], rtol=1e-13, atol=0)


def test_empty_batch():
    lay = _small("bf16", T=0)
    r = L.moe_layer(lay)
    assert r["out"].shape == (0, 64) and r["idx"].shape == (0, 2)
    assert r["offsets"].tolist() == [0] * 5


# ------------------------------------------------------ fp32 logit bound ----

@pytest.mark.parametrize("router_fp32", [False, True])
def test_logit_error_bound_covers_fp32_sums(router_fp32):
    """beta bounds float32 evaluations of the logits in several orders."""
    shape = mi.LayerShape("t", 512, 16, 2, 32, "bf16", router_fp32=router_fp32, zipf_s=1.1)
    lay = mi.draw_layer(shape, 8, seed=2)
    x, wr, b = L.to_f64(lay["x"]), L.to_f64(lay["router"]), L.to_f64(lay["bias"])
    exact = L.router_logits(x, wr, b)
    x32, w32, b32 = x.astype(np.float32), wr.astype(np.float32), b.astype(np.float32)
    prod = x32[:, None, :] * w32[None, :, :]  # products rounded to fp32
    seq = np.zeros(exact.shape, np.float32)
    for i in range(512):  # one long chain
        seq = seq + prod[:, :, i]
    seq = seq + b32
    beta_seq = L.logit_error_bound(x, wr, b, chain=512)
    assert np.all(np.abs(seq - exact) <= beta_seq[:, None])
    # a 16-lane tree: lanes sum strided terms, then a pairwise fold
    lanes = prod.reshape(8, 16, 32, 16).sum(axis=2, dtype=np.float32)
    while lanes.shape[-1] > 1:
        lanes = lanes[..., 0::2] + lanes[..., 1::2]
    tree = lanes[..., 0] + b32
    beta_tree = L.logit_error_bound(x, wr, b, chain=32 + 4)
    assert np.all(np.abs(tree - exact) <= beta_tree[:, None])


# ----------------------------------------------------- planted mistakes ----

def test_pins_reject_planted_mistakes(monkeypatch):
    # gate and up swapped inside the FFN
    orig_ffn = L.swiglu_ffn

    def swapped(xrows, w13, w2):
        f = w13.shape[0] // 2
        return orig_ffn(xrows, np.concatenate([w13[f:], w13[:f]]), w2)
    with monkeypatch.context() as m:
        m.setattr(L, "swiglu_ffn", swapped)
        assert not pin_dense_single_expert(L.moe_layer, "bf16")

    # renormalisation dropped (softmax over all E kept)
    def no_renorm(logits, k):
        idx, gates, margin = _orig_topk(logits, k)
        p = scipy.special.softmax(logits, axis=1)
        return idx, np.take_along_axis(p, idx.astype(np.int64), 1), margin
    assert not pin_topk(no_renorm)

    # tie rule reversed (higher index wins)
    def high_index_wins(logits, k):
        E = logits.shape[1]
        rev = logits[:, ::-1]
        idx, g, m = _orig_topk(rev, k)
        return (E - 1 - idx).astype(np.int32), g, m
    assert not pin_topk(high_index_wins)

    # permutation ordered by token descending inside an expert
    def unstable(idx, E):
        c, o, rt, inv = L.permute(idx[::-1], E)
        T = idx.shape[0]
        return c, o, (T - 1 - rt) if T else rt, inv
    assert not pin_permute(unstable)

    # shared expert dropped
    def no_shared(lay, **kw):
        return L.moe_layer(dict(lay, shared=None), **kw)
    assert not pin_shared_only(no_shared)

    # uniform-average pin catches a combine that ignores the gates (sum, not mean)
    def ungated(lay, **kw):
        r = L.moe_layer(lay, **kw)
        r = dict(r)
        r["out"] = r["out"] * lay["shape"].top_k
        return r
    assert not pin_uniform_average(ungated)

    # forced-selection gates without the renormalisation (softmax over all E)
    def forced_no_renorm(logits, idx):
        p = scipy.special.softmax(logits, axis=1)
        return np.take_along_axis(p, idx.astype(np.int64), 1)
    assert not pin_gates_for(forced_no_renorm)

    # forced-selection gates taken from the wrong token's logits
    def forced_wrong_token(logits, idx):
        return L.gates_for(np.roll(logits, 1, axis=0), idx)
    assert not pin_gates_for(forced_wrong_token)

    # forced-selection gates in sorted instead of the selection's order
    def forced_sorted(logits, idx):
        return L.gates_for(logits, np.sort(idx, axis=1))
    assert not pin_gates_for(forced_sorted)

    # the layer ignoring a forced selection (keeps its own top-k)
    def ignores_forced(lay, forced_idx=None, **kw):
        return L.moe_layer(lay, **kw)
    assert not pin_forced_worked_example(ignores_forced)

    # the layer forcing the selection but keeping the top-k gates
    orig_gates_for = L.gates_for

    def stale_gates(logits, idx):
        return L.topk_select(logits, idx.shape[1])[1]
    with monkeypatch.context() as m:
        m.setattr(L, "gates_for", stale_gates)
        assert not pin_forced_worked_example(L.moe_layer)
    assert L.gates_for is orig_gates_for


_orig_topk = L.topk_select
