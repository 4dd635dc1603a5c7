"""Test-side harness: run the CUDA library through its C ABI on a drawn layer
and compare every result with the oracle.

Comparison rules:
* expert indices, per-expert counts, offsets, row order and inverse rows are
  compared bit for bit.  A token whose routing margin m_t is not larger than
  2*beta_t (beta_t the fp32 error bound of a logit for the kernel's
  documented summation depth) has no unique answer under fp32; for such a
  token the GPU's choice must be *valid* (every chosen logit within 2*beta_t
  of every unchosen one, in the right order), and the oracle is re-run with
  the GPU's choice for the value checks;
* gates: |g_gpu - g_ref| <= 1e-5 + 2*g*beta (softmax perturbation bound);
* outputs: max|gpu - ref| <= 1e-2 * max|ref| over the compared tokens.
"""
from __future__ import annotations

import numpy as np
import torch

import expert_ffn_layer_route_b200 as moe
import moe_inputs as mi
from oracle import layer as OL

OUT_RTOL = 1e-2


def to_device(lay, device="cuda"):
    out = dict(lay)
    out["x"] = lay["x"].to(device)
    out["router"] = lay["router"].to(device)
    out["bias"] = lay["bias"].to(device) if lay.get("bias") is not None else None
    out["experts"] = {k: v.to(device) for k, v in lay["experts"].items()}
    out["shared"] = {k: v.to(device) for k, v in lay["shared"].items()} if lay.get("shared") else None
    return out


def to_host(lay):
    return to_device(lay, "cpu")


def run_layer(dlay, stream=None):
    """moe_layer_forward on device tensors; returns out and the routing read from the workspace."""
    shape, T = dlay["shape"], dlay["x"].shape[0]
    desc = moe.make_desc(shape, T)
    ws = torch.empty(max(moe.moe_workspace_size(desc), 16), dtype=torch.uint8, device="cuda")
    out = torch.empty(T, shape.d_model, dtype=torch.bfloat16, device="cuda")
    routed = moe.make_weights(dlay["experts"])
    shared = moe.make_weights(dlay["shared"]) if dlay.get("shared") else None
    moe.moe_layer_forward(desc, dlay["x"], dlay["router"], dlay["bias"], routed, shared, out, ws, stream)
    torch.cuda.synchronize()
    L = moe.moe_workspace_layout_of(desc)
    R = T * shape.top_k

    def view(off, n, dt):
        return ws[off: off + n * 4].view(dt).clone() if n else torch.empty(0, dtype=dt, device="cuda")

    return {
        "out": out,
        "idx": view(L.topk_idx, R, torch.int32).view(T, shape.top_k),
        "gates": view(L.topk_w, R, torch.float32).view(T, shape.top_k),
        "offsets": view(L.offsets, shape.n_experts + 1, torch.int32),
        "row_token": view(L.row_token, R, torch.int32),
        "inv": view(L.inv, R, torch.int32),
        "ws": ws,
        "desc": desc,
    }


def run_steps(dlay, stream=None):
    """The same layer through the four separate entry points."""
    shape, T = dlay["shape"], dlay["x"].shape[0]
    desc = moe.make_desc(shape, T)
    dev = "cuda"
    ws = torch.empty(max(moe.moe_workspace_size(desc), 16), dtype=torch.uint8, device=dev)
    k, E, d = shape.top_k, shape.n_experts, shape.d_model
    idx = torch.empty(T, k, dtype=torch.int32, device=dev)
    gw = torch.empty(T, k, dtype=torch.float32, device=dev)
    offs = torch.empty(E + 1, dtype=torch.int32, device=dev)
    rtok = torch.empty(T * k, dtype=torch.int32, device=dev)
    inv = torch.empty(T * k, dtype=torch.int32, device=dev)
    y = torch.empty(max(T * k, 1), d, dtype=torch.bfloat16, device=dev)
    ysh = torch.empty(max(shape.n_shared, 1) * max(T, 1), d, dtype=torch.bfloat16, device=dev)
    out = torch.empty(T, d, dtype=torch.bfloat16, device=dev)
    moe.moe_route_topk(desc, dlay["x"], dlay["router"], dlay["bias"], idx, gw, ws, stream)
    moe.moe_permute(desc, idx, offs, rtok, inv, stream)
    routed = moe.make_weights(dlay["experts"])
    shared = moe.make_weights(dlay["shared"]) if dlay.get("shared") else None
    moe.moe_grouped_ffn(desc, routed, shared, offs, rtok, dlay["x"], y, ysh if shape.n_shared else None, ws,
                        stream)
    moe.moe_combine(desc, y, inv, gw, ysh if shape.n_shared else None, out, stream)
    torch.cuda.synchronize()
    return {"out": out, "idx": idx, "gates": gw, "offsets": offs, "row_token": rtok, "inv": inv, "y": y}


def _routing_only(hlay, tokens, chain):
    """The oracle's routing of the given tokens (no expert FFN)."""
    shape = hlay["shape"]
    x = OL.to_f64(hlay["x"])
    tok = np.arange(x.shape[0]) if tokens is None else np.asarray(list(tokens), dtype=np.int64)
    x = x[tok]
    wr = OL.to_f64(hlay["router"])
    b = OL.to_f64(hlay["bias"]) if hlay.get("bias") is not None else None
    logits = OL.router_logits(x, wr, b)
    idx, gates, margin = OL.topk_select(logits, shape.top_k)
    beta = OL.logit_error_bound(x, wr, b, chain)
    return {"idx": idx, "gates": gates, "logits": logits, "margin": margin, "beta": beta, "tokens": tok}


def check_routing(hlay, idx_gpu, gates_gpu, tokens=None, values=True):
    """Bit-exact indices for unique tokens, validity for the others.

    Returns (ref, n_ambiguous) where ref is the oracle run (forced to the
    GPU's choice where the choice is not unique).  values=False checks the
    routing alone (no expert FFN in the oracle)."""
    shape = hlay["shape"]
    chain = moe.router_sum_depth(shape.d_model)
    ref = OL.moe_layer(hlay, tokens=tokens, chain=chain) if values else _routing_only(hlay, tokens, chain)
    idx_g = idx_gpu.cpu().numpy()
    if tokens is not None:
        idx_g = idx_g[np.asarray(list(tokens))]
    unique = ref["margin"] > 2 * ref["beta"]
    n_amb = int((~unique).sum())
    assert np.array_equal(idx_g[unique], ref["idx"][unique]), "expert indices differ on tokens with a unique choice"
    if n_amb:
        lg, beta = ref["logits"], ref["beta"]
        for p in np.nonzero(~unique)[0]:
            ch = idx_g[p]
            assert len(set(ch.tolist())) == shape.top_k
            rest = np.setdiff1d(np.arange(shape.n_experts), ch)
            assert lg[p, ch].min() >= lg[p, rest].max() - 2 * beta[p] if rest.size else True
            assert np.all(np.diff(lg[p, ch]) <= 2 * beta[p])
        forced = np.zeros((hlay["x"].shape[0], shape.top_k), dtype=np.int32)
        forced[ref["tokens"]] = idx_g
        if values:
            ref = OL.moe_layer(hlay, forced_idx=forced, tokens=tokens, chain=chain)
        else:
            ref = dict(ref, idx=idx_g, gates=OL.gates_for(ref["logits"], idx_g))
    g = gates_gpu.cpu().double().numpy()
    if tokens is not None:
        g = g[np.asarray(list(tokens))]
    tol = 1e-5 + 2 * ref["gates"] * ref["beta"][:, None]
    assert np.all(np.abs(g - ref["gates"]) <= tol), float(np.abs(g - ref["gates"]).max())
    return ref, n_amb


def check_permutation(res, shape):
    idx = res["idx"].cpu().numpy()
    counts, offsets, row_token, inv = OL.permute(idx, shape.n_experts)
    assert np.array_equal(res["offsets"].cpu().numpy(), offsets)
    assert np.array_equal(res["row_token"].cpu().numpy(), row_token)
    assert np.array_equal(res["inv"].cpu().numpy(), inv)


def check_output(out_gpu, ref_out, tokens=None, rtol=OUT_RTOL):
    o = out_gpu.float().cpu().double().numpy()
    if tokens is not None:
        o = o[np.asarray(list(tokens))]
    scale = np.abs(ref_out).max()
    err = np.abs(o - ref_out).max() if o.size else 0.0
    assert np.all(np.isfinite(o))
    assert err <= rtol * scale, f"max err {err:.3e} > {rtol} * {scale:.3e}"
    return err / scale if scale else 0.0


def full_check(lay_host, res):
    ref, n_amb = check_routing(lay_host, res["idx"], res["gates"])
    check_permutation(res, lay_host["shape"])
    rel = check_output(res["out"], ref["out"])
    return rel, n_amb
