"""Seeded synthetic inputs for one sparse mixture-of-experts layer.

This module is shared by the CPU oracle (``oracle/``) and by the CUDA library's
tests and benchmark.  It only *draws* inputs: activations, router weights,
per-expert offsets and expert weights, and encodes the expert weights into the
storage formats the layer consumes (bf16, MXFP4, NVFP4, INT4 group-128).  It
decodes nothing and computes nothing of the layer itself (no router product, no
top-k, no permutation, no FFN, no combine); the decoders live, independently, in
``oracle/formats.py`` and in the CUDA kernels.

Workload shapes follow the five layer configurations this library is measured
on (tiny; gpt-oss-120b-shaped decode; Mixtral-8x7B-shaped prefill;
Kimi/DeepSeek-shaped decode with a shared expert and Zipf-skewed routing; an
offloaded NVFP4 bank).  Value distributions the configurations leave open are
fixed here: activations N(0,1) in bf16; expert weights N(0,0.02) before
encoding; routers N(0,0.02) except the gpt-oss router, uniform in
(-1/sqrt(d), 1/sqrt(d)); Zipf(s) offsets b_e = -s*ln(r_e) over a seeded
permutation r of 1..E.

Everything is drawn with ``torch.Generator`` on the requested device so that a
full-size benchmark layer can be drawn on the GPU in seconds; small test layers
are drawn on the CPU.  The same seed on different devices gives different (but
equally distributed) values.

Storage layout (the library's documented layout):
  * expert matrices are K-major ``[E][N][K]``; W13 rows ``[0, d_ff)`` are the
    gate projection and rows ``[d_ff, 2*d_ff)`` the up projection; W2 is
    ``[E][d][d_ff]``;
  * 4-bit codes are packed two per byte, the even-K element in the low nibble;
  * MXFP4 scales: E8M0 bytes ``[E][N][K/32]``; NVFP4 scales: E4M3 bytes
    ``[E][N][K/16]`` plus one fp32 global scale per expert and matrix;
    INT4 scales: bf16 ``[E][N][K/128]``;
  * bf16 tensors are torch bf16 tensors (their raw bits are what the C ABI sees).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional

import torch

WDTYPES = ("bf16", "mxfp4", "nvfp4", "int4")
BLOCK = {"bf16": 1, "mxfp4": 32, "nvfp4": 16, "int4": 128}


@dataclasses.dataclass(frozen=True)
class LayerShape:
    """Shape and encoding of one MoE layer."""

    name: str
    d_model: int
    n_experts: int
    top_k: int
    d_ff: int
    wdtype: str
    n_shared: int = 0
    router_fp32: bool = False
    router_init: str = "normal"  # "normal": N(0,0.02); "uniform": U(-1/sqrt(d), 1/sqrt(d))
    zipf_s: float = 0.0  # > 0: add Zipf(s) per-expert logit offsets
    weight_std: float = 0.02

    def replace(self, **kw) -> "LayerShape":
        return dataclasses.replace(self, **kw)


# The five measured configurations.  Token counts are per call.
TINY = LayerShape("tiny", 256, 8, 2, 512, "bf16", router_fp32=True)
GPTOSS = LayerShape("gptoss_decode", 2880, 128, 4, 2880, "mxfp4", router_init="uniform")
MIXTRAL = LayerShape("mixtral_prefill", 4096, 8, 2, 14336, "bf16")
KIMI = LayerShape("kimi_decode", 7168, 384, 8, 2048, "int4", n_shared=1, zipf_s=1.1)
BANK = LayerShape("offload_bank", 4096, 256, 8, 1536, "nvfp4", zipf_s=1.1)

# The Mixtral-shaped prefill layer with 4-bit experts (4-bit prefill on the
# tensor cores); not among the five measured configurations above.
MIXTRAL_MXFP4 = MIXTRAL.replace(name="mixtral_prefill_mxfp4", wdtype="mxfp4")
MIXTRAL_NVFP4 = MIXTRAL.replace(name="mixtral_prefill_nvfp4", wdtype="nvfp4")
MIXTRAL_INT4 = MIXTRAL.replace(name="mixtral_prefill_int4", wdtype="int4")

CONFIG_TOKENS = {
    "tiny": (16,),
    "gptoss_decode": (1, 8, 32, 64),
    "mixtral_prefill": (4096,),
    "kimi_decode": (1, 8, 32, 128),
    "offload_bank": (1, 4, 16),
}
BANK_LAYERS = 48
BANK_SLOTS_PER_LAYER = 64  # 25% of 256 experts
BANK_STEPS = 512

CONFIGS = {c.name: c for c in (TINY, GPTOSS, MIXTRAL, KIMI, BANK, MIXTRAL_MXFP4, MIXTRAL_NVFP4, MIXTRAL_INT4)}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) & 0x7FFFFFFFFFFFFFFF)
    return g


# ----------------------------------------------------------------------------
# Encoders (storage formats).  These turn fp32 draws into codes + scales; they
# are data preparation only.  Rounding is round-to-nearest-even throughout.
# ----------------------------------------------------------------------------

# Non-negative E2M1 grid (OCP MX v1.0 FP4 element type); index = 3-bit magnitude code.
_E2M1_GRID = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)


def _encode_e2m1(v: torch.Tensor) -> torch.Tensor:
    """fp32 -> 4-bit E2M1 code (uint8 in [0,16)), round-to-nearest-even, saturating at 6."""
    a = v.abs()
    # Midpoints between grid neighbours; at an exact midpoint pick the even
    # mantissa (codes 0, 2, 4, 6 have mantissa bit 0).
    mids = (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0)
    code = torch.zeros_like(a, dtype=torch.uint8)
    for i, m in enumerate(mids):
        lower_even = (i % 2) == 0  # grid[i] has an even code when i is even
        above = (a > m) | ((a == m) & (not lower_even))
        code = torch.where(above, torch.full_like(code, i + 1), code)
    sign = (v < 0) & (code > 0)
    return code | (sign.to(torch.uint8) << 3)


def _pack_nibbles(codes: torch.Tensor) -> torch.Tensor:
    """[..., K] uint8 codes in [0,16) -> [..., K/2] bytes, even K in the low nibble."""
    lo = codes[..., 0::2]
    hi = codes[..., 1::2]
    return (lo | (hi << 4)).contiguous()


def encode_mxfp4(w: torch.Tensor):
    """[..., K] fp32 -> (codes [..., K/2] u8, scales [..., K/32] u8 E8M0).

    Shared exponent = floor(log2(block amax)) - 2 (the E2M1 element's largest
    exponent), clamped to [-40, 20] so that no element can overflow fp32/bf16.
    """
    K = w.shape[-1]
    assert K % 32 == 0
    blk = w.reshape(*w.shape[:-1], K // 32, 32)
    amax = blk.abs().amax(dim=-1)
    e = torch.floor(torch.log2(torch.where(amax > 0, amax, torch.ones_like(amax)))) - 2
    e = torch.where(amax > 0, e, torch.full_like(e, -40.0)).clamp(-40, 20)
    q = _encode_e2m1(blk / torch.exp2(e).unsqueeze(-1)).reshape(w.shape)
    return _pack_nibbles(q), (e + 127).to(torch.uint8).contiguous()


def encode_nvfp4(w: torch.Tensor):
    """[E, N, K] fp32 -> (codes [E,N,K/2] u8, scales [E,N,K/16] u8 E4M3, gscale [E] fp32).

    Per expert matrix: g = amax / (6*448); per 16-block s = E4M3(amax_blk / (6*g));
    element = E2M1(w / (s*g)).
    """
    E, N, K = w.shape
    assert K % 16 == 0
    amax_t = w.abs().reshape(E, -1).amax(dim=1)
    g = torch.where(amax_t > 0, amax_t / (6.0 * 448.0), torch.ones_like(amax_t)).float()
    blk = w.reshape(E, N, K // 16, 16)
    amax_b = blk.abs().amax(dim=-1)
    s8 = (amax_b / (6.0 * g.view(E, 1, 1))).clamp(max=448.0).to(torch.float8_e4m3fn)
    s = s8.float()
    denom = (s * g.view(E, 1, 1)).unsqueeze(-1)
    ratio = torch.where(denom > 0, blk / torch.where(denom > 0, denom, torch.ones_like(denom)),
                        torch.zeros_like(blk))
    q = _encode_e2m1(ratio).reshape(E, N, K)
    return _pack_nibbles(q), s8.view(torch.uint8).contiguous(), g.contiguous()


def encode_int4_g128(w: torch.Tensor):
    """[..., K] fp32 -> (codes [..., K/2] u8 two's complement, scales [..., K/128] bf16).

    Symmetric: s = bf16(amax_grp / 7); q = clamp(RNE(w / s), -8, 7).
    """
    K = w.shape[-1]
    assert K % 128 == 0
    blk = w.reshape(*w.shape[:-1], K // 128, 128)
    s = (blk.abs().amax(dim=-1) / 7.0).to(torch.bfloat16)
    sf = s.float().unsqueeze(-1)
    q = torch.where(sf > 0, torch.round(blk / torch.where(sf > 0, sf, torch.ones_like(sf))),
                    torch.zeros_like(blk)).clamp(-8, 7)
    q = q.to(torch.int8).reshape(w.shape)
    return _pack_nibbles((q.to(torch.uint8) & 0xF)), s.contiguous()


def encode_matrix(w: torch.Tensor, wdtype: str) -> Dict[str, torch.Tensor]:
    """Encode an ``[E, N, K]`` fp32 stack in ``wdtype``; returns codes/scales/gscale."""
    if wdtype == "bf16":
        return {"w": w.to(torch.bfloat16).contiguous()}
    if wdtype == "mxfp4":
        c, s = encode_mxfp4(w)
        return {"w": c, "s": s}
    if wdtype == "nvfp4":
        c, s, g = encode_nvfp4(w)
        return {"w": c, "s": s, "g": g}
    if wdtype == "int4":
        c, s = encode_int4_g128(w)
        return {"w": c, "s": s}
    raise ValueError(wdtype)


# ----------------------------------------------------------------------------
# Layer draws
# ----------------------------------------------------------------------------

EXPERT_CHUNK = 8


def draw_experts(shape: LayerShape, n: int, seed: int, device="cpu", chunks: Optional[list] = None):
    """Draw and encode ``n`` experts of ``shape`` (W13 and W2).

    Returns dict with keys w13, s13, g13, w2, s2, g2 (absent keys = not used by
    the format).  Experts are drawn EXPERT_CHUNK at a time, each chunk from its
    own generator seeded by (seed, chunk), so that a subset of chunks can be
    drawn alone (``chunks``: list of chunk indices; the result then holds only
    those chunks' experts, in order).
    """
    d, f = shape.d_model, shape.d_ff
    parts13, parts2 = [], []
    todo = range(0, (n + EXPERT_CHUNK - 1) // EXPERT_CHUNK) if chunks is None else chunks
    for ci in todo:
        e0 = ci * EXPERT_CHUNK
        m = min(EXPERT_CHUNK, n - e0)
        gen = _gen(seed * 65537 + ci, device)
        w13 = torch.randn(m, 2 * f, d, generator=gen, device=device) * shape.weight_std
        w2 = torch.randn(m, d, f, generator=gen, device=device) * shape.weight_std
        parts13.append(encode_matrix(w13, shape.wdtype))
        parts2.append(encode_matrix(w2, shape.wdtype))
        del w13, w2
    out = {}
    for key in parts13[0]:
        out[key + "13" if key != "w" else "w13"] = torch.cat([p[key] for p in parts13]).contiguous()
        out[key + "2" if key != "w" else "w2"] = torch.cat([p[key] for p in parts2]).contiguous()
    return out


def zipf_offsets(n_experts: int, s: float, seed: int, device="cpu") -> torch.Tensor:
    """Per-expert logit offsets b_e = -s*ln(r_e), r a seeded permutation of 1..E (fp32)."""
    gen = _gen(seed ^ 0x5A17F, "cpu")
    r = torch.randperm(n_experts, generator=gen).double() + 1.0
    return (-s * torch.log(r)).float().to(device)


def draw_router(shape: LayerShape, seed: int, device="cpu") -> torch.Tensor:
    gen = _gen(seed ^ 0x20F7E5, device)
    E, d = shape.n_experts, shape.d_model
    if shape.router_init == "uniform":
        r = (torch.rand(E, d, generator=gen, device=device) * 2 - 1) / math.sqrt(d)
    else:
        r = torch.randn(E, d, generator=gen, device=device) * 0.02
    return r.float().contiguous() if shape.router_fp32 else r.to(torch.bfloat16).contiguous()


def draw_tokens(T: int, d: int, seed: int, device="cpu") -> torch.Tensor:
    gen = _gen(seed ^ 0x70CE45, device)
    return torch.randn(T, d, generator=gen, device=device).to(torch.bfloat16).contiguous()


def draw_layer(shape: LayerShape, T: int, seed: int = 0, device="cpu",
               identical_experts: bool = False) -> Dict[str, object]:
    """All inputs of one layer call: x, router, bias, routed and shared experts."""
    lay: Dict[str, object] = {"shape": shape, "T": T, "seed": seed}
    lay["x"] = draw_tokens(T, shape.d_model, seed, device)
    lay["router"] = draw_router(shape, seed, device)
    lay["bias"] = zipf_offsets(shape.n_experts, shape.zipf_s, seed, device) if shape.zipf_s > 0 else None
    if identical_experts:
        one = draw_experts(shape, 1, seed * 7919 + 1, device)
        lay["experts"] = {k: v.expand(shape.n_experts, *v.shape[1:]).contiguous() for k, v in one.items()}
    else:
        lay["experts"] = draw_experts(shape, shape.n_experts, seed * 7919 + 1, device)
    lay["shared"] = draw_experts(shape, shape.n_shared, seed * 7919 + 2, device) if shape.n_shared else None
    return lay


def draw_verify_tokens(n_seq: int, depth: int, d: int, rho: float, seed: int, device="cpu") -> torch.Tensor:
    """Activations of ``n_seq`` speculative verification blocks of ``depth + 1``
    positions each (the target's own position and ``depth`` drafted ones),
    block-major: row b*(depth+1) + i is position i of sequence b.  Positions
    of one sequence are correlated, x = sqrt(rho) u_b + sqrt(1 - rho) z_(b,i)
    with u, z ~ N(0, 1), so that they tend to select the same experts; bf16."""
    gen = _gen(seed ^ 0x5EC0DE, device)
    u = torch.randn(n_seq, 1, d, generator=gen, device=device)
    z = torch.randn(n_seq, depth + 1, d, generator=gen, device=device)
    x = math.sqrt(rho) * u + math.sqrt(1.0 - rho) * z
    return x.reshape(n_seq * (depth + 1), d).to(torch.bfloat16).contiguous()


def draw_accepts(n_seq: int, depth: int, alpha: float, seed: int) -> torch.Tensor:
    """Seeded accept flags of the drafted tokens, bool [n_seq, depth]: each
    drafted token is accepted with probability ``alpha`` (the verifier keeps
    the leading run of accepted drafts)."""
    gen = _gen(seed ^ 0xACCE97, "cpu")
    return torch.rand(n_seq, depth, generator=gen) < alpha


def expert_bytes(shape: LayerShape) -> int:
    """Bytes of one expert's W13 + W2 codes and scales (global scales excluded)."""
    d, f = shape.d_model, shape.d_ff
    vals = 3 * d * f
    if shape.wdtype == "bf16":
        return vals * 2
    scale_bytes = {"mxfp4": 1, "nvfp4": 1, "int4": 2}[shape.wdtype]
    return vals // 2 + (vals // BLOCK[shape.wdtype]) * scale_bytes


def bank_step_tokens(step: int, T: int, d: int, seed: int, device="cpu") -> torch.Tensor:
    """Fresh x_0 for step ``step`` of the offloaded-bank decode (seeded by (seed, step))."""
    return draw_tokens(T, d, seed * 1_000_003 + step, device)


def bank_layer(shape: LayerShape, layer: int, seed: int, device="cpu", n_experts: Optional[int] = None):
    """Router, offsets and experts of layer ``layer`` of the offloaded bank."""
    E = n_experts or shape.n_experts
    sh = shape.replace(n_experts=E)
    s = seed * 4099 + layer
    return {
        "router": draw_router(sh, s, device),
        "bias": zipf_offsets(E, sh.zipf_s, s, device) if sh.zipf_s > 0 else None,
        "experts": draw_experts(sh, E, s * 7919 + 1, device),
    }
