"""Exact float64 decoders of the expert weight storage formats.

The pages name the formats but do not define them: gpt-oss and DeepSeek-V4-Flash
ship FP4 experts and Kimi-K2.6 INT4 experts ("Mixture of experts VRAM: total vs
active parameters", section "How current MoE models route each token"); the
Galactus measurements list "MXFP4 experts" and "native-INT4 MoE" exports
("Understanding MoE Inference Costs on Galactus", section "The August
comparison", table).  The decoders below follow the public format definitions:

* E2M1 (the FP4 element of OCP Microscaling v1.0 and of NVFP4): 1 sign bit,
  2 exponent bits with bias 1, 1 mantissa bit; exponent field 0 is subnormal
  (value m * 0.5); no inf/NaN.
* E8M0 (the MX shared scale): value 2^(v - 127); v = 255 is NaN.
* E4M3 (the NVFP4 block scale, OCP FP8 "E4M3FN"): 1 sign, 4 exponent bits with
  bias 7, 3 mantissa bits; exponent field 0 is subnormal (m/8 * 2^-6); the
  all-ones pattern S.1111.111 is NaN; no infinities.
* INT4: 4-bit two's complement, q in [-8, 7].
* bf16: 1 sign, 8 exponent bits (bias 127), 7 mantissa bits.

Block sizes: MXFP4 one E8M0 scale per 32 elements along K; NVFP4 one E4M3 scale
per 16 elements times an fp32 per-matrix global scale; INT4 one bf16 scale per
128 elements.  4-bit codes are packed two per byte with the even-K element in
the low nibble.
"""
from __future__ import annotations

import numpy as np


def _as_np(a) -> np.ndarray:
    if hasattr(a, "detach"):  # torch tensor
        t = a.detach().cpu()
        import torch  # local: the oracle itself only needs numpy

        if t.dtype == torch.bfloat16:
            t = t.view(torch.int16)
        return t.numpy()
    return np.asarray(a)


def bf16_bits_to_f64(bits) -> np.ndarray:
    """bf16 raw 16-bit patterns -> float64, from the field definition (through
    the definition's table of all 65536 patterns: same values, one lookup per
    element)."""
    b = _as_np(bits).astype(np.uint16)
    return _bf16_table()[b]


_BF16_TABLE = None


def _bf16_table() -> np.ndarray:
    global _BF16_TABLE
    if _BF16_TABLE is None:
        _BF16_TABLE = _bf16_fields_to_f64(np.arange(65536, dtype=np.int64))
    return _BF16_TABLE


def _bf16_fields_to_f64(b: np.ndarray) -> np.ndarray:
    """sign, 8-bit exponent (bias 127, 0 = subnormal, 255 = inf/NaN), 7-bit mantissa."""
    s = (b >> 15) & 1
    e = (b >> 7) & 0xFF
    m = b & 0x7F
    mag = np.where(
        e == 0,
        np.ldexp(m.astype(np.float64) / 128.0, -126),
        np.ldexp(1.0 + m.astype(np.float64) / 128.0, (e - 127).astype(np.int64)),
    )
    mag = np.where(e == 0xFF, np.where(m == 0, np.inf, np.nan), mag)
    return np.where(s == 1, -mag, mag)


def e2m1_to_f64(code) -> np.ndarray:
    """4-bit E2M1 codes (0..15) -> float64."""
    c = _as_np(code).astype(np.int64) & 0xF
    s = (c >> 3) & 1
    e = (c >> 1) & 3
    m = c & 1
    mag = np.where(e == 0, 0.5 * m, np.ldexp(1.0 + 0.5 * m, e - 1))
    return np.where(s == 1, -mag, mag)


def e8m0_to_f64(v) -> np.ndarray:
    """E8M0 scale bytes -> 2^(v-127); 0xFF -> NaN."""
    b = _as_np(v).astype(np.int64) & 0xFF
    return np.where(b == 0xFF, np.nan, np.ldexp(1.0, b - 127))


def e4m3_to_f64(v) -> np.ndarray:
    """E4M3 (FN) bytes -> float64; S.1111.111 -> NaN."""
    b = _as_np(v).astype(np.int64) & 0xFF
    s = (b >> 7) & 1
    e = (b >> 3) & 0xF
    m = b & 7
    mag = np.where(e == 0, np.ldexp(m / 8.0, -6), np.ldexp(1.0 + m / 8.0, e - 7))
    mag = np.where((e == 0xF) & (m == 7), np.nan, mag)
    return np.where(s == 1, -mag, mag)


def int4_to_f64(code) -> np.ndarray:
    """4-bit two's complement codes -> float64 in [-8, 7]."""
    c = _as_np(code).astype(np.int64) & 0xF
    return np.where(c >= 8, c - 16, c).astype(np.float64)


def unpack_nibbles(packed) -> np.ndarray:
    """[..., K/2] bytes -> [..., K] codes, even K from the low nibble."""
    p = _as_np(packed).astype(np.uint8)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = p & 0xF
    out[..., 1::2] = p >> 4
    return out


def _decode_codes(codes: np.ndarray, element_decoder) -> np.ndarray:
    """Apply a 4-bit element decoder through its 16-entry table (same values,
    one lookup per element)."""
    table = element_decoder(np.arange(16))
    return table[codes]


def _times_blocks(values: np.ndarray, scale: np.ndarray, block: int) -> np.ndarray:
    """values [..., K] * scale [..., K/block], each scale covering `block` consecutive K."""
    shp = values.shape
    v = values.reshape(shp[:-1] + (shp[-1] // block, block))
    return (v * scale[..., None]).reshape(shp)


def dequant(wdtype: str, w, s=None, g=None) -> np.ndarray:
    """Decode one stored matrix (or a stack of them) to float64 ``[..., N, K]``.

    ``w``: bf16 values, or packed 4-bit codes ``[..., N, K/2]``.
    ``s``: block scales ``[..., N, K/blk]`` (E8M0 / E4M3 bytes, or bf16 for INT4).
    ``g``: NVFP4 fp32 global scale, scalar or one per leading matrix.
    """
    if wdtype == "bf16":
        return bf16_bits_to_f64(w)
    codes = unpack_nibbles(w)
    if wdtype == "mxfp4":
        return _times_blocks(_decode_codes(codes, e2m1_to_f64), e8m0_to_f64(s), 32)
    if wdtype == "nvfp4":
        gs = np.asarray(_as_np(g), dtype=np.float64)
        v = _times_blocks(_decode_codes(codes, e2m1_to_f64), e4m3_to_f64(s), 16)
        if gs.ndim == 0:
            return v * gs
        return v * gs.reshape(gs.shape + (1,) * (v.ndim - gs.ndim))
    if wdtype == "int4":
        return _times_blocks(_decode_codes(codes, int4_to_f64), bf16_bits_to_f64(s), 128)
    raise ValueError(wdtype)


def dequant_expert(wdtype: str, experts: dict, e: int):
    """(W13 [2*d_ff, d], W2 [d, d_ff]) of expert ``e`` as float64."""
    def pick(key):
        v = experts.get(key)
        return None if v is None else v[e]

    w13 = dequant(wdtype, pick("w13"), pick("s13"), pick("g13"))
    w2 = dequant(wdtype, pick("w2"), pick("s2"), pick("g2"))
    return w13, w2
