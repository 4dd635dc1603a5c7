"""Pins for the oracle's format decoders (CPU only).

Each decoder is checked against something other than itself: the published
E2M1 grid, torch's own float8_e4m3fn and bfloat16 decoders (library
routines), Python's exact power-of-two arithmetic for E8M0, and the
two's-complement definition for INT4.  Then every code times a sweep of
scales, and encode -> decode -> encode round trips with the independent
encoders in ``moe_inputs``.
"""
import math

import numpy as np
import pytest
import torch

import moe_inputs as mi
from oracle import formats as F

# OCP Microscaling Formats v1.0, FP4 (E2M1) element: codes 0..15 in order.
E2M1_SPEC = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0,
             -0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0]


def test_e2m1_all_codes_match_spec_grid():
    got = F.e2m1_to_f64(np.arange(16))
    assert got.tolist() == E2M1_SPEC
    assert np.signbit(got[8])  # code 8 is -0


def test_e4m3_all_codes_match_torch_decoder():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = F.e4m3_to_f64(np.arange(256))
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    assert np.array_equal(ref[~nan], got[~nan])
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9


def test_e8m0_is_power_of_two():
    got = F.e8m0_to_f64(np.arange(256))
    for v in range(255):
        assert got[v] == math.ldexp(1.0, v - 127)
    assert math.isnan(got[255])


def test_bf16_all_patterns_match_torch():
    bits = torch.arange(65536, dtype=torch.int32).to(torch.int16)
    ref = bits.view(torch.bfloat16).to(torch.float64).numpy()
    got = F.bf16_bits_to_f64(bits.numpy())
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    assert np.array_equal(ref[~nan], got[~nan])


def test_int4_twos_complement():
    assert F.int4_to_f64(np.arange(16)).tolist() == [0, 1, 2, 3, 4, 5, 6, 7, -8, -7, -6, -5, -4, -3, -2, -1]


def test_nibble_order_even_k_low():
    assert F.unpack_nibbles(np.array([[0x21, 0xF0]], dtype=np.uint8)).tolist() == [[1, 2, 0, 15]]


def _packed_all_codes(reps):
    codes = np.tile(np.arange(16, dtype=np.uint8), reps)
    return (codes[0::2] | (codes[1::2] << 4)).astype(np.uint8), codes


def test_mxfp4_every_code_times_scale_sweep():
    packed, codes = _packed_all_codes(2)  # 32 elements = one block
    for s in range(87, 148):  # 2^-40 .. 2^20
        v = F.dequant("mxfp4", packed[None], np.array([[s]], dtype=np.uint8))[0]
        ref = np.array([E2M1_SPEC[c] * math.ldexp(1.0, s - 127) for c in codes])
        assert np.array_equal(v, ref)


def test_nvfp4_every_code_times_every_scale():
    packed, codes = _packed_all_codes(1)  # 16 elements = one block
    g = np.float32(0.37)
    for sb in range(0x7F):  # every non-negative finite E4M3 scale
        sv = torch.tensor([sb], dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).double().item()
        v = F.dequant("nvfp4", packed[None], np.array([[sb]], dtype=np.uint8), g)[0]
        ref = np.array([E2M1_SPEC[c] * sv * float(g) for c in codes])
        assert np.array_equal(v, ref)


def test_int4_every_code_times_scale_sweep():
    codes = np.tile(np.arange(16, dtype=np.uint8), 8)  # 128 elements
    packed = (codes[0::2] | (codes[1::2] << 4)).astype(np.uint8)
    for sval in (1e-3, 0.0123, 0.5, 3.0, -0.25):
        sb = torch.tensor([sval]).to(torch.bfloat16)
        v = F.dequant("int4", packed[None], sb.view(torch.int16).numpy()[None])[0]
        ref = np.array([(c - 16 if c >= 8 else c) * sb.double().item() for c in codes.tolist()])
        assert np.array_equal(v, ref)


@pytest.mark.parametrize("wdtype", ["mxfp4", "nvfp4", "int4", "bf16"])
def test_encode_decode_error_bounds(wdtype):
    """Generator encoders + oracle decoders agree: each decoded weight lies
    within half a grid step (or the saturation bound) of the fp32 draw."""
    torch.manual_seed(0)
    w = torch.randn(3, 64, 256) * 0.02
    w[0, 0, :32] = 0.0  # an all-zero block
    enc = mi.encode_matrix(w, wdtype)
    if wdtype == "nvfp4":
        deq = np.stack([F.dequant("nvfp4", enc["w"][e], enc["s"][e], enc["g"][e]) for e in range(3)])
    else:
        deq = F.dequant(wdtype, enc["w"], enc.get("s"))
    wf = w.double().numpy()
    err = np.abs(deq - wf)
    if wdtype == "bf16":
        assert np.all(err <= np.abs(wf) * 2.0 ** -8)
    elif wdtype == "mxfp4":
        blk = np.abs(wf).reshape(3, 64, 8, 32).max(-1)
        # step at most 2 on the [4, 6] segment, scaled by 2^e with 2^e <= amax/4
        assert np.all(err.reshape(3, 64, 8, 32) <= (blk / 4.0 * 2.0)[..., None] + 1e-30)
    elif wdtype == "int4":
        s = F.bf16_bits_to_f64(enc["s"]).reshape(3, 64, 2, 1)
        assert np.all(err.reshape(3, 64, 2, 128) <= s * 0.5 + np.abs(s) * 1e-2 + 1e-30)
    else:
        blk = np.abs(wf).reshape(3, 64, 16, 16).max(-1)
        assert np.all(err.reshape(3, 64, 16, 16) <= (blk / 3.0)[..., None] + 1e-9)
    assert np.all(deq[0, 0, :32] == 0.0)


@pytest.mark.parametrize("wdtype", ["mxfp4", "int4"])
def test_quantise_dequant_roundtrip(wdtype):
    """Re-encoding decoded weights reproduces the codes (quantise(dequant(q)) = q)."""
    torch.manual_seed(1)
    w = torch.randn(2, 32, 256) * 0.02
    enc = mi.encode_matrix(w, wdtype)
    deq = torch.from_numpy(F.dequant(wdtype, enc["w"], enc["s"])).float()
    enc2 = mi.encode_matrix(deq, wdtype)
    assert torch.equal(enc["w"], enc2["w"])
