"""The table-lookup E2M1 decode of the 4-bit tensor-core path (NVFP4
experts), checked on the CPU in exact arithmetic.

The converter warps turn eight E2M1 codes (one 32-bit word, nibble i = K i)
into four fp16 pairs with byte permutes only: magnitudes through an 8-entry
byte table of fp16 high bytes (the low bytes being zero), a spreading
permute, and the sign bits moved to bit 15 / 31 of each pair.  This test restates those steps (the PTX prmt semantics: bytes 0-3 from
the first operand, 4-7 from the second, selector nibble n picks output byte n)
and compares every result with the E2M1 value from the format definition,
for every code in every nibble position.
"""
import numpy as np

E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def prmt(a, b, sel):
    src = [(a >> (8 * i)) & 0xFF for i in range(4)] + [(b >> (8 * i)) & 0xFF for i in range(4)]
    out = 0
    for n in range(4):
        nib = (sel >> (4 * n)) & 0xF
        assert nib < 8  # the decoder never uses the sign-replicate mode
        out |= src[nib] << (8 * n)
    return out


def lut_decode(w):
    m = w & 0x77777777
    m2 = m >> 16
    s8 = w & 0x88888888
    t = (s8 << 4) & 0xFFFFFFFF
    hA, hB = prmt(0x3E3C3800, 0x46444240, m), prmt(0x3E3C3800, 0x46444240, m2)
    o = [prmt(hA, 0, 0x1404), prmt(hA, 0, 0x3424), prmt(hB, 0, 0x1404), prmt(hB, 0, 0x3424)]
    for b in range(4):
        sg = prmt(t, s8, b * 0x11 | (4 + b) * 0x1100)
        o[b] |= sg & 0x80008000
    return o


def f16_bits_to_float(h):
    return float(np.array([h], dtype=np.uint16).view(np.float16)[0])


def e2m1(code):
    v = E2M1[code & 7]
    return -v if code & 8 else v


def check_word(w):
    o = lut_decode(w)
    for i in range(8):
        h = (o[i // 2] >> (16 * (i % 2))) & 0xFFFF
        got = f16_bits_to_float(h)
        want = e2m1((w >> (4 * i)) & 0xF)
        assert got == want and (np.signbit(got) == bool((w >> (4 * i + 3)) & 1) or want != 0), (hex(w), i, got, want)


def test_every_code_in_every_position():
    for pos in range(8):
        for code in range(16):
            for fill in (0x0, 0x9, 0xF, 0x7):
                w = 0
                for i in range(8):
                    w |= (code if i == pos else fill) << (4 * i)
                check_word(w)


def test_random_words():
    rng = np.random.default_rng(0)
    for w in rng.integers(0, 2 ** 32, size=3000, dtype=np.uint64).tolist():
        check_word(int(w))
