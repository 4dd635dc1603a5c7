"""The algebra behind the INT4 decode of the streaming FFN, checked exactly on
the CPU (no GPU code involved).

The kernel turns a two's-complement code q in [-8, 7] into the fp16 integer
1024 + (q + 8) when it sits in an even nibble and 1024 + 16 (q + 8) in an odd
one; the activations that meet odd nibbles are divided by 16 beforehand (a
power of two), and per 128-wide scale group the constant
    1032 * sum_{even k} h_k + 1152 * sum_{odd k} h_k
(h = the stored fp16 activations) is subtracted from the group's dot product.
What is left must be sum_k x_k q_k exactly (before fp32 rounding), and every
offset value must be exactly representable in fp16.
"""
import numpy as np
import pytest


def _offset_f16(q, odd):
    u = q + 8
    return np.where(odd, 1024 + 16 * u, 1024 + u).astype(np.float64)


def test_offset_values_are_exact_fp16():
    q = np.arange(-8, 8)
    for odd in (False, True):
        v = _offset_f16(q, np.full(q.shape, odd))
        assert np.array_equal(v.astype(np.float16).astype(np.float64), v)
        # the bit pattern the kernel builds: 0x6400 | (u << 4 * odd)
        bits = (0x6400 | ((q + 8) << (4 if odd else 0))).astype(np.uint16)
        assert np.array_equal(bits.view(np.float16).astype(np.float64), v)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_group_constant_recovers_dot_product(seed):
    rng = np.random.default_rng(seed)
    K = 128
    for trial in range(50):
        q = rng.integers(-8, 8, size=K)
        # activations as the prep kernel stores them: fp16, odd K divided by 16
        x = rng.standard_normal(K) * (2.0 ** rng.integers(-6, 10))
        if trial % 5 == 0:
            x = np.abs(x) + 1.0  # no cancellation inside the constant
        x16 = x.astype(np.float16).astype(np.float64)
        odd = (np.arange(K) % 2) == 1
        h = np.where(odd, (x16 / 16).astype(np.float16).astype(np.float64), x16)
        mma = np.sum(h * _offset_f16(q, odd))  # exact in fp64 at these sizes
        const = 1032.0 * h[~odd].sum() + 1152.0 * h[odd].sum()
        ref = np.sum(np.where(odd, 16 * h, h) * q)
        assert mma - const == pytest.approx(ref, rel=0, abs=1e-9 * max(1.0, np.abs(h).sum() * 2048))
