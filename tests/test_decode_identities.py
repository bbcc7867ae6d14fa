"""The bf16 identities the decode kernels' code-to-operand conversion rests on, checked on the CPU.

A bf16 in [128, 256) has exponent 2^7 and 7 mantissa bits worth 1 each, so the bits
0x4300 | (q << p) encode 128 + q 2^p whenever the code's bits stay inside bits 0..6.  The
kernels build their MMA operands that way: 4-bit codes at p = 0; 2-bit codes at p = 0, 2, 4
with the paired activations scaled by 1, 1/4, 1/16; 3-bit codes at p = 0, 3 (scales 1, 1/8);
8-bit codes as a low nibble at p = 0 and a high nibble at p = 3 against a doubled activation.
The GPU parity tests check the kernels themselves; these pin the arithmetic they assume.
"""
import numpy as np
import pytest
import torch


def bf16_value(bits):
    return torch.tensor(np.asarray(bits, np.int32).astype(np.int16)).view(torch.bfloat16).double().numpy()


def bf16_round(x):
    return torch.tensor(np.asarray(x, np.float32)).to(torch.bfloat16).double().numpy()


@pytest.mark.parametrize("width,positions", [(4, [0]), (2, [0, 2, 4]), (3, [0, 3]), (4, [3])])
def test_codes_at_mantissa_positions_encode_128_plus_scaled_code(width, positions):
    q = np.arange(1 << width)
    for p in positions:
        assert p + width <= 7
        assert np.array_equal(bf16_value(0x4300 | (q << p)), 128.0 + q * 2.0 ** p)


@pytest.mark.parametrize("scale", [1.0, 0.25, 0.0625, 0.125])
def test_power_of_two_activation_scaling_is_exact_and_products_undo_it(scale):
    """(128 + s q)(a / s) = 128 a / s + q a exactly in fp32 for bf16 a (products of two bf16 are
    exact in fp32), and a / s itself is exact in bf16 (a power-of-two scaling of a normal value)."""
    rng = np.random.default_rng(3)
    a = bf16_round(rng.standard_normal(4096) * 3.0)
    a_s = bf16_round(a * scale)
    assert np.array_equal(a_s, a * scale)
    s_code = 1.0 / scale
    for q in range(8):
        w = 128.0 + s_code * q
        if w >= 256:
            continue
        prod = (np.float32(w) * a_s.astype(np.float32)).astype(np.float64)
        assert np.array_equal(prod, w * a_s)
        assert np.array_equal(prod, 128.0 * a_s + q * a)  # 128 a / s + q a when s_code = 1 / scale


def test_eight_bit_code_as_two_nibbles_gives_384_a_plus_q_a():
    """Low nibble (128 + lo) against a, high nibble at bits 3..6 (128 + 8 hi) against 2a: the two
    products add to 384 a + (16 hi + lo) a = 384 a + q a, every step exact."""
    rng = np.random.default_rng(8)
    a = bf16_round(rng.standard_normal(256) * 2.0)
    q = np.arange(256)
    lo, hi = q & 15, q >> 4
    x = q | (q << 16)  # a code in each half of a 32-bit word, as the kernel sees two codes
    lo_bits = (x & 0x000F000F) | 0x43004300
    hi_bits = ((x >> 1) & 0x00780078) | 0x43004300
    assert np.array_equal(bf16_value(lo_bits & 0xFFFF), 128.0 + lo)
    assert np.array_equal(bf16_value(hi_bits & 0xFFFF), 128.0 + 8 * hi)
    assert np.array_equal(bf16_value(hi_bits >> 16), 128.0 + 8 * hi)
    total = (128.0 + lo) * a + (128.0 + 8 * hi) * (2 * a)
    assert np.array_equal(total, 384.0 * a + q * a)
