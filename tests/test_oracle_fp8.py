"""Pins of the oracle's FP8 block-scaled weight dequantisation ("DeepSeek-V3.2-Exp · Attention
update", mla-decode: weight_dequant(wkv_b.weight, wkv_b.scale) gives the bf16 weight the
absorbed decode uses).  No GPU needed."""
import numpy as np
import pytest

import oracle


def test_e4m3_closed_forms():
    v = oracle.fp8_e4m3_value
    assert v(0x38) == 1.0                      # exponent 7 (bias 7), mantissa 0
    assert v(0xB8) == -1.0
    assert v(0x7E) == 448.0                    # largest finite: 1.75 * 2^8
    assert v(0x08) == 2.0 ** -6                # smallest normal
    assert v(0x01) == 2.0 ** -9                # smallest subnormal: 1/8 * 2^-6
    assert v(0x07) == 7 * 2.0 ** -9
    assert v(0x00) == 0.0 and np.signbit(v(0x80))
    assert v(0x3C) == 1.5 and v(0x40) == 2.0
    assert np.isnan(v(0x7F)) and np.isnan(v(0xFF))


def test_e4m3_all_codes_match_torch():
    import torch
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = oracle.fp8_e4m3_value(codes)
    np.testing.assert_array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    np.testing.assert_array_equal(got[ok], ref[ok])


def test_e4m3_values_are_monotone_in_the_code():
    v = oracle.fp8_e4m3_value(np.arange(0x7F))
    assert np.all(np.diff(v) > 0)


def test_block_scales_apply_per_128_block():
    rng = np.random.default_rng(8)
    bits = rng.integers(0, 0x7E, (256, 384)).astype(np.uint8)   # finite positive codes
    scale = np.ones((2, 3))
    base = oracle.dequant_block_fp8(bits, scale)
    np.testing.assert_array_equal(base, oracle.round_bf16(oracle.fp8_e4m3_value(bits)))
    scale[1, 2] = 0.25                                          # a power of two: exact
    w = oracle.dequant_block_fp8(bits, scale)
    np.testing.assert_array_equal(w[128:, 256:], base[128:, 256:] * 0.25)
    np.testing.assert_array_equal(w[:128], base[:128])
    np.testing.assert_array_equal(w[128:, :256], base[128:, :256])


def test_dequant_rounds_the_scaled_product_to_bf16():
    bits = np.full((1, 1), 0x39, np.uint8)                      # 1.125
    w = oracle.dequant_block_fp8(bits, np.array([[1.0 + 2.0 ** -10]]))
    assert w[0, 0] == 1.125                                     # 1.125*(1+2^-10) rounds back
    assert oracle.round_bf16(np.array(1.125 * (1 + 2.0 ** -10))) == 1.125
