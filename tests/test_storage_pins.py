"""Pins of the oracle's storage decoders to the IEEE formats themselves.

The cache holds bf16 values (coefficients, bases, factors, K/V) and fp16
per-token residual scales ("DepthWeave-KV: Smarter KV Cache Compression by
Sharing Across Layers and Adapting Per Token", Core Mechanism diagram: a
quantised low-rank residual beside a shared basis; the 16-bit storage types are
this library's reading). The oracle turns their bit patterns into exact fp64
values with ``bf16_bits_to_f64`` and ``f16_bits_to_f64``. Each expected value
below follows from the format's definition alone (sign, biased exponent,
fraction), written as a power of two, never through the decoder under test:

* bf16: 1 sign bit, 8 exponent bits (bias 127), 7 fraction bits; subnormals at
  exponent 0 are fraction * 2^-133.
* fp16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits; subnormals at
  exponent 0 are fraction * 2^-24.

Planted mistakes (a shift of 8 instead of 16, fp16 bits read as bf16 and the
other way round, a dropped sign) each fail these pins.
"""
import math

import numpy as np
import pytest

import oracle.kvshare_ref as ref

BF16_CASES = [
    (0x3F80, 1.0),
    (0xC000, -2.0),
    (0x0001, 2.0 ** -133),                          # smallest subnormal
    (0x007F, 127 * 2.0 ** -133),                    # largest subnormal
    (0x0080, 2.0 ** -126),                          # smallest normal
    (0x7F7F, (2 - 2.0 ** -7) * 2.0 ** 127),         # largest finite
    (0x3E00, 0.125),
    (0x3FC0, 1.5),
    (0x4049, (1 + 73 / 128) * 2.0),                 # 3.140625
    (0xBF81, -(1 + 1 / 128)),
    (0x8000, -0.0),
    (0x0000, 0.0),
]

F16_CASES = [
    (0x3C00, 1.0),
    (0x0001, 2.0 ** -24),                           # smallest subnormal
    (0x03FF, 1023 * 2.0 ** -24),                    # largest subnormal
    (0x0400, 2.0 ** -14),                           # smallest normal
    (0x7BFF, 65504.0),                              # largest finite
    (0x8400, -(2.0 ** -14)),
    (0x3555, (1 + 341 / 1024) * 2.0 ** -2),         # closest fp16 to 1/3
    (0xC500, -5.0),
    (0x1C00, 2.0 ** -8),
    (0x8000, -0.0),
]


def decode_rule_bf16(bits):
    """The bf16 value of a 16-bit pattern, from sign, exponent and fraction fields."""
    s, e, f = bits >> 15, (bits >> 7) & 0xFF, bits & 0x7F
    mag = f * 2.0 ** -133 if e == 0 else (1 + f / 128) * 2.0 ** (e - 127)
    return -mag if s else mag


def decode_rule_f16(bits):
    s, e, f = bits >> 15, (bits >> 10) & 0x1F, bits & 0x3FF
    mag = f * 2.0 ** -24 if e == 0 else (1 + f / 1024) * 2.0 ** (e - 15)
    return -mag if s else mag


def check_bf16(fn):
    bits = np.array([b for b, _ in BF16_CASES], dtype=np.uint16)
    got = fn(bits)
    for (b, want), g in zip(BF16_CASES, got):
        assert g == want and math.copysign(1.0, g) == math.copysign(1.0, want), hex(b)


def check_f16(fn):
    bits = np.array([b for b, _ in F16_CASES], dtype=np.uint16)
    got = fn(bits)
    for (b, want), g in zip(F16_CASES, got):
        assert g == want and math.copysign(1.0, g) == math.copysign(1.0, want), hex(b)


def check_all_finite_patterns(fn, rule, exp_mask):
    """Every finite pattern (both signs) against the field-by-field rule."""
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    finite = (bits & exp_mask) != exp_mask
    got = fn(bits[finite])
    want = np.array([rule(int(b)) for b in bits[finite]])
    assert np.array_equal(got, want)


def test_bf16_known_patterns():
    check_bf16(ref.bf16_bits_to_f64)


def test_f16_known_patterns():
    check_f16(ref.f16_bits_to_f64)


def test_bf16_every_finite_pattern():
    check_all_finite_patterns(ref.bf16_bits_to_f64, decode_rule_bf16, 0x7F80)


def test_f16_every_finite_pattern():
    check_all_finite_patterns(ref.f16_bits_to_f64, decode_rule_f16, 0x7C00)


def test_to_f64_dispatches_on_the_storage_tag():
    assert ref.to_f64(np.array([0x3F80], np.uint16), "bf16")[0] == 1.0
    assert ref.to_f64(np.array([0.1], np.float32), "f32")[0] == float(np.float32(0.1))


# ---------------------------------------------------------------- planted mistakes
def shift8(bits):
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(8)
    return b.view(np.float32).astype(np.float64)


def drop_sign_bf16(bits):
    return np.abs(ref.bf16_bits_to_f64(bits))


@pytest.mark.parametrize("wrong,check", [
    (shift8, check_bf16),                       # shift of 8 instead of 16
    (ref.f16_bits_to_f64, check_bf16),          # bf16 bits read as fp16
    (drop_sign_bf16, check_bf16),               # sign dropped
    (ref.bf16_bits_to_f64, check_f16),          # fp16 scales read as bf16
    (lambda b: np.abs(ref.f16_bits_to_f64(b)), check_f16),
], ids=["bf16_shift8", "bf16_as_f16", "bf16_no_sign", "f16_as_bf16", "f16_no_sign"])
def test_pins_catch_planted_decoder_mistakes(wrong, check):
    with pytest.raises(AssertionError):
        check(wrong)
