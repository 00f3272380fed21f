"""The seeded generator: Philox known answers, series accuracy, distribution, slicing."""
import math

import numpy as np
import pytest

from synth import philox
from synth.configs import PRESETS, BY_NAME


# Known-answer vectors published with the Random123 library for philox4x32-10.
KAT = [
    ((0, 0, 0, 0), (0, 0), (0x6627e8d5, 0xe169c58d, 0xbc57ac4c, 0x9b00dbd8)),
    ((0xffffffff,) * 4, (0xffffffff,) * 2, (0x408f276d, 0x41c83b0e, 0xa20bc7c6, 0x6d5451fd)),
    ((0x243f6a88, 0x85a308d3, 0x13198a2e, 0x03707344), (0xa4093822, 0x299f31d0),
     (0xd16cfe09, 0x94fdcceb, 0x5001e420, 0x24126ea1)),
]


@pytest.mark.parametrize("ctr,key,expect", KAT)
def test_philox_known_answers(ctr, key, expect):
    out = philox.philox4x32_10(*[np.array([c], dtype=np.uint64) for c in ctr], *key)
    assert tuple(int(o[0]) for o in out) == expect


def test_series_log_matches_libm():
    w = philox.raw_words(20000, 0, 11, 1)
    w = np.concatenate([w, np.array([0, 1, 2, 0x7fffffff, 0xb504f333, 0xfffffffe, 0xffffffff], np.uint64)])
    got = philox.series_log_u32(w)
    ref = np.array([math.log((int(x) + 1) * 2.0 ** -32) for x in w])
    assert np.max(np.abs(got - ref) / np.maximum(np.abs(ref), 1e-300)) < 2e-15
    assert got[-1] == 0.0                       # ln 1


def test_series_sincos_matches_libm():
    w = philox.raw_words(20000, 0, 11, 2)
    w = np.concatenate([w, np.array([0, 1 << 30, 2 << 30, 3 << 30, 0xffffffff], np.uint64)])
    c, s = philox.series_sincos_u32(w)
    th = np.array([2 * math.pi * int(x) * 2.0 ** -32 for x in w])
    assert np.max(np.abs(c - np.cos(th))) < 2e-15
    assert np.max(np.abs(s - np.sin(th))) < 2e-15
    assert np.max(np.abs(c * c + s * s - 1)) < 4e-15


def test_normal_moments_and_independence():
    z = philox.normal_f64(1 << 19, 0, 20261202, 3)
    n = z.size
    assert abs(z.mean()) < 5 / math.sqrt(n)
    assert abs(z.var() - 1) < 5 * math.sqrt(2 / n)
    assert abs(np.mean(z ** 3)) < 5 * math.sqrt(15 / n)
    assert abs(np.mean(z ** 4) - 3) < 5 * math.sqrt(96 / n)
    # the cos and sin halves of a Box-Muller pair are uncorrelated
    assert abs(np.mean(z[0::2] * z[1::2])) < 5 / math.sqrt(n / 2)
    # fraction within one sigma
    assert abs(np.mean(np.abs(z) < 1) - 0.6826894921370859) < 5 * math.sqrt(0.25 / n)


def test_uniform_range_and_mean():
    u = philox.uniform_f32((1 << 18,), 5, 4)
    assert u.dtype == np.float32 and u.min() >= 0 and u.max() < 1
    assert abs(u.mean() - 0.5) < 5 * math.sqrt(1 / 12 / u.size)
    # exactly 24 random bits: every value is a multiple of 2**-24
    assert np.all(np.floor(u.astype(np.float64) * 2 ** 24) == u.astype(np.float64) * 2 ** 24)


def test_bf16_rounding_is_nearest_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -8 + 2 ** -20, -2.5, 0.0],
                 dtype=np.float32)
    got = philox.bf16_bits_to_f64(philox.f32_bits_to_bf16_bits(x))
    assert list(got) == [1.0, 1.0, 1.0 + 4 * 2 ** -8, 1.0 + 2 ** -7, -2.5, 0.0]


def test_slices_equal_full_draws():
    full = philox.normal((3, 4, 5, 6), 9, 2, 0.5, "bf16")
    assert np.array_equal(full[2, 1], philox.normal_slice((3, 4, 5, 6), (2, 1), 9, 2, 0.5, "bf16"))
    assert np.array_equal(full[1:3, :, 4], philox.normal_slice((3, 4, 5, 6), (slice(1, 3), slice(None), 4),
                                                               9, 2, 0.5, "bf16"))
    f32 = philox.normal((7, 9), 9, 5, 1.0, "f32")
    assert np.array_equal(f32[3], philox.normal_slice((7, 9), (3,), 9, 5, 1.0, "f32"))
    u = philox.uniform_f32((4, 33), 9, 6)
    assert np.array_equal(u[1, 3:20], philox.uniform_slice((4, 33), (1, slice(3, 20)), 9, 6))


def test_offsets_continue_the_stream():
    a = philox.normal_f64(37, 0, 1, 1)
    b = philox.normal_f64(30, 7, 1, 1)
    assert np.array_equal(a[7:], b)


def test_presets_match_the_workloads():
    c0, c1, c2, c3, c4, c5 = PRESETS
    assert (c0.layers, c0.q_heads, c0.kv_heads, c0.head_dim, c0.batch, c0.context, c0.dtype) == \
        (4, 4, 2, 64, 1, 128, "f32")
    assert [m[1] for m in c0.layer_map] == [0, 0, 1, 1]
    assert (c1.layers, c1.slots, c1.q_heads, c1.kv_heads, c1.head_dim, c1.batch, c1.context) == \
        (22, 11, 32, 4, 64, 32, 2048)
    assert c1.qkv_scale == 1 / math.sqrt(64)
    assert c2.layer_map[16 + 3] == (1, 3, 11) and all(c2.layer_map[l] == (0, l, 0) for l in range(16))
    assert c3.layer_map == c2.layer_map and c3.mode == "prefill" and c3.context == 4096
    assert (c4.layers, c4.pairs, c4.q_heads, c4.kv_heads, c4.context) == (32, 16, 32, 8, 65536)
    assert BY_NAME["depthweave_decode"] is c4
    assert c5.layer_map == c4.layer_map and c5.mode == "prefill" and (c5.q_heads, c5.kv_heads) == (32, 8)
    assert len({c.seed for c in PRESETS}) == 6
