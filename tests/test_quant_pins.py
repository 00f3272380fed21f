"""Pins of the rank router and the int8 residual quantiser of the oracle.

The rule is defined in fp32 with correctly rounded operations (see
oracle/quant_ref.py). It is checked against:
* hand-derived examples in tests/golden/quant_examples.jsonl;
* an exact-rational model of IEEE rounding (fractions.Fraction), independent of
  numpy's float32 and float16 arithmetic, on random and adversarial inputs;
* invariants: the largest kept magnitude maps to +-127, codes beyond the rank are
  zero, dequantisation error is at most half a step for unclamped codes.
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle.quant_ref as qr

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "quant_examples.jsonl")


# ----------------------------------------------------------------------------- exact IEEE model
def _round_half_even(x: Fraction) -> int:
    n = x.numerator // x.denominator
    rem = x - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    return n


def _rne_float(x: Fraction, mant_bits: int, emin: int, emax_finite: Fraction):
    """Round a rational to a binary format with ``mant_bits`` fraction bits (nearest even)."""
    if x == 0:
        return Fraction(0)
    sgn = -1 if x < 0 else 1
    a = abs(x)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    e = max(e, emin)
    q = Fraction(2) ** (e - mant_bits)
    r = _round_half_even(a / q) * q
    if r > emax_finite:
        return Fraction(sgn) * Fraction(10) ** 400          # overflow marker (inf)
    return sgn * r


def f32(x: Fraction) -> Fraction:
    return _rne_float(x, 23, -126, Fraction(2) ** 127 * (2 - Fraction(1, 2 ** 23)))


def f16(x: Fraction) -> Fraction:
    return _rne_float(x, 10, -14, Fraction(65504))


def exact_quantize(u, rank):
    u = [Fraction(float(np.float32(v))) for v in u]
    amax = max([abs(v) for v in u[:rank]], default=Fraction(0))
    s32 = min(f32(amax / 127), Fraction(65504))
    s = f16(s32)
    codes = []
    for i, v in enumerate(u):
        if i >= rank or s == 0:
            codes.append(0)
        else:
            codes.append(max(-127, min(127, _round_half_even(f32(v / s)))))
    return s, codes


def f16_value(bits: int) -> Fraction:
    return Fraction(float(np.array([bits], dtype=np.uint16).view(np.float16)[0]))


# ----------------------------------------------------------------------------- golden
def load_golden():
    with open(GOLDEN) as f:
        return [json.loads(line) for line in f if line.strip()]


def parse(v: str) -> float:
    return float.fromhex(v) if v.startswith(("0x", "-0x")) else float(v)


@pytest.mark.parametrize("case", load_golden(), ids=lambda c: c["case"])
def test_golden_examples(case):
    u = np.array([parse(v) for v in case["u"]], dtype=np.float32)
    codes, scale = qr.quantize(u[None], np.array([case["rank"]]))
    assert int(scale[0]) == int(case["scale_bits"], 16)
    assert codes[0].tolist() == case["codes"]
    s, c = exact_quantize(u, case["rank"])            # the exact model agrees with the fixture too
    assert s == f16_value(int(case["scale_bits"], 16)) and c == case["codes"]


def test_router_thresholds_exact():
    f = np.float32
    s = np.array([0.0, np.nextafter(f(0.7), f(0)), f(0.7), np.nextafter(f(0.9), f(0)), f(0.9),
                  np.nextafter(f(1.0), f(0))], dtype=np.float32)
    assert qr.route_rank(s).tolist() == [0, 0, 8, 8, 16, 16]


def test_router_rates_on_uniform_scores():
    u = (np.arange(1 << 24, dtype=np.float64) * 2.0 ** -24).astype(np.float32)   # every 24-bit uniform
    r = qr.route_rank(u)
    frac = [np.mean(r == k) for k in (0, 8, 16)]
    assert abs(frac[0] - 0.7) < 1e-6 and abs(frac[1] - 0.2) < 1e-6 and abs(frac[2] - 0.1) < 1e-6


def test_quantizer_matches_exact_rational_model():
    g = np.random.default_rng(5)
    rows = []
    for _ in range(300):
        scale = 10.0 ** g.uniform(-9, 6)
        rows.append((g.standard_normal(16) * scale).astype(np.float32))
    # adversarial rows: exact ties, huge/tiny magnitudes, repeated extremes
    rows.append(np.array([127, 0.5, 1.5, 2.5, -0.5, -1.5, 126.5, -126.5] + [0] * 8, np.float32) * np.float32(2 ** -9))
    rows.append(np.array([3e-8, 1e-8, -2e-8] + [0] * 13, np.float32))
    rows.append(np.array([1e30, -1e30] + [1.0] * 14, np.float32))
    U = np.stack(rows)
    for rank in (0, 8, 16):
        codes, scales = qr.quantize(U, np.full(U.shape[0], rank))
        for i in range(U.shape[0]):
            s, c = exact_quantize(U[i], rank)
            assert f16_value(int(scales[i])) == s, (i, rank)
            assert codes[i].tolist() == c, (i, rank)


def test_quantizer_invariants():
    g = np.random.default_rng(6)
    U = (g.standard_normal((2000, 16)) / 4).astype(np.float32)
    rank = g.choice([0, 8, 16], size=2000)
    codes, scales = qr.quantize(U, rank)
    s = scales.view(np.float16).astype(np.float64)
    for i in range(2000):
        r = rank[i]
        assert np.all(codes[i, r:] == 0)
        if r == 0:
            assert s[i] == 0
            continue
        k = np.argmax(np.abs(U[i, :r]))
        assert abs(int(codes[i, k])) == 127 and np.sign(codes[i, k]) == np.sign(U[i, k])
        err = np.abs(codes[i, :r] * s[i] - U[i, :r])
        assert np.all(err <= 0.5 * s[i] * (1 + 1e-6) + 1e-12 + np.abs(U[i, :r]) * 2 ** -10)


def test_pack_shares_rank_across_heads_and_kv():
    g = np.random.default_rng(7)
    score = g.uniform(size=(2, 1, 50)).astype(np.float32)
    uk = g.standard_normal((2, 1, 3, 50, 16)).astype(np.float32)
    uv = g.standard_normal((2, 1, 3, 50, 16)).astype(np.float32)
    rank, ck, cv, sk, sv = qr.pack_residual(score, uk, uv)
    assert rank.shape == (2, 1, 50) and ck.shape == uk.shape and sk.shape == (2, 1, 3, 50)
    for h in range(3):
        c1, s1 = qr.quantize(uk[:, :, h], rank)
        assert np.array_equal(c1, ck[:, :, h]) and np.array_equal(s1, sk[:, :, h])
        c2, s2 = qr.quantize(uv[:, :, h], rank)
        assert np.array_equal(c2, cv[:, :, h]) and np.array_equal(s2, sv[:, :, h])


def test_planted_rounding_mistake_is_caught(monkeypatch):
    """Rounding half away from zero instead of half to even fails the golden tie case."""
    case = [c for c in load_golden() if c["case"].startswith("ties")][0]
    monkeypatch.setattr(qr.np, "rint", lambda x: np.sign(x) * np.floor(np.abs(x) + 0.5))
    u = np.array([parse(v) for v in case["u"]], dtype=np.float32)
    codes, _ = qr.quantize(u[None], np.array([case["rank"]]))
    assert codes[0].tolist() != case["codes"]
