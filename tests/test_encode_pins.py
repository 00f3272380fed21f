"""Pins of the oracle's write side for one new token (oracle/encode_ref.py).

* bf16 rounding against torch's float32 -> bfloat16 conversion (round to nearest
  even), ties and edge values included;
* the fp32 dot products against an exact-rational model of the stated order
  (each product, then each sum, rounded to fp32 from index 0 up);
* exact cases built from unit-vector bases, where every value is known in closed
  form: a token in the span of the basis leaves no residual (codes and scale 0 at
  any rank); a token with components outside it has residual coordinates equal to
  those components, so its codes are the quantiser's on them; the shared
  coefficients are the bf16-rounded mean of the two layers' vectors;
* random orthonormal bases: coefficients and residual coordinates agree with an
  fp64 evaluation of c = B m and u = R (k - B^T c_stored);
* the calibration fit spans the data it was fitted to;
* planted mistakes each fail one of these pins.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle.encode_ref as er
import oracle.quant_ref as qr
from test_quant_pins import f32

RB, D = 32, 128


def bf16_round(x):
    return er.f32_to_bf16_bits(np.asarray(x, np.float32))


def to_bf16_values(x):
    return er.bf16_bits_to_f32(bf16_round(x))


# ----------------------------------------------------------------------------- rounding and order
def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(5000).astype(np.float32) * 10.0 ** rng.integers(-30, 30, 5000),
                        np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -1.0 - 2 ** -8, 2 ** -126, 3.0e38, 0.0, -0.0,
                                  1.00390625, 1.01171875], np.float32)]).astype(np.float32)
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(er.f32_to_bf16_bits(x), want)


def exact_dot(a, x):
    acc = f32(Fraction(float(a[0])) * Fraction(float(x[0])))
    for i in range(1, len(a)):
        acc = f32(acc + f32(Fraction(float(a[i])) * Fraction(float(x[i]))))
    return acc


def check_dot_order(dot=er.dot_rows_f32):
    rng = np.random.default_rng(1)
    A = (rng.standard_normal((6, 40)) * 10.0 ** rng.integers(-3, 4, (6, 40))).astype(np.float32)
    x = (rng.standard_normal(40) * 10.0 ** rng.integers(-3, 4, 40)).astype(np.float32)
    got = dot(A, x)
    for r in range(A.shape[0]):
        assert Fraction(float(got[r])) == exact_dot(A[r], x), r


def test_dot_products_follow_the_stated_fp32_order():
    check_dot_order()


def test_combine_rows_follow_the_stated_fp32_order():
    rng = np.random.default_rng(2)
    c = rng.standard_normal(9).astype(np.float32)
    A = (rng.standard_normal((9, 30)) * 10.0 ** rng.integers(-3, 4, (9, 30))).astype(np.float32)
    got = er.combine_rows_f32(c, A)
    for i in range(A.shape[1]):
        assert Fraction(float(got[i])) == exact_dot(c, A[:, i]), i


# ----------------------------------------------------------------------------- exact cases
def unit_rows(idx, d=D):
    m = np.zeros((len(idx), d), np.float32)
    m[np.arange(len(idx)), idx] = 1.0
    return m


def check_token_in_span(encode=er.encode_pair):
    rng = np.random.default_rng(3)
    B = unit_rows(range(RB))
    R = unit_rows(range(RB, RB + 16))
    k = np.zeros(D, np.float32)
    k[:RB] = to_bf16_values(rng.standard_normal(RB))
    for rank in (0, 8, 16):
        cb, u0, c0, s0, u1, c1, s1 = encode(k, k, B, R, R, rank, rank)
        assert np.array_equal(er.bf16_bits_to_f32(cb), k[:RB])
        for u, c, s in ((u0, c0, s0), (u1, c1, s1)):
            assert np.all(u == 0.0) and np.all(c == 0) and s == 0


def check_components_outside_the_span(encode=er.encode_pair):
    rng = np.random.default_rng(4)
    B = unit_rows(range(RB))
    R = unit_rows(range(RB, RB + 16))
    k0 = to_bf16_values(rng.standard_normal(D))
    k1 = to_bf16_values(rng.standard_normal(D))
    cb, u0, c0, s0, u1, c1, s1 = encode(k0, k1, B, R, R, 8, 16)
    mean = ((k0[:RB].astype(np.float64) + k1[:RB]) / 2).astype(np.float32)      # exact: bf16 + bf16 fits fp32
    assert np.array_equal(cb, bf16_round(mean))
    assert np.array_equal(u0, k0[RB:RB + 16]) and np.array_equal(u1, k1[RB:RB + 16])
    want0 = qr.quantize(k0[None, RB:RB + 16], np.array([8]))
    want1 = qr.quantize(k1[None, RB:RB + 16], np.array([16]))
    assert np.array_equal(c0, want0[0][0]) and s0 == want0[1][0]
    assert np.array_equal(c1, want1[0][0]) and s1 == want1[1][0]


def check_residual_sees_the_stored_coefficients(encode=er.encode_pair):
    """A residual row on a basis coordinate sees k - c_stored there, the bf16 rounding included."""
    B = unit_rows(range(RB))
    R = unit_rows([0] + list(range(RB, RB + 15)))
    k0 = np.zeros(D, np.float32)
    k1 = np.zeros(D, np.float32)
    k0[0], k1[0] = 1.0, 1.0 + 2 ** -7           # mean 1 + 2^-8: a bf16 tie, rounds to 1.0
    cb, u0, _, _, u1, _, _ = encode(k0, k1, B, R, R, 16, 16)
    assert er.bf16_bits_to_f32(cb)[0] == 1.0
    assert u0[0] == 0.0 and u1[0] == np.float32(2 ** -7)


def test_token_in_the_span_leaves_no_residual():
    check_token_in_span()


def test_components_outside_the_span_are_the_residual():
    check_components_outside_the_span()


def test_residual_is_taken_against_the_stored_coefficients():
    check_residual_sees_the_stored_coefficients()


# ----------------------------------------------------------------------------- random orthonormal bases
def random_orthonormal(rng, rows, d=D):
    q, _ = np.linalg.qr(rng.standard_normal((d, rows)))
    return q.T


def test_random_bases_agree_with_fp64():
    rng = np.random.default_rng(5)
    for trial in range(5):
        W = random_orthonormal(rng, RB + 32)
        B = to_bf16_values(W[:RB])
        R0 = to_bf16_values(W[RB:RB + 16])
        R1 = to_bf16_values(W[RB + 16:RB + 32])
        k0 = to_bf16_values(rng.standard_normal(D))
        k1 = to_bf16_values(k0 + 0.3 * rng.standard_normal(D))
        cb, u0, _, _, u1, _, _ = er.encode_pair(k0, k1, B, R0, R1, 16, 16)
        m = (k0.astype(np.float64) + k1) / 2
        c64 = B.astype(np.float64) @ m
        c = er.bf16_bits_to_f32(cb).astype(np.float64)
        assert np.max(np.abs(c - c64)) <= 2 ** -8 * np.max(np.abs(c64)) + 1e-6
        for k, R, u in ((k0, R0, u0), (k1, R1, u1)):
            e = k.astype(np.float64) - B.astype(np.float64).T @ c
            u64 = R.astype(np.float64) @ e
            assert np.max(np.abs(u - u64)) <= 1e-5 * (np.max(np.abs(u64)) + 1)


def test_calibration_fit_spans_its_window():
    rng = np.random.default_rng(6)
    basis = random_orthonormal(rng, RB)
    K0 = rng.standard_normal((200, RB)) @ basis
    K1 = rng.standard_normal((200, RB)) @ basis
    V = er.fit_pair_basis(K0, K1, RB)
    assert np.allclose(V @ V.T, np.eye(RB), atol=1e-12)
    X = np.concatenate([K0, K1])
    assert np.allclose(X @ V.T @ V, X, atol=1e-10)


# ----------------------------------------------------------------------------- planted mistakes
def test_pins_catch_planted_mistakes(monkeypatch):
    def fma_dot(A, x):      # one rounding per term instead of two
        A = np.asarray(A, np.float64)
        acc = np.float32(0) * np.zeros(A.shape[0], np.float32)
        for i in range(A.shape[1]):
            acc = (acc.astype(np.float64) + A[:, i] * float(x[i])).astype(np.float32)
        return acc
    with pytest.raises(AssertionError):
        check_dot_order(fma_dot)

    def sum_not_mean(k0, k1, basis, r0, r1, rank0, rank1):
        return er.encode_pair(np.asarray(k0) * 2, np.asarray(k1) * 0, basis, r0, r1, rank0, rank1)
    with pytest.raises(AssertionError):
        check_components_outside_the_span(sum_not_mean)

    def first_layer_twice(k0, k1, basis, r0, r1, rank0, rank1):
        return er.encode_pair(k0, k0, basis, r0, r1, rank0, rank1)
    with pytest.raises(AssertionError):
        check_components_outside_the_span(first_layer_twice)

    orig_round = er.f32_to_bf16_bits
    monkeypatch.setattr(er, "f32_to_bf16_bits", lambda x: (np.asarray(x, np.float32).view(np.uint32) >> 16).astype(np.uint16))
    with pytest.raises(AssertionError):
        test_bf16_rounding_matches_torch()
    monkeypatch.setattr(er, "f32_to_bf16_bits", orig_round)

    def unrounded_residual(k0, k1, basis, r0, r1, rank0, rank1):
        k0 = np.asarray(k0, np.float32)
        k1 = np.asarray(k1, np.float32)
        m = ((k0 + k1) * np.float32(0.5)).astype(np.float32)
        c = er.dot_rows_f32(basis, m)
        rebuilt = er.combine_rows_f32(c, basis)
        out = [er.f32_to_bf16_bits(c)]
        for k, R, rank in ((k0, r0, rank0), (k1, r1, rank1)):
            u = er.dot_rows_f32(R, (k - rebuilt).astype(np.float32))
            codes, scale = qr.quantize(u[None, :], np.array([rank]))
            out += [u, codes[0], scale[0]]
        return tuple(out)
    with pytest.raises(AssertionError):
        check_residual_sees_the_stored_coefficients(unrounded_residual)
