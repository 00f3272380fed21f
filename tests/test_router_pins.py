"""Pins of the oracle's attention statistics, router score and per-sequence lengths.

* closed forms: equal keys give uniform weights (entropy ln T, peak 1/T, mass
  g/T per token); one dominant key gives entropy 0 and peak 1; two tokens give
  the logistic weight and its binary entropy, computed here as lse - sum p z;
* conservation: each kv head's masses sum to g over the tokens;
* brute force at 50 digits (mpmath, pure-Python loops) on tiny inputs;
* the fp32 router score against an exact-rational model of IEEE rounding, its
  monotonicity and the uniform-share point;
* per-sequence lengths: decode over a sequence's first n tokens equals torch's
  SDPA with a key mask (fp64), length 0 gives 0 and -inf, the full length equals
  no lengths at all, and nothing past the length matters;
* planted mistakes each fail one of these pins.
"""
import math
from fractions import Fraction

import mpmath
import numpy as np
import pytest
import torch

import oracle.kvshare_ref as ref
import oracle.quant_ref as qr
import oracle.router_ref as rr
from test_quant_pins import f32

SINGLE = ref.SINGLE


def group_p(q, K, scale=None):
    d = K.shape[1]
    _, _, p = ref.attend(q, K, np.zeros_like(K), 1 / math.sqrt(d) if scale is None else scale)
    return p


# ----------------------------------------------------------------------------- closed forms
def check_uniform(stats=rr.attention_stats, mass=rr.kv_mass):
    T, g = 37, 4
    K = np.tile(np.random.default_rng(0).standard_normal((1, 16)), (T, 1))
    q = np.random.default_rng(1).standard_normal((g, 16))
    p = group_p(q, K)
    e, pk = stats(p)
    assert np.allclose(e, math.log(T), rtol=0, atol=1e-13)
    assert np.allclose(pk, 1.0 / T, rtol=1e-14)
    assert np.allclose(mass(p, g), g / T, rtol=1e-13)


def check_dominant(stats=rr.attention_stats):
    T = 9
    K = np.zeros((T, 4))
    K[5] = [100.0, 0, 0, 0]
    q = np.array([[40.0, 0, 0, 0]])
    p = group_p(q, K, scale=1.0)     # score gap 4000: every other weight is exp(-4000) = 0
    e, pk = stats(p)
    assert abs(e[0]) < 1e-12 and pk[0] == 1.0


def check_two_tokens(stats=rr.attention_stats):
    for dz in (-3.0, -0.25, 0.0, 0.7, 5.0):
        z = np.array([[0.3, 0.3 + dz]])
        p = np.exp(z - z.max()) / np.exp(z - z.max()).sum()
        lse = z.max() + math.log(np.exp(z - z.max()).sum())
        want = lse - float(np.sum(p * z))                       # -sum p ln p = lse - sum p z
        e, pk = stats(p)
        assert abs(e[0] - want) < 1e-14
        assert abs(pk[0] - 1.0 / (1.0 + math.exp(-abs(dz)))) < 1e-15


def test_uniform_attention():
    check_uniform()


def test_one_dominant_key():
    check_dominant()


def test_two_tokens_binary_entropy():
    check_two_tokens()


def test_masses_sum_to_the_group_size():
    rng = np.random.default_rng(5)
    Hq, g, T = 12, 3, 50
    p = np.concatenate([group_p(rng.standard_normal((g, 8)), rng.standard_normal((T, 8))) for _ in range(Hq // g)])
    m = rr.kv_mass(p, g)
    assert m.shape == (Hq // g, T)
    assert np.allclose(m.sum(axis=1), g, atol=1e-12)
    # each kv head's mass comes from its own contiguous group of heads only
    for j in range(Hq // g):
        assert np.allclose(m[j], p[j * g:(j + 1) * g].sum(axis=0), atol=0)


# ----------------------------------------------------------------------------- brute force
def brute_stats(q, K, scale):
    """Entropy, peak and mass at 50 digits with pure-Python loops."""
    mpmath.mp.dps = 50
    n, T = len(q), len(K)
    ent, peak, mass = [], [], [mpmath.mpf(0)] * T
    for i in range(n):
        z = [mpmath.fsum(mpmath.mpf(float(q[i][c])) * mpmath.mpf(float(K[t][c])) for c in range(len(K[t]))) *
             mpmath.mpf(scale) for t in range(T)]
        den = mpmath.fsum(mpmath.exp(x) for x in z)
        p = [mpmath.exp(x) / den for x in z]
        ent.append(-mpmath.fsum(x * mpmath.log(x) for x in p))
        peak.append(max(p))
        mass = [a + b for a, b in zip(mass, p)]
    return [float(x) for x in ent], [float(x) for x in peak], [float(x) for x in mass]


def test_brute_force_statistics():
    rng = np.random.default_rng(11)
    for trial in range(4):
        g, T, d = 1 + trial % 3, 3 + trial * 2, 5
        q = rng.standard_normal((g, d)) * 2
        K = rng.standard_normal((T, d))
        sc = 1 / math.sqrt(d)
        e, pk = rr.attention_stats(group_p(q, K, sc))
        m = rr.kv_mass(group_p(q, K, sc), g)[0]
        be, bp, bm = brute_stats(q.tolist(), K.tolist(), sc)
        assert np.allclose(e, be, rtol=1e-12, atol=1e-14)
        assert np.allclose(pk, bp, rtol=1e-12)
        assert np.allclose(m, bm, rtol=1e-12, atol=1e-15)


def test_decode_stats_matches_per_group_statistics():
    rng = np.random.default_rng(2)
    L, B, Hq, Hkv, T, d = 2, 2, 6, 2, 11, 8
    cache = {"k": rng.standard_normal((L, B, Hkv, T, d)), "v": rng.standard_normal((L, B, Hkv, T, d))}
    q = rng.standard_normal((L, B, Hq, d))
    lmap = tuple((SINGLE, l, 0) for l in range(L))
    mass, ent, peak = rr.decode_stats(lmap, q, lambda n, i: cache[n][i])
    g = Hq // Hkv
    for l in range(L):
        for b in range(B):
            for j in range(Hkv):
                be, bp, bm = brute_stats(q[l, b, j * g:(j + 1) * g].tolist(), cache["k"][l, b, j].tolist(),
                                         1 / math.sqrt(d))
                assert np.allclose(ent[l, b, j * g:(j + 1) * g], be, rtol=1e-12)
                assert np.allclose(peak[l, b, j * g:(j + 1) * g], bp, rtol=1e-12)
                assert np.allclose(mass[l, b, j], bm, rtol=1e-12)


# ----------------------------------------------------------------------------- router score
def exact_score(mass_col, T, Hq):
    total = Fraction(float(np.float32(mass_col[0])))
    for m in mass_col[1:]:
        total = f32(total + Fraction(float(np.float32(m))))
    x = f32(f32(Fraction(T) * total) / Hq)
    return f32(x / f32(1 + x))


def test_route_score_is_the_exact_fp32_sequence():
    rng = np.random.default_rng(7)
    for Hkv, Hq, T in ((1, 4, 100), (4, 16, 8192), (8, 32, 65536), (3, 3, 7)):
        mass = (rng.exponential(1.0, size=(Hkv, 64)) * (Hq // Hkv) / T * rng.choice([0.1, 1, 10, 50], size=64))
        mass = mass.astype(np.float32)
        got = rr.route_score(mass, T, Hq)
        for t in range(mass.shape[1]):
            assert Fraction(float(got[t])) == exact_score(mass[:, t], T, Hq)


def test_route_score_monotone_with_the_uniform_share_at_one_half():
    T, Hq, Hkv = 4096, 32, 8
    share = np.float32(Hq) / np.float32(T) / np.float32(Hkv)     # per-kv-head mass of a uniform token
    mass = np.full((Hkv, 1), share, np.float32)
    assert rr.route_score(mass, T, Hq)[0] == np.float32(0.5)
    grid = np.sort(np.random.default_rng(3).exponential(20.0, size=2000)).astype(np.float32) * share
    s = rr.route_score(np.tile(grid, (Hkv, 1)), T, Hq)
    assert np.all(np.diff(s) >= 0)
    r = qr.route_rank(s)
    x = grid.astype(np.float64) / share
    # rank 8 from 7/3 of the uniform share, rank 16 from 9 (up to fp32 rounding at the edges)
    assert np.all(r[x < 7 / 3 - 1e-4] == 0) and np.all(r[(x > 7 / 3 + 1e-4) & (x < 9 - 1e-3)] == 8)
    assert np.all(r[x > 9 + 1e-3] == 16)


# ----------------------------------------------------------------------------- per-sequence lengths
def ragged_case(seed=0):
    rng = np.random.default_rng(seed)
    L, B, Hq, Hkv, T, d = 2, 4, 8, 2, 23, 16
    cache = {"k": rng.standard_normal((L, B, Hkv, T, d)), "v": rng.standard_normal((L, B, Hkv, T, d))}
    q = rng.standard_normal((L, B, Hq, d))
    return tuple((SINGLE, l, 0) for l in range(L)), q, cache, np.array([23, 1, 9, 0])


def check_lengths_against_masked_sdpa(decode=ref.decode):
    lmap, q, cache, lens = ragged_case()
    out, lse = decode(lmap, q, lambda n, i: cache[n][i], lengths=lens)
    L, B, Hq, d = q.shape
    g = Hq // cache["k"].shape[2]
    for l in range(L):
        for b in range(B):
            n = int(lens[b])
            if n == 0:
                assert np.all(out[l, b] == 0.0) and np.all(lse[l, b] == -np.inf)
                continue
            k = torch.from_numpy(cache["k"][l, b]).repeat_interleave(g, dim=0)[None]   # [1, Hq, T, d]
            v = torch.from_numpy(cache["v"][l, b]).repeat_interleave(g, dim=0)[None]
            qq = torch.from_numpy(q[l, b])[None, :, None, :]
            mask = (torch.arange(k.shape[2]) < n)[None, None, None, :]
            want = torch.nn.functional.scaled_dot_product_attention(qq, k, v, attn_mask=mask)[0, :, 0].numpy()
            assert np.allclose(out[l, b], want, rtol=0, atol=1e-13)


def test_lengths_equal_key_masked_sdpa():
    check_lengths_against_masked_sdpa()


def test_full_lengths_equal_no_lengths_and_the_tail_is_ignored():
    lmap, q, cache, _ = ragged_case(1)
    T = cache["k"].shape[3]
    B = q.shape[1]
    a, la = ref.decode(lmap, q, lambda n, i: cache[n][i], lengths=np.full(B, T))
    b_, lb = ref.decode(lmap, q, lambda n, i: cache[n][i])
    assert np.array_equal(a, b_) and np.array_equal(la, lb)
    lens = np.array([5, 17, 1, 23])
    junk = {k: v.copy() for k, v in cache.items()}
    for b in range(B):
        junk["k"][:, b, :, lens[b]:] = 1e30
        junk["v"][:, b, :, lens[b]:] = np.nan
    c, lc = ref.decode(lmap, q, lambda n, i: junk[n][i], lengths=lens)
    d_, ld = ref.decode(lmap, q, lambda n, i: cache[n][i], lengths=lens)
    assert np.array_equal(c, d_) and np.array_equal(lc, ld)


def test_stats_with_lengths():
    lmap, q, cache, lens = ragged_case(2)
    mass, ent, peak = rr.decode_stats(lmap, q, lambda n, i: cache[n][i], lengths=lens)
    g = q.shape[2] // cache["k"].shape[2]
    for b, n in enumerate(lens):
        assert np.all(mass[:, b, :, n:] == 0.0)
        if n == 0:
            assert np.all(ent[:, b] == 0.0) and np.all(peak[:, b] == 0.0)
        else:
            assert np.allclose(mass[:, b].sum(axis=-1), g, atol=1e-12)
    assert np.all(ent[:, 1] == 0.0) and np.all(peak[:, 1] == 1.0)     # one token: certain


# ----------------------------------------------------------------------------- planted mistakes
def test_pins_catch_planted_mistakes(monkeypatch):
    log2_entropy = lambda p: (rr.attention_stats(p)[0] / math.log(2), rr.attention_stats(p)[1])  # noqa: E731
    min_peak = lambda p: (rr.attention_stats(p)[0], np.min(np.atleast_2d(p), axis=1))  # noqa: E731
    with pytest.raises(AssertionError):
        check_uniform(stats=log2_entropy)
    with pytest.raises(AssertionError):
        check_dominant(stats=min_peak)
    with pytest.raises(AssertionError):
        check_two_tokens(stats=log2_entropy)

    def strided_mass(p, g):     # heads grouped as h % Hkv instead of contiguous blocks
        p = np.asarray(p)
        return p.reshape(g, p.shape[0] // g, -1).sum(axis=0)
    with pytest.raises(AssertionError):
        monkeypatch.setattr(rr, "kv_mass", strided_mass)
        test_masses_sum_to_the_group_size()
    monkeypatch.undo()

    def no_plus_one(mass, context, num_q_heads):
        m = np.asarray(mass, dtype=np.float32)
        x = (np.float32(context) * m.sum(axis=0, dtype=np.float32) / np.float32(num_q_heads)).astype(np.float32)
        return (x / (x + np.float32(2.0))).astype(np.float32)
    monkeypatch.setattr(rr, "route_score", no_plus_one)
    with pytest.raises(AssertionError):
        test_route_score_monotone_with_the_uniform_share_at_one_half()
    monkeypatch.undo()

    orig = ref.decode_head_group

    def one_extra_token(layer_map, l, b, j, q_group, get, w=None, scale=None, length=None):
        return orig(layer_map, l, b, j, q_group, get, w, scale, None if length is None else length + 1)
    monkeypatch.setattr(ref, "decode_head_group", one_extra_token)
    with pytest.raises(AssertionError):
        check_lengths_against_masked_sdpa()
