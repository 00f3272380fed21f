"""CPU check of the algebra the decode kernels use to carry entropy and peak.

The kernels never form the normalised weights: beside the running max m and the
weight sum lx = sum 2^(s - m) they keep z = sum 2^(s - m) (m - s) (log2 domain), move
both to a new reference m' as lx' = 2^(m - m') lx, z' = 2^(m - m') (z + lx (m' - m)),
merge warps and split partials the same way against the common max M, and finish with
H = ln 2 (log2 lx + z / lx) and max p = 1 / lx. This test runs those rules in fp64
over random tiles, splits and merge orders (the structure of the online softmax, not
the kernels' code) and compares them with -sum p ln p and max p computed directly,
so a wrong sign, a scale taken after instead of before the update, or a missing
lx (M - m) term fails here.
"""
import numpy as np


def online(scores, tile):
    """Running (m, lx, z) over one split's scores, tile by tile."""
    m, lx, z = -np.inf, 0.0, 0.0
    for t0 in range(0, len(scores), tile):
        s = scores[t0:t0 + tile]
        mn = max(m, float(np.max(s)))
        cr = 0.0 if m == -np.inf else 2.0 ** (m - mn)
        z = cr * (z + (lx * (mn - m) if m != -np.inf else 0.0))
        lx = cr * lx
        p = 2.0 ** (s - mn)
        lx += float(np.sum(p))
        z += float(np.sum(p * (mn - s)))
        m = mn
    return m, lx, z


def merge(parts):
    """Merge of (m, lx, z) statistics against their common max."""
    M = max(p[0] for p in parts)
    lx = z = 0.0
    for m, l, zz in parts:
        if m == -np.inf:
            continue
        f = 2.0 ** (m - M)
        lx += f * l
        z += f * (zz + l * (M - m))
    return M, lx, z


def finish(lx, z):
    return np.log(2.0) * (np.log2(lx) + z / lx), 1.0 / lx


def direct(scores):
    z = scores * np.log(2.0)                  # log2-domain scores -> natural log domain
    p = np.exp(z - z.max())
    p /= p.sum()
    return float(-np.sum(p * np.log(p))), float(p.max())


def test_online_update_and_split_merge_match_the_direct_entropy_and_peak():
    rng = np.random.default_rng(5)
    for trial in range(40):
        n = int(rng.integers(1, 3000))
        spread = float(rng.choice([0.1, 1.0, 8.0, 40.0]))
        s = rng.normal(0.0, spread, n)
        if trial % 5 == 0:
            s = np.sort(s)                    # the max rises on every tile
        n_split = int(rng.integers(1, 9))
        cuts = np.sort(rng.integers(0, n + 1, n_split - 1))
        parts = [online(c, int(rng.choice([16, 32, 64]))) for c in np.split(s, cuts) if len(c)]
        parts += [(-np.inf, 0.0, 0.0)]        # a split with no tokens weighs nothing
        rng.shuffle(parts)
        _, lx, z = merge(parts)
        h, pk = finish(lx, z)
        hw, pw = direct(s)
        assert abs(h - hw) <= 1e-9 * max(1.0, abs(hw)), (trial, h, hw)
        assert abs(pk - pw) <= 1e-12 * pw, (trial, pk, pw)


def test_one_hot_row_has_zero_entropy_without_cancellation():
    # a peaked row: every term of z is non-negative and tiny, so H stays near 0
    s = np.array([60.0] + [0.0] * 1000)
    m, lx, z = online(s, 32)
    h, pk = finish(lx, z)
    hw, pw = direct(s)
    assert 0.0 <= h < 1e-12 and abs(h - hw) < 1e-15
    assert abs(pk - 1.0) < 1e-15 and abs(pk - pw) < 1e-15


def test_uniform_row_has_entropy_ln_n_and_peak_one_over_n():
    for n in (1, 7, 4096):
        m, lx, z = merge([online(np.full(n, 3.25), 16)])
        h, pk = finish(lx, z)
        assert abs(h - np.log(n)) < 1e-12 and abs(pk - 1.0 / n) < 1e-15
