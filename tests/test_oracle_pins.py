"""Pins of the fp64 oracle to things other than itself.

* I1: an identity layer map is standard GQA attention -> torch SDPA (fp64, CPU).
* I2: mix endpoints w=1 / w=0 and equal sources.
* I3: a full-rank identity basis with zero residual reproduces K/V bit for bit.
* I4: softmax weights sum to one; V = 1 gives o = 1.
* I5: brute force at 50 digits (mpmath, pure-Python loops) on tiny inputs, all
  three forms; the absorbed low-rank algebra the kernels use agrees.
* I6: decode is invariant under a joint permutation of the cached tokens.
* I8: causal prefill row i equals decode over tokens 0..i; an identity map's
  prefill equals torch's causal SDPA (fp64).
* closed forms: equal keys average V; two tokens give a logistic weight.
* planted mistakes: each pin fails when a plausible bug is planted in the oracle.
"""
import math

import mpmath
import numpy as np
import pytest
import torch

import oracle.kvshare_ref as ref

SINGLE, MIX, LOWRANK = ref.SINGLE, ref.MIX, ref.LOWRANK
rng = np.random.default_rng(1234)


def dict_get(arrs):
    return lambda name, index: arrs[name][index]


def rand_cache(slots, B, Hkv, T, d, seed=0):
    r = np.random.default_rng(seed)
    return {"k": r.standard_normal((slots, B, Hkv, T, d)), "v": r.standard_normal((slots, B, Hkv, T, d))}


def rand_lowrank(L, P, B, Hkv, T, d, Rb, Rm, seed=0, ranks=(0, 8, 16)):
    r = np.random.default_rng(seed)
    c = {}
    for s in "kv":
        c["coef_" + s] = r.standard_normal((P, B, Hkv, T, Rb)) / math.sqrt(Rb)
        c["basis_" + s] = r.standard_normal((P, Hkv, Rb, d)) / math.sqrt(Rb)
        c["u_" + s] = r.integers(-127, 128, size=(L, B, Hkv, T, Rm)).astype(np.float64)
        c["s_" + s] = r.uniform(0.001, 0.02, size=(L, B, Hkv, T))
        c["r_" + s] = r.standard_normal((L, Hkv, Rm, d)) / math.sqrt(Rm)
    c["rank"] = r.choice(np.array(ranks), size=(L, B, T))
    return c


# ----------------------------------------------------------------------------- I1
def check_identity_map_is_sdpa(L=3, B=2, Hq=8, Hkv=2, T=37, d=16):
    cache = rand_cache(L, B, Hkv, T, d, seed=1)
    q = np.random.default_rng(2).standard_normal((L, B, Hq, d))
    lmap = tuple((SINGLE, l, 0) for l in range(L))
    out, lse = ref.decode(lmap, q, dict_get(cache))
    g = Hq // Hkv
    for l in range(L):
        k = torch.from_numpy(cache["k"][l]).repeat_interleave(g, dim=1)     # [B, Hq, T, d]
        v = torch.from_numpy(cache["v"][l]).repeat_interleave(g, dim=1)
        qq = torch.from_numpy(q[l])[:, :, None, :]                            # [B, Hq, 1, d]
        o = torch.nn.functional.scaled_dot_product_attention(qq, k, v)[:, :, 0, :].numpy()
        assert np.max(np.abs(out[l] - o)) < 1e-12
        z = torch.einsum("bhd,bhtd->bht", torch.from_numpy(q[l]), k) / math.sqrt(d)
        assert np.max(np.abs(lse[l] - torch.logsumexp(z, dim=-1).numpy())) < 1e-12


def test_identity_map_is_sdpa():
    check_identity_map_is_sdpa()
    check_identity_map_is_sdpa(L=1, B=1, Hq=4, Hkv=4, T=5, d=64)    # MHA
    check_identity_map_is_sdpa(L=2, B=1, Hq=6, Hkv=1, T=9, d=8)     # MQA


def test_cla_map_equals_sdpa_on_the_shared_slot():
    cache = rand_cache(2, 1, 2, 11, 8, seed=3)
    q = rng.standard_normal((4, 1, 4, 8))
    lmap = tuple((SINGLE, l // 2, 0) for l in range(4))
    out, _ = ref.decode(lmap, q, dict_get(cache))
    for l in range(4):
        k = torch.from_numpy(cache["k"][l // 2]).repeat_interleave(2, dim=1)
        v = torch.from_numpy(cache["v"][l // 2]).repeat_interleave(2, dim=1)
        o = torch.nn.functional.scaled_dot_product_attention(torch.from_numpy(q[l])[:, :, None], k, v)
        assert np.max(np.abs(out[l] - o[:, :, 0].numpy())) < 1e-12


# ----------------------------------------------------------------------------- I2
def check_mix_endpoints():
    cache = rand_cache(3, 1, 2, 13, 8, seed=4)
    q = rng.standard_normal((1, 1, 4, 8))
    get = dict_get(cache)
    single0, _ = ref.decode(((SINGLE, 0, 0),), q, get)
    single2, _ = ref.decode(((SINGLE, 2, 0),), q, get)
    w1, _ = ref.decode(((MIX, 0, 2),), q, get, w=np.ones((1, 2)))
    w0, _ = ref.decode(((MIX, 0, 2),), q, get, w=np.zeros((1, 2)))
    assert np.array_equal(w1, single0)
    assert np.array_equal(w0, single2)
    same = {"k": np.concatenate([cache["k"][:1], cache["k"][:1]]),
            "v": np.concatenate([cache["v"][:1], cache["v"][:1]])}
    a, _ = ref.decode(((MIX, 0, 1),), q, dict_get(same), w=np.full((1, 2), 0.3))
    b, _ = ref.decode(((MIX, 0, 1),), q, dict_get(same), w=np.full((1, 2), 0.9))
    assert np.max(np.abs(a - b)) < 1e-14
    # per-kv-head weight: head group j uses w[l][j]
    wm = np.array([[1.0, 0.0]])
    m, _ = ref.decode(((MIX, 0, 2),), q, get, w=wm)
    assert np.array_equal(m[:, :, :2], single0[:, :, :2]) and np.array_equal(m[:, :, 2:], single2[:, :, 2:])


def test_mix_endpoints():
    check_mix_endpoints()


def test_mix_is_linear_in_w():
    K1, K2 = rng.standard_normal((2, 9, 4))
    for w in (0.0, 0.25, 0.5, 1.0):
        assert np.max(np.abs(ref.kv_mix(w, K1, K2) - (K2 + w * (K1 - K2)))) < 1e-15


# ----------------------------------------------------------------------------- I3
def test_full_rank_identity_basis_reproduces_kv_exactly():
    L, B, Hkv, T, d = 2, 1, 2, 10, 8
    cache = rand_cache(1, B, Hkv, T, d, seed=5)
    # bf16-representable values so the coefficients are the K/V bits themselves
    for k in ("k", "v"):
        cache[k] = ref.bf16_bits_to_f64((cache[k].astype(np.float32).view(np.uint32) >> 16).astype(np.uint16))
    lr = {"coef_k": cache["k"], "coef_v": cache["v"],
          "basis_k": np.broadcast_to(np.eye(d), (1, Hkv, d, d)).copy(),
          "basis_v": np.broadcast_to(np.eye(d), (1, Hkv, d, d)).copy(),
          "u_k": rng.standard_normal((L, B, Hkv, T, 16)), "u_v": rng.standard_normal((L, B, Hkv, T, 16)),
          "s_k": np.ones((L, B, Hkv, T)), "s_v": np.ones((L, B, Hkv, T)),
          "r_k": rng.standard_normal((L, Hkv, 16, d)), "r_v": rng.standard_normal((L, Hkv, 16, d)),
          "rank": np.zeros((L, B, T), dtype=np.int64)}
    for l in range(L):
        for j in range(Hkv):
            K, V = ref.layer_kv(((LOWRANK, 0, 0),) * L, l, 0, j, dict_get(lr))
            assert np.array_equal(K, cache["k"][0, 0, j]) and np.array_equal(V, cache["v"][0, 0, j])
    q = rng.standard_normal((L, B, 4, d))
    a, _ = ref.decode(((LOWRANK, 0, 0),) * L, q, dict_get(lr))
    b, _ = ref.decode(((SINGLE, 0, 0),) * L, q, dict_get(cache))
    assert np.array_equal(a, b)


# ----------------------------------------------------------------------------- I4
def test_softmax_rows_sum_to_one_and_constant_v():
    q = rng.standard_normal((5, 16)) * 3
    K = rng.standard_normal((300, 16)) * 3
    V = np.ones((300, 16))
    o, lse, p = ref.attend(q, K, V, 0.25)
    assert np.max(np.abs(p.sum(axis=1) - 1)) < 1e-12
    assert np.max(np.abs(o - 1)) < 1e-12
    assert np.all(p >= 0)


# ----------------------------------------------------------------------------- closed forms
def test_equal_keys_average_values():
    K = np.tile(rng.standard_normal((1, 8)), (7, 1))
    V = rng.standard_normal((7, 8))
    o, lse, _ = ref.attend(rng.standard_normal((3, 8)), K, V, 0.5)
    assert np.max(np.abs(o - V.mean(axis=0))) < 1e-14


def test_two_tokens_logistic_weight():
    q = np.array([[1.0, 2.0]])
    K = np.array([[0.5, -1.0], [2.0, 0.25]])
    V = np.array([[1.0, 0.0], [0.0, 1.0]])
    z0, z1 = (q @ K.T)[0] * 0.7
    w1 = 1.0 / (1.0 + math.exp(z0 - z1))
    o, lse, _ = ref.attend(q, K, V, 0.7)
    assert abs(o[0, 1] - w1) < 1e-15 and abs(o[0, 0] - (1 - w1)) < 1e-15
    assert abs(lse[0] - math.log(math.exp(z0) + math.exp(z1))) < 1e-14


def test_single_visible_token_and_dominant_key():
    K = rng.standard_normal((6, 4))
    V = rng.standard_normal((6, 4))
    o, lse, _ = ref.attend(rng.standard_normal((1, 4)), K, V, 1.0, visible=[1])
    assert np.array_equal(o[0], V[0])
    q = np.array([[1.0, 0, 0, 0]])
    K2 = np.zeros((6, 4)); K2[3, 0] = 2000.0
    o2, _, _ = ref.attend(q, K2, V, 1.0)
    assert np.max(np.abs(o2[0] - V[3])) < 1e-300 + 1e-12


# ----------------------------------------------------------------------------- I5
def brute_force_decode(lmap, q, cache, w, scale, Rm=None):
    """50-digit evaluation with plain loops of the three forms' definitions."""
    mpmath.mp.dps = 50
    L, B, Hq, d = q.shape
    out = np.zeros((L, B, Hq, d))
    for l in range(L):
        kind, s0, s1 = lmap[l]
        for b in range(B):
            if kind == LOWRANK:
                Hkv = cache["basis_k"].shape[1]
                T = cache["coef_k"].shape[3]
            else:
                Hkv = cache["k"].shape[2]
                T = cache["k"].shape[3]
            g = Hq // Hkv
            for h in range(Hq):
                j = h // g
                Ks, Vs = [], []
                for t in range(T):
                    if kind == SINGLE:
                        kr = [mpmath.mpf(float(x)) for x in cache["k"][s0, b, j, t]]
                        vr = [mpmath.mpf(float(x)) for x in cache["v"][s0, b, j, t]]
                    elif kind == MIX:
                        ww = mpmath.mpf(float(w[l][j]))
                        kr = [ww * mpmath.mpf(float(a)) + (1 - ww) * mpmath.mpf(float(c))
                              for a, c in zip(cache["k"][s0, b, j, t], cache["k"][s1, b, j, t])]
                        vr = [ww * mpmath.mpf(float(a)) + (1 - ww) * mpmath.mpf(float(c))
                              for a, c in zip(cache["v"][s0, b, j, t], cache["v"][s1, b, j, t])]
                    else:
                        r = int(cache["rank"][l, b, t])
                        rows = []
                        for s in "kv":
                            C = cache["coef_" + s][s0, b, j, t]
                            Bs = cache["basis_" + s][s0, j]
                            U = cache["u_" + s][l, b, j, t]
                            R = cache["r_" + s][l, j]
                            sc = mpmath.mpf(float(cache["s_" + s][l, b, j, t]))
                            row = []
                            for e in range(d):
                                acc = mpmath.mpf(0)
                                for i in range(C.shape[0]):
                                    acc += mpmath.mpf(float(C[i])) * mpmath.mpf(float(Bs[i, e]))
                                res = mpmath.mpf(0)
                                for i in range(r):
                                    res += mpmath.mpf(float(U[i])) * mpmath.mpf(float(R[i, e]))
                                row.append(acc + sc * res)
                            rows.append(row)
                        kr, vr = rows
                    Ks.append(kr)
                    Vs.append(vr)
                z = [sum(mpmath.mpf(float(q[l, b, h, e])) * Ks[t][e] for e in range(d)) * mpmath.mpf(scale)
                     for t in range(T)]
                ez = [mpmath.exp(x) for x in z]
                den = sum(ez)
                for e in range(d):
                    out[l, b, h, e] = float(sum(ez[t] * Vs[t][e] for t in range(T)) / den)
    return out


def check_brute_force_forms():
    B, Hkv, Hq, T, d = 1, 2, 4, 5, 3
    cache = rand_cache(2, B, Hkv, T, d, seed=7)
    w = np.array([[0.0, 0.0], [0.3, 0.8]])
    lmap = ((SINGLE, 1, 0), (MIX, 0, 1))
    q = rng.standard_normal((2, B, Hq, d))
    got, _ = ref.decode(lmap, q, dict_get(cache), w=w)
    exp = brute_force_decode(lmap, q, cache, w, 1 / math.sqrt(d))
    assert np.max(np.abs(got - exp)) < 1e-13
    lr = rand_lowrank(2, 1, 1, 2, 6, 3, Rb=4, Rm=16, seed=8, ranks=(0, 8, 16))
    lr["rank"][0, 0, :3] = [0, 8, 16]
    lmap2 = ((LOWRANK, 0, 0), (LOWRANK, 0, 0))
    q2 = rng.standard_normal((2, 1, 4, 3))
    got2, _ = ref.decode(lmap2, q2, dict_get(lr))
    exp2 = brute_force_decode(lmap2, q2, lr, None, 1 / math.sqrt(3))
    assert np.max(np.abs(got2 - exp2)) < 1e-12 * max(1.0, np.max(np.abs(exp2)))


def test_brute_force_forms():
    check_brute_force_forms()


def test_absorbed_lowrank_algebra_matches_reconstruction():
    """score_t = c_t.(B q) + s_t u_t.(R q);  o = ((sum p c) B_V + (sum p s u) R_V) / sum p."""
    L, P, B, Hkv, T, d, Rb, Rm = 2, 1, 1, 2, 40, 16, 8, 16
    lr = rand_lowrank(L, P, B, Hkv, T, d, Rb, Rm, seed=9)
    q = rng.standard_normal((L, B, 4, d))
    lmap = ((LOWRANK, 0, 0),) * L
    want, _ = ref.decode(lmap, q, dict_get(lr))
    for l in range(L):
        for h in range(4):
            j = h // 2
            r = lr["rank"][l, 0]
            mask = np.arange(Rm)[None, :] < r[:, None]
            qt = lr["basis_k"][0, j] @ q[l, 0, h]
            qh = lr["r_k"][l, j] @ q[l, 0, h]
            z = (lr["coef_k"][0, 0, j] @ qt + lr["s_k"][l, 0, j] * ((lr["u_k"][l, 0, j] * mask) @ qh)) / math.sqrt(d)
            p = np.exp(z - z.max())
            chat = p @ lr["coef_v"][0, 0, j]
            uhat = (p * lr["s_v"][l, 0, j]) @ (lr["u_v"][l, 0, j] * mask)
            o = (chat @ lr["basis_v"][0, j] + uhat @ lr["r_v"][l, j]) / p.sum()
            assert np.max(np.abs(o - want[l, 0, h])) < 1e-12


# ----------------------------------------------------------------------------- I6, I8
def test_token_permutation_invariance():
    lr = rand_lowrank(1, 1, 1, 2, 50, 8, 4, 16, seed=10)
    q = rng.standard_normal((1, 1, 2, 8))
    lmap = ((LOWRANK, 0, 0),)
    a, la = ref.decode(lmap, q, dict_get(lr))
    perm = np.random.default_rng(11).permutation(50)
    pl = dict(lr)
    for s in "kv":
        pl["coef_" + s] = lr["coef_" + s][:, :, :, perm]
        pl["u_" + s] = lr["u_" + s][:, :, :, perm]
        pl["s_" + s] = lr["s_" + s][:, :, :, perm]
    pl["rank"] = lr["rank"][:, :, perm]
    b, lb = ref.decode(lmap, q, dict_get(pl))
    assert np.max(np.abs(a - b)) < 1e-13 and np.max(np.abs(la - lb)) < 1e-13


def test_prefill_row_equals_decode_over_prefix():
    cache = rand_cache(2, 1, 2, 20, 8, seed=12)
    w = np.array([[0.0, 0.0], [0.0, 0.0], [0.4, 0.6]])
    lmap = ((SINGLE, 0, 0), (SINGLE, 1, 0), (MIX, 0, 1))
    qrows = rng.standard_normal((20, 8))
    rows = np.arange(20)
    o, lse = ref.prefill_rows(lmap, 2, 0, 3, 2, qrows, rows, dict_get(cache), w=w)
    for i in (0, 1, 7, 19):
        pref = {k: v[:, :, :, :i + 1] for k, v in cache.items()}
        d, ld = ref.decode_head_group(lmap, 2, 0, 1, qrows[i:i + 1], dict_get(pref), w=w)
        assert np.max(np.abs(o[i] - d[0])) < 1e-13 and abs(lse[i] - ld[0]) < 1e-13


def check_prefill_identity_map_is_causal_sdpa(L=2, B=2, Hq=8, Hkv=2, T=29, d=16):
    g = Hq // Hkv
    cache = rand_cache(L, B, Hkv, T, d, seed=21)
    q = np.random.default_rng(22).standard_normal((L, B, Hq, T, d))
    lmap = tuple((SINGLE, l, 0) for l in range(L))
    rows = np.arange(T)
    for l in range(L):
        k = torch.from_numpy(cache["k"][l]).repeat_interleave(g, dim=1)     # [B, Hq, T, d]
        v = torch.from_numpy(cache["v"][l]).repeat_interleave(g, dim=1)
        qq = torch.from_numpy(q[l])
        want = torch.nn.functional.scaled_dot_product_attention(qq, k, v, is_causal=True).numpy()
        z = torch.einsum("bhid,bhtd->bhit", qq, k) / math.sqrt(d)
        z = z.masked_fill(torch.triu(torch.ones(T, T, dtype=torch.bool), 1), float("-inf"))
        want_lse = torch.logsumexp(z, dim=-1).numpy()
        for b in range(B):
            for h in range(Hq):
                o, lse = ref.prefill_rows(lmap, l, b, h, g, q[l, b, h], rows, dict_get(cache))
                assert np.max(np.abs(o - want[b, h])) < 1e-12
                assert np.max(np.abs(lse - want_lse[b, h])) < 1e-12


def test_prefill_identity_map_is_causal_sdpa():
    # independent of the decode oracle: causal GQA attention by torch in fp64, each
    # q head h reading kv head h // g, position i seeing tokens 0..i
    check_prefill_identity_map_is_causal_sdpa()


# ----------------------------------------------------------------------------- I9
def test_stored_bytes_reproduce_the_pages_ratios():
    # Cross-Layer Attention, Abstract: CLA2 halves the cache.
    cla = tuple((SINGLE, l // 2, 0) for l in range(22))
    assert ref.stored_bytes(cla, 32, 4, 2048, 64) * 2 == ref.full_cache_bytes(22, 32, 4, 2048, 64)
    # DepthGraft, Abstract: roughly one third of the cache removed (8 of 24 layers store nothing).
    dg = tuple([(SINGLE, l, 0) for l in range(16)] + [(MIX, j, 8 + j) for j in range(8)])
    st = ref.stored_bytes(dg, 16, 4, 8192, 128)
    assert st * 3 == ref.full_cache_bytes(24, 16, 4, 8192, 128) * 2
    # DepthWeave-style layout at ranks 0/8/16 with 70/20/10 %: ~7.1x smaller
    # per layer, kv head and token: 64 B of coefficients (half of a pair's 128 B), 2 * E[r] = 6.4 B
    # of codes, 4 B of scales on the 30 % of tokens with r > 0, 1/8 B of rank: 71.725 B vs 512 B
    T = 65536
    ranks = np.zeros((32, 1, T), dtype=np.int64)
    ranks[:, :, int(0.7 * T):int(0.9 * T)] = 8
    ranks[:, :, int(0.9 * T):] = 16
    dw = tuple((LOWRANK, l // 2, 0) for l in range(32))
    ratio = ref.full_cache_bytes(32, 1, 8, T, 128) / ref.stored_bytes(dw, 1, 8, T, 128, ranks=ranks)
    assert 7.10 < ratio < 512 / 71.725


# ----------------------------------------------------------------------------- planted mistakes
def test_pins_catch_planted_mistakes(monkeypatch):
    orig_mix, orig_attend, orig_lr = ref.kv_mix, ref.attend, ref.kv_lowrank

    monkeypatch.setattr(ref, "kv_mix", lambda w, a, b: orig_mix(1.0 - w, a, b))      # swapped weights
    with pytest.raises(AssertionError):
        check_mix_endpoints()
    monkeypatch.setattr(ref, "kv_mix", orig_mix)

    monkeypatch.setattr(ref, "attend", lambda q, K, V, s, visible=None: orig_attend(q, K, V, s * s, visible))
    with pytest.raises(AssertionError):                                              # 1/d scale
        check_identity_map_is_sdpa()
    monkeypatch.setattr(ref, "attend", orig_attend)

    def lr_off_by_one(C, Bas, s, U, R, r):
        return orig_lr(C, Bas, s, U, R, np.asarray(r) + 1)
    monkeypatch.setattr(ref, "kv_lowrank", lr_off_by_one)                          # i <= r
    with pytest.raises(AssertionError):
        check_brute_force_forms()
    monkeypatch.setattr(ref, "kv_lowrank", orig_lr)

    orig_layer_kv = ref.layer_kv

    def wrong_group(layer_map, l, b, j, get, w=None):                              # V of the wrong head
        K, _ = orig_layer_kv(layer_map, l, b, j, get, w)
        _, V = orig_layer_kv(layer_map, l, b, (j + 1) % 2, get, w)
        return K, V
    monkeypatch.setattr(ref, "layer_kv", wrong_group)
    with pytest.raises(AssertionError):
        check_identity_map_is_sdpa()
    with pytest.raises(AssertionError):
        check_prefill_identity_map_is_causal_sdpa()
    monkeypatch.setattr(ref, "layer_kv", orig_layer_kv)

    def one_future_token(q, K, V, s, visible=None):                                # sees 0..i+1
        return orig_attend(q, K, V, s, None if visible is None else np.asarray(visible) + 1)
    monkeypatch.setattr(ref, "attend", one_future_token)
    with pytest.raises(AssertionError):
        check_prefill_identity_map_is_causal_sdpa()
    monkeypatch.setattr(ref, "attend", orig_attend)
