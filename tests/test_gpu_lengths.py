"""GPU parity of decode with per-sequence lengths (all three forms) against the fp64 oracle.

A decode batch of real requests has ragged lengths ("A Systematic Study of
Cross-Layer KV Sharing for Efficient LLM Inference", TL;DR: serving throughput
across batch sizes). Each case mixes length 0, length 1, lengths that end inside a
token tile, a whole number of tiles and the full store; the cache past every
length holds NaN, which must not reach any output.
"""
import numpy as np
import pytest

import oracle.kvshare_ref as ref
import oracle.quant_ref as qr
from synth.configs import MIX, SINGLE, Config, depthweave_map

from gpu_helpers import assert_close, make_ctx, to_dev

pytestmark = pytest.mark.gpu
TOL = 2e-2


@pytest.fixture(scope="module")
def K():
    from cross_layer_kv_shared_b200 import kvshare
    return kvshare


def kv_cfg(name, dtype, L, lmap, slots, Hq, Hkv, d, B, T, seed):
    return Config(name, "decode", layers=L, q_heads=Hq, kv_heads=Hkv, head_dim=d, batch=B, context=T, dtype=dtype,
                  layer_map=tuple(lmap), slots=slots, seed=seed)


def lengths_for(B, T, seed):
    base = [0, 1, T, 17, 64, T - 1, 33, 200]
    rng = np.random.default_rng(seed)
    out = [min(x, T) for x in base[:B]] + list(rng.integers(1, T + 1, size=max(0, B - len(base))))
    return np.array(out[:B], dtype=np.int32)


def poison_tail(a, lens, dtype):
    """NaN in every stored token at or past each sequence's length (axis 1 = batch, axis -2 = token)."""
    a = a.copy()
    nan = np.uint16(0x7FC0) if dtype == "bf16" else np.float32(np.nan)
    for b, n in enumerate(lens):
        a[:, b, ..., int(n):, :] = nan
    return a


CASES = [
    kv_cfg("len_f32", "f32", 2, [(SINGLE, 0, 0), (MIX, 0, 1)], 2, 4, 2, 64, 5, 150, 61),
    kv_cfg("len_bf16_d64", "bf16", 3, [(SINGLE, 0, 0), (SINGLE, 0, 0), (MIX, 1, 0)], 2, 8, 1, 64, 6, 300, 62),
    kv_cfg("len_bf16_d128_g16", "bf16", 2, [(SINGLE, 0, 0), (MIX, 0, 1)], 2, 32, 2, 128, 7, 257, 63),
]


def run_kv(K, cfg, inp, lens, grid=0, kv_overlap=False, splits=0):
    import torch
    d = {n: to_dev(a, cfg.dtype) for n, a in inp.items()}
    lens_d = torch.from_numpy(lens).cuda()
    h = make_ctx(K, cfg, splits)
    try:
        if grid:
            K.kvshare_debug_set_grid(h, grid)
        K.kvshare_set_kv_overlap(h, kv_overlap)
        K.kvshare_set_map(h, cfg.layer_map, inp["w"])
        out = torch.full((cfg.layers, cfg.batch, cfg.q_heads, cfg.head_dim), float("nan"), device="cuda")
        lse = torch.full((cfg.layers, cfg.batch, cfg.q_heads), float("nan"), device="cuda")
        cache = K.Cache(batch=cfg.batch, context=cfg.context, k=d["k"], v=d["v"], slots=cfg.slots, lengths=lens_d)
        K.kvshare_decode(h, cache, d["q"], out, lse)
        assert K.kvshare_sync_status(h) == K.KVS_OK
    finally:
        K.kvshare_destroy(h)
    return out.cpu().numpy(), lse.cpu().numpy()


def check_against_oracle(cfg, inp, lens, out, lse):
    get = lambda name, index: ref.to_f64(inp[name][index], cfg.dtype)  # noqa: E731
    want, want_lse = ref.decode(cfg.layer_map, ref.to_f64(inp["q"], cfg.dtype), get, w=inp["w"], lengths=lens)
    tol = 1e-4 if cfg.dtype == "f32" else TOL
    err = np.max(np.abs(np.nan_to_num(out, nan=1e9) - np.nan_to_num(want, nan=0.0)), axis=(2, 3))
    print(f"{cfg.name}: max|d| per (layer, sequence) with lengths {list(lens)}:\n{err}")
    empty = lens == 0
    assert np.all(out[:, empty] == 0.0) and np.all(lse[:, empty] == -np.inf)
    full = ~empty
    _, rel = assert_close(out[:, full], want[:, full], tol, cfg.name)
    assert rel < 2e-2
    assert_close(lse[:, full], want_lse[:, full], tol, cfg.name + " lse")


@pytest.mark.parametrize("cfg", CASES, ids=lambda c: c.name)
def test_ragged_lengths_match_the_oracle(K, cfg):
    inp = cfg.make_all()
    lens = lengths_for(cfg.batch, cfg.context, cfg.seed)
    inp["k"] = poison_tail(inp["k"], lens, cfg.dtype)
    inp["v"] = poison_tail(inp["v"], lens, cfg.dtype)
    out, lse = run_kv(K, cfg, inp, lens)
    check_against_oracle(cfg, inp, lens, out, lse)
    if cfg.dtype == "bf16":
        # the same lengths under dependent-launch overlap, and on grids whose CTA ranges
        # cross units (tiles past a sequence are skipped one by one there)
        out2, lse2 = run_kv(K, cfg, inp, lens, kv_overlap=True)
        assert np.array_equal(out, out2) and np.array_equal(lse, lse2)
        for grid in (7, 3 * cfg.batch * cfg.kv_heads + 1):
            out3, lse3 = run_kv(K, cfg, inp, lens, grid=grid)
            check_against_oracle(cfg, inp, lens, out3, lse3)


@pytest.mark.parametrize("cfg", CASES[1:], ids=lambda c: c.name)
def test_ragged_lengths_on_a_clean_cache(K, cfg):
    # the same lengths with ordinary values past them: only the lengths decide
    inp = cfg.make_all()
    lens = lengths_for(cfg.batch, cfg.context, cfg.seed)
    out, lse = run_kv(K, cfg, inp, lens)
    check_against_oracle(cfg, inp, lens, out, lse)


def test_all_lengths_full_equals_no_lengths(K):
    import torch
    cfg = CASES[1]
    inp = cfg.make_all()
    full = np.full(cfg.batch, cfg.context, np.int32)
    out, lse = run_kv(K, cfg, inp, full)
    d = {n: to_dev(a, cfg.dtype) for n, a in inp.items()}
    h = make_ctx(K, cfg)
    try:
        K.kvshare_set_map(h, cfg.layer_map, inp["w"])
        o2 = torch.empty(out.shape, device="cuda")
        l2 = torch.empty(lse.shape, device="cuda")
        K.kvshare_decode(h, K.Cache(batch=cfg.batch, context=cfg.context, k=d["k"], v=d["v"], slots=cfg.slots),
                         d["q"], o2, l2)
        assert K.kvshare_sync_status(h) == K.KVS_OK
    finally:
        K.kvshare_destroy(h)
    assert np.array_equal(out, o2.cpu().numpy()) and np.array_equal(lse, l2.cpu().numpy())


def test_length_out_of_range_is_reported_and_clamped(K):
    import torch
    cfg = CASES[1]
    inp = cfg.make_all()
    d = {n: to_dev(a, cfg.dtype) for n, a in inp.items()}
    lens = np.array([cfg.context + 5, -3, 10, 10, 10, 10], np.int32)
    h = make_ctx(K, cfg)
    try:
        K.kvshare_set_map(h, cfg.layer_map, inp["w"])
        out = torch.empty(cfg.layers, cfg.batch, cfg.q_heads, cfg.head_dim, device="cuda")
        lse = torch.empty(cfg.layers, cfg.batch, cfg.q_heads, device="cuda")
        cache = K.Cache(batch=cfg.batch, context=cfg.context, k=d["k"], v=d["v"], slots=cfg.slots,
                        lengths=torch.from_numpy(lens).cuda())
        K.kvshare_decode(h, cache, d["q"], out, lse)
        assert K.kvshare_sync_status(h) == K.KVS_EINVAL
        assert K.kvshare_sync_status(h) == K.KVS_OK          # the report clears
        clamped = np.clip(lens, 0, cfg.context)
        check_against_oracle(cfg, inp, clamped, out.cpu().numpy(), lse.cpu().numpy())
        host = K.Cache(batch=cfg.batch, context=cfg.context, k=d["k"], v=d["v"], slots=cfg.slots,
                       lengths=torch.from_numpy(lens).pin_memory())
        assert K.kvshare_decode(h, host, d["q"], out, lse, check=False) == K.KVS_EINVAL   # host pointer
    finally:
        K.kvshare_destroy(h)


LR_CASES = [
    Config("len_lowrank", "decode", layers=2, q_heads=8, kv_heads=2, head_dim=128, batch=6, context=300, dtype="bf16",
           layer_map=depthweave_map(2), pairs=1, seed=64),
    Config("len_lowrank_d64_g16", "decode", layers=2, q_heads=16, kv_heads=1, head_dim=64, batch=5, context=129,
           dtype="bf16", layer_map=depthweave_map(2), pairs=1, seed=65),
]


def run_lowrank(K, cfg, inp, lens, splits=0, kv_overlap=False):
    import torch
    from test_gpu_lowrank import pack_gpu
    d = {n: to_dev(a, "bf16") for n, a in inp.items()}
    _, h = K.kvshare_create(cfg.layers, cfg.q_heads, cfg.kv_heads, cfg.head_dim, K.KVS_BF16, cfg.batch, cfg.context,
                            basis_rank=cfg.basis_rank)
    try:
        K.kvshare_set_map(h, cfg.layer_map, None)
        K.kvshare_set_kv_overlap(h, kv_overlap)
        if splits:
            K.kvshare_set_splits(h, splits)
        rank, ck, cv, sk, sv = pack_gpu(K, h, cfg, d["score"], d["u_k"], d["u_v"])
        out = torch.full((cfg.layers, cfg.batch, cfg.q_heads, cfg.head_dim), float("nan"), device="cuda")
        lse = torch.full((cfg.layers, cfg.batch, cfg.q_heads), float("nan"), device="cuda")
        cache = K.Cache(batch=cfg.batch, context=cfg.context, coef_k=d["coef_k"], coef_v=d["coef_v"],
                        basis_k=d["basis_k"], basis_v=d["basis_v"], u_k=ck, u_v=cv, s_k=sk, s_v=sv, r_k=d["r_k"],
                        r_v=d["r_v"], rank=rank, pairs=cfg.pairs, lengths=torch.from_numpy(lens).cuda())
        K.kvshare_decode(h, cache, d["q"], out, lse)
        assert K.kvshare_sync_status(h) == K.KVS_OK
    finally:
        K.kvshare_destroy(h)
    return out.cpu().numpy(), lse.cpu().numpy()


@pytest.mark.parametrize("cfg", LR_CASES, ids=lambda c: c.name)
def test_ragged_lengths_lowrank(K, cfg):
    inp = cfg.make_all()
    lens = lengths_for(cfg.batch, cfg.context, cfg.seed)
    inp["coef_k"] = poison_tail(inp["coef_k"], lens, "bf16")
    inp["coef_v"] = poison_tail(inp["coef_v"], lens, "bf16")
    out, lse = run_lowrank(K, cfg, inp, lens)
    rank, ck, cv, sk, sv = qr.pack_residual(inp["score"], inp["u_k"], inp["u_v"])
    arrs = {"coef_k": ref.bf16_bits_to_f64(inp["coef_k"]), "coef_v": ref.bf16_bits_to_f64(inp["coef_v"]),
            "basis_k": ref.bf16_bits_to_f64(inp["basis_k"]), "basis_v": ref.bf16_bits_to_f64(inp["basis_v"]),
            "u_k": ck.astype(np.float64), "u_v": cv.astype(np.float64),
            "s_k": ref.f16_bits_to_f64(sk), "s_v": ref.f16_bits_to_f64(sv),
            "r_k": ref.bf16_bits_to_f64(inp["r_k"]), "r_v": ref.bf16_bits_to_f64(inp["r_v"]), "rank": rank}
    want, want_lse = ref.decode(cfg.layer_map, ref.bf16_bits_to_f64(inp["q"]), lambda n, i: arrs[n][i], lengths=lens)
    empty = lens == 0
    assert np.all(out[:, empty] == 0.0) and np.all(lse[:, empty] == -np.inf)
    _, rel = assert_close(out[:, ~empty], want[:, ~empty], TOL, cfg.name)
    assert rel < 2e-2
    assert_close(lse[:, ~empty], want_lse[:, ~empty], TOL, cfg.name + " lse")
    out2, lse2 = run_lowrank(K, cfg, inp, lens, kv_overlap=True)
    assert np.array_equal(out, out2) and np.array_equal(lse, lse2)
    out3, _ = run_lowrank(K, cfg, inp, lens, splits=1)
    assert np.max(np.abs(out3 - out)) <= 2.0 ** -8 * np.max(np.abs(out))
