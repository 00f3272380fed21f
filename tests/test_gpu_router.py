"""GPU parity of the attention statistics and the online router (kvshare_decode_stats).

The router reads attention statistics online, per token and step ("DepthWeave-KV:
Smarter KV Cache Compression by Sharing Across Layers and Adapting Per Token",
Core Mechanism, second component; Key Concepts). Checked against the fp64 oracle
(oracle/router_ref.py) element by element:
* mass per kv head and token within 1e-4 relative; entropy and peak per head
  within 1e-4 relative;
* the router score bit for bit against the oracle's fp32 map applied to the
  GPU's masses (both sides take the rank decision in fp32), and the ranks,
  codes and scales kvshare_pack_residual makes from it bit for bit against the
  oracle's packer on the same scores;
* the decode outputs of kvshare_decode_stats are the bits of kvshare_decode.
"""
import numpy as np
import pytest

import oracle.kvshare_ref as ref
import oracle.quant_ref as qr
import oracle.router_ref as rr
import synth.gpu as sgpu
from synth.configs import DEPTHWEAVE_DECODE, MIX, SINGLE, Config, depthweave_map

import code_layout as cl
from gpu_helpers import make_ctx, to_dev

pytestmark = pytest.mark.gpu
REL = 1e-4


@pytest.fixture(scope="module")
def K():
    from cross_layer_kv_shared_b200 import kvshare
    return kvshare


def assert_rel(got, want, what, rel=REL, floor=1e-30):
    got = np.asarray(got, np.float64)
    assert np.all(np.isfinite(got)), what
    err = np.abs(got - want)
    bad = err > rel * np.abs(want) + floor
    assert not np.any(bad), f"{what}: {int(bad.sum())} of {bad.size} beyond {rel} relative, worst " \
                            f"{float(np.max(err / (np.abs(want) + 1e-30))):.3e}"


def stats_outputs(torch, cfg):
    L, B, Hq, Hkv, T = cfg.layers, cfg.batch, cfg.q_heads, cfg.kv_heads, cfg.context
    nan = float("nan")
    return (torch.full((L, B, Hkv, T), nan, device="cuda"), torch.full((L, B, T), nan, device="cuda"),
            torch.full((L, B, Hq), nan, device="cuda"), torch.full((L, B, Hq), nan, device="cuda"))


def check_stats(cfg, got, want, lens=None):
    mass, score, ent, peak = (x.cpu().numpy() for x in got)
    wmass, went, wpeak = want
    assert_rel(mass, wmass, "mass")
    # an entropy of (near) zero carries the scores' absolute rounding (about 1e-6 nats)
    assert_rel(ent, went, "entropy", floor=1e-5)
    assert_rel(peak, wpeak, "peak")
    for l in range(cfg.layers):
        for b in range(cfg.batch):
            n = cfg.context if lens is None else int(lens[b])
            s = rr.route_score(mass[l, b], n, cfg.q_heads)
            assert np.array_equal(score[l, b], s), (l, b)
    return score


KV_CASES = [
    Config("st_bf16_d128", "decode", layers=3, q_heads=16, kv_heads=4, head_dim=128, batch=3, context=333,
           dtype="bf16", layer_map=((SINGLE, 0, 0), (SINGLE, 1, 0), (MIX, 0, 1)), slots=2, seed=71),
    Config("st_bf16_d64_g8", "decode", layers=2, q_heads=16, kv_heads=2, head_dim=64, batch=2, context=1000,
           dtype="bf16", layer_map=((SINGLE, 0, 0), (SINGLE, 0, 0)), slots=1, qkv_scale=0.5, seed=72),
    Config("st_f32", "decode", layers=2, q_heads=4, kv_heads=2, head_dim=64, batch=2, context=150, dtype="f32",
           layer_map=((SINGLE, 0, 0), (MIX, 0, 1)), slots=2, seed=73),
]


@pytest.mark.parametrize("lengths", [False, True], ids=["full", "ragged"])
@pytest.mark.parametrize("cfg", KV_CASES, ids=lambda c: c.name)
def test_stats_match_the_oracle(K, cfg, lengths):
    import torch
    inp = cfg.make_all()
    d = {n: to_dev(a, cfg.dtype) for n, a in inp.items()}
    lens = None
    if lengths:
        lens = np.array([0, 1, cfg.context - 31][:cfg.batch] + [77] * max(0, cfg.batch - 3), np.int32)
    h = make_ctx(K, cfg)
    try:
        K.kvshare_set_map(h, cfg.layer_map, inp["w"])
        cache = K.Cache(batch=cfg.batch, context=cfg.context, k=d["k"], v=d["v"], slots=cfg.slots,
                        lengths=None if lens is None else torch.from_numpy(lens).cuda())
        out = torch.empty(cfg.layers, cfg.batch, cfg.q_heads, cfg.head_dim, device="cuda")
        lse = torch.empty(cfg.layers, cfg.batch, cfg.q_heads, device="cuda")
        st = stats_outputs(torch, cfg)
        n0 = K.kvshare_launch_count(h)
        K.kvshare_decode_stats(h, cache, d["q"], out, lse, *st)
        assert K.kvshare_sync_status(h) == K.KVS_OK
        # per layer: the decode (entropy and peak from its merge) and the per-token statistics
        assert K.kvshare_launch_count(h) - n0 == 2 * cfg.layers
        out2 = torch.empty_like(out)
        lse2 = torch.empty_like(lse)
        K.kvshare_decode(h, cache, d["q"], out2, lse2)
        assert K.kvshare_sync_status(h) == K.KVS_OK
        assert torch.equal(out, out2) and torch.equal(lse, lse2)
    finally:
        K.kvshare_destroy(h)
    get = lambda name, index: ref.to_f64(inp[name][index], cfg.dtype)  # noqa: E731
    want = rr.decode_stats(cfg.layer_map, ref.to_f64(inp["q"], cfg.dtype), get, w=inp["w"], lengths=lens)
    check_stats(cfg, st, want, lens)


@pytest.mark.parametrize("grid", [None, 7, 13], ids=["default", "grid7", "grid13"])
@pytest.mark.parametrize("cfg", KV_CASES, ids=lambda c: c.name)
def test_entropy_and_peak_alone_from_the_decode_merge(K, cfg, grid):
    """Entropy and peak without mass or score: no score buffer and no statistics kernel,
    the values come out of the decode's online softmax and its merge of warps, saved
    unit states (straddling debug grids) and split partials (forced splits on the fp32
    path); the same bits on a second call, and against the oracle."""
    import torch
    inp = cfg.make_all()
    d = {n: to_dev(a, cfg.dtype) for n, a in inp.items()}
    lens = np.array([1, cfg.context - 31, 77][:cfg.batch] + [5] * max(0, cfg.batch - 3), np.int32)
    h = make_ctx(K, cfg)
    try:
        K.kvshare_set_map(h, cfg.layer_map, inp["w"])
        if grid is not None:
            if cfg.dtype == "f32":
                K.kvshare_set_splits(h, grid)
            else:
                K.kvshare_debug_set_grid(h, grid)
        cache = K.Cache(batch=cfg.batch, context=cfg.context, k=d["k"], v=d["v"], slots=cfg.slots,
                        lengths=torch.from_numpy(lens).cuda())
        out = torch.empty(cfg.layers, cfg.batch, cfg.q_heads, cfg.head_dim, device="cuda")
        lse = torch.empty(cfg.layers, cfg.batch, cfg.q_heads, device="cuda")
        ent, peak = stats_outputs(torch, cfg)[2:]
        n0 = K.kvshare_launch_count(h)
        K.kvshare_decode_stats(h, cache, d["q"], out, lse, None, None, ent, peak)
        assert K.kvshare_sync_status(h) == K.KVS_OK
        assert K.kvshare_launch_count(h) - n0 == cfg.layers      # the decode kernels only
        ent2, peak2 = torch.empty_like(ent), torch.empty_like(peak)
        K.kvshare_decode_stats(h, cache, d["q"], out, lse, None, None, ent2, peak2)
        assert K.kvshare_sync_status(h) == K.KVS_OK
        assert torch.equal(ent, ent2) and torch.equal(peak, peak2)
    finally:
        K.kvshare_destroy(h)
    get = lambda name, index: ref.to_f64(inp[name][index], cfg.dtype)  # noqa: E731
    _, went, wpeak = rr.decode_stats(cfg.layer_map, ref.to_f64(inp["q"], cfg.dtype), get, w=inp["w"], lengths=lens)
    assert_rel(ent.cpu().numpy(), went, "entropy", floor=1e-5)
    assert_rel(peak.cpu().numpy(), wpeak, "peak")


def test_stats_feed_the_packer_bit_for_bit(K):
    """Scores from a low-rank decode step re-route every token: the packer's ranks, codes
    and scales from the GPU score equal the oracle packer's on the same score."""
    import torch
    from test_gpu_lowrank import pack_gpu
    cfg = Config("st_lowrank", "decode", layers=2, q_heads=8, kv_heads=2, head_dim=128, batch=2, context=700,
                 dtype="bf16", layer_map=depthweave_map(2), pairs=1, seed=74)
    inp = cfg.make_all()
    d = {n: to_dev(a, "bf16") for n, a in inp.items()}
    _, h = K.kvshare_create(cfg.layers, cfg.q_heads, cfg.kv_heads, cfg.head_dim, K.KVS_BF16, cfg.batch, cfg.context)
    try:
        K.kvshare_set_map(h, cfg.layer_map, None)
        rank, ck, cv, sk, sv = pack_gpu(K, h, cfg, d["score"], d["u_k"], d["u_v"])
        cache = K.Cache(batch=cfg.batch, context=cfg.context, coef_k=d["coef_k"], coef_v=d["coef_v"],
                        basis_k=d["basis_k"], basis_v=d["basis_v"], u_k=ck, u_v=cv, s_k=sk, s_v=sv, r_k=d["r_k"],
                        r_v=d["r_v"], rank=rank, pairs=cfg.pairs)
        out = torch.empty(cfg.layers, cfg.batch, cfg.q_heads, cfg.head_dim, device="cuda")
        lse = torch.empty(cfg.layers, cfg.batch, cfg.q_heads, device="cuda")
        st = stats_outputs(torch, cfg)
        K.kvshare_decode_stats(h, cache, d["q"], out, lse, *st)
        assert K.kvshare_sync_status(h) == K.KVS_OK
        new = pack_gpu(K, h, cfg, st[1], d["u_k"], d["u_v"])
        assert K.kvshare_sync_status(h) == K.KVS_OK
    finally:
        K.kvshare_destroy(h)
    packed = qr.pack_residual(inp["score"], inp["u_k"], inp["u_v"])
    arrs = {"coef_k": ref.bf16_bits_to_f64(inp["coef_k"]), "coef_v": ref.bf16_bits_to_f64(inp["coef_v"]),
            "basis_k": ref.bf16_bits_to_f64(inp["basis_k"]), "basis_v": ref.bf16_bits_to_f64(inp["basis_v"]),
            "u_k": packed[1].astype(np.float64), "u_v": packed[2].astype(np.float64),
            "s_k": ref.f16_bits_to_f64(packed[3]), "s_v": ref.f16_bits_to_f64(packed[4]),
            "r_k": ref.bf16_bits_to_f64(inp["r_k"]), "r_v": ref.bf16_bits_to_f64(inp["r_v"]), "rank": packed[0]}
    want = rr.decode_stats(cfg.layer_map, ref.bf16_bits_to_f64(inp["q"]), lambda n, i: arrs[n][i])
    score = check_stats(cfg, st, want)
    repacked = qr.pack_residual(score, inp["u_k"], inp["u_v"])
    new = [x.cpu().numpy() for x in new]
    new[1], new[2] = cl.unpack(new[1], new[0]), cl.unpack(new[2], new[0])   # group-packed codes as dense
    for name, got, exp in zip(("rank", "codes_k", "codes_v", "scale_k", "scale_v"), new, repacked):
        assert np.array_equal(got.view(exp.dtype), exp), name


def test_stats_validation(K):
    import torch
    cfg = KV_CASES[0]
    inp = cfg.make_all()
    d = {n: to_dev(a, cfg.dtype) for n, a in inp.items()}
    h = make_ctx(K, cfg)
    try:
        K.kvshare_set_map(h, cfg.layer_map, inp["w"])
        cache = K.Cache(batch=cfg.batch, context=cfg.context, k=d["k"], v=d["v"], slots=cfg.slots)
        out = torch.empty(cfg.layers, cfg.batch, cfg.q_heads, cfg.head_dim, device="cuda")
        mass, score, ent, peak = stats_outputs(torch, cfg)
        n0 = K.kvshare_launch_count(h)
        assert K.kvshare_decode_stats(h, cache, d["q"], out, None, mass, check=False) == K.KVS_EINVAL   # no lse
        lse = torch.empty(cfg.layers, cfg.batch, cfg.q_heads, device="cuda")
        assert K.kvshare_decode_stats(h, cache, d["q"], out, lse, mass.cpu(), check=False) == K.KVS_EINVAL
        assert K.kvshare_launch_count(h) == n0
    finally:
        K.kvshare_destroy(h)


def test_full_size_depthweave_stats_every_layer(K):
    """The 64K-token low-rank workload: statistics of every layer and kv head, and the
    router's ranks from them, against the oracle."""
    import torch
    from test_gpu_lowrank import pack_gpu
    cfg = DEPTHWEAVE_DECODE
    dev = {n: sgpu.make_device(cfg, n) for n in cfg.recipe()}
    _, h = K.kvshare_create(cfg.layers, cfg.q_heads, cfg.kv_heads, cfg.head_dim, K.KVS_BF16, cfg.batch, cfg.context)
    try:
        K.kvshare_set_map(h, cfg.layer_map, None)
        rank, ck, cv, sk, sv = pack_gpu(K, h, cfg, dev["score"], dev["u_k"], dev["u_v"])
        cache = K.Cache(batch=1, context=cfg.context, coef_k=dev["coef_k"], coef_v=dev["coef_v"],
                        basis_k=dev["basis_k"], basis_v=dev["basis_v"], u_k=ck, u_v=cv, s_k=sk, s_v=sv,
                        r_k=dev["r_k"], r_v=dev["r_v"], rank=rank, pairs=cfg.pairs)
        out = torch.empty(cfg.layers, 1, cfg.q_heads, cfg.head_dim, device="cuda")
        lse = torch.empty(cfg.layers, 1, cfg.q_heads, device="cuda")
        st = stats_outputs(torch, cfg)
        K.kvshare_decode_stats(h, cache, dev["q"], out, lse, *st)
        assert K.kvshare_sync_status(h) == K.KVS_OK
        new_rank = pack_gpu(K, h, cfg, st[1], dev["u_k"], dev["u_v"])[0]
        assert K.kvshare_sync_status(h) == K.KVS_OK
    finally:
        K.kvshare_destroy(h)
    mass, score, ent, peak = (x.cpu().numpy() for x in st)
    new_rank = new_rank.cpu().numpy()
    import oracle_pool
    units = [(l, j) for l in range(cfg.layers) for j in range(cfg.kv_heads)]
    res = oracle_pool.run(oracle_pool.lowrank_stats_unit, [(cfg.name, l, j) for (l, j) in units])
    g = cfg.group
    for (l, j), (wm, we, wp) in zip(units, res):
        assert_rel(mass[l, 0, j], wm, f"mass l{l} j{j}")
        assert_rel(ent[l, 0, j * g:(j + 1) * g], we, f"entropy l{l} j{j}", floor=1e-5)
        assert_rel(peak[l, 0, j * g:(j + 1) * g], wp, f"peak l{l} j{j}")
    for l in range(cfg.layers):
        s = rr.route_score(mass[l, 0], cfg.context, cfg.q_heads)
        assert np.array_equal(score[l, 0], s), l
        assert np.array_equal(new_rank[l, 0], qr.route_rank(s)), l
    shares = np.bincount(new_rank.ravel(), minlength=17)[[0, 8, 16]] / new_rank.size
    print(f"depthweave_decode router: rank 0/8/16 shares {shares}")
