"""GPU parity of the low-rank causal prefill (absorbed form on tcgen05) with the fp64 oracle.

The kernel attends with [B_K q | R_K q] against [C | s U] operands built per tile
and projects once through [B_V; R_V] ("DepthWeave-KV: Token-Adaptive Cross-Layer
Residual Factorization for Long-Context KV Cache Compression", Detailed
Explanation); the oracle rebuilds K~, V~ explicitly (oracle/kvshare_ref.py) and
attends causally row by row. Codes and scales come from the packer on both sides
(bit-identical, checked elsewhere).
"""
import numpy as np
import pytest

import oracle.kvshare_ref as ref
import oracle.quant_ref as qr
from synth.configs import DEPTHWEAVE_DECODE, LOWRANK, MIX, SINGLE, Config

from gpu_helpers import assert_close, assert_scaled, to_dev

pytestmark = pytest.mark.gpu
TOL = 2e-2


@pytest.fixture(scope="module")
def K():
    from cross_layer_kv_shared_b200 import kvshare
    return kvshare


def make_inputs(cfg, lmap, slots, seed):
    """Low-rank tensors of a layer table that may also hold SINGLE / MIX layers."""
    lr = Config(cfg.name + "_lr", "prefill", layers=cfg.layers, q_heads=cfg.q_heads, kv_heads=cfg.kv_heads,
                head_dim=cfg.head_dim, batch=cfg.batch, context=cfg.context, dtype="bf16",
                layer_map=tuple((LOWRANK, max(0, s0), 0) for (_, s0, _) in lmap), pairs=cfg.pairs, seed=seed)
    inp = lr.make_all()
    if any(k != LOWRANK for k, _, _ in lmap):
        kv = Config(cfg.name + "_kv", "prefill", layers=cfg.layers, q_heads=cfg.q_heads, kv_heads=cfg.kv_heads,
                    head_dim=cfg.head_dim, batch=cfg.batch, context=cfg.context, dtype="bf16",
                    layer_map=((SINGLE, 0, 0),) * cfg.layers, slots=slots, seed=seed + 1000).make_all()
        inp.update(k=kv["k"], v=kv["v"], w=kv["w"])
    return inp


def run(K, cfg, lmap, slots, inp, S):
    import torch
    from test_gpu_lowrank import pack_gpu
    d = {n: to_dev(a, "bf16") for n, a in inp.items()}
    _, h = K.kvshare_create(cfg.layers, cfg.q_heads, cfg.kv_heads, cfg.head_dim, K.KVS_BF16, cfg.batch, cfg.context)
    try:
        K.kvshare_set_map(h, lmap, inp.get("w"))
        rank, ck, cv, sk, sv = pack_gpu(K, h, cfg, d["score"], d["u_k"], d["u_v"])
        out = torch.full((cfg.layers, cfg.batch, cfg.q_heads, S, cfg.head_dim), float("nan"), dtype=torch.bfloat16,
                         device="cuda")
        lse = torch.full((cfg.layers, cfg.batch, cfg.q_heads, S), float("nan"), device="cuda")
        cache = K.Cache(batch=cfg.batch, context=cfg.context, k=d.get("k"), v=d.get("v"), slots=slots,
                        coef_k=d["coef_k"], coef_v=d["coef_v"], basis_k=d["basis_k"], basis_v=d["basis_v"], u_k=ck,
                        u_v=cv, s_k=sk, s_v=sv, r_k=d["r_k"], r_v=d["r_v"], rank=rank, pairs=cfg.pairs)
        q = d["q"][:, :, :, :S].contiguous()
        n0 = K.kvshare_launch_count(h)
        K.kvshare_prefill(h, cache, q, out, lse, seqlen=S)
        st = K.kvshare_sync_status(h)
        assert st == K.KVS_OK, K.kvshare_status_string(st)
        launches = K.kvshare_launch_count(h) - n0
    finally:
        K.kvshare_destroy(h)
    o = out.view(torch.int16).cpu().numpy().view(np.uint16)
    return ref.bf16_bits_to_f64(o), lse.cpu().numpy(), launches


def oracle_getter(inp):
    rank, ck, cv, sk, sv = qr.pack_residual(inp["score"], inp["u_k"], inp["u_v"])
    arrs = {"coef_k": ref.bf16_bits_to_f64(inp["coef_k"]), "coef_v": ref.bf16_bits_to_f64(inp["coef_v"]),
            "basis_k": ref.bf16_bits_to_f64(inp["basis_k"]), "basis_v": ref.bf16_bits_to_f64(inp["basis_v"]),
            "u_k": ck.astype(np.float64), "u_v": cv.astype(np.float64),
            "s_k": ref.f16_bits_to_f64(sk), "s_v": ref.f16_bits_to_f64(sv),
            "r_k": ref.bf16_bits_to_f64(inp["r_k"]), "r_v": ref.bf16_bits_to_f64(inp["r_v"]), "rank": rank}
    if "k" in inp:
        arrs["k"] = ref.bf16_bits_to_f64(inp["k"])
        arrs["v"] = ref.bf16_bits_to_f64(inp["v"])
    return lambda name, index: arrs[name][index]


def base_cfg(name, L, Hq, Hkv, d, B, T, pairs):
    return Config(name, "prefill", layers=L, q_heads=Hq, kv_heads=Hkv, head_dim=d, batch=B, context=T, dtype="bf16",
                  layer_map=tuple((LOWRANK, l // 2, 0) for l in range(L)), pairs=pairs)


CASES = [
    # name, L, Hq, Hkv, d, B, T, S, layer map, slots
    ("lr_d128_g4", 2, 8, 2, 128, 2, 320, 300, [(LOWRANK, 0, 0), (LOWRANK, 0, 0)], 0),
    ("lr_d64_g16", 2, 16, 1, 64, 1, 257, 257, [(LOWRANK, 0, 0), (LOWRANK, 0, 0)], 0),
    ("lr_s1", 1, 4, 4, 128, 1, 64, 1, [(LOWRANK, 0, 0)], 0),
    ("lr_s513_g1", 2, 2, 2, 128, 1, 600, 513, [(LOWRANK, 0, 0), (LOWRANK, 0, 0)], 0),
    ("mixed_kinds", 4, 8, 2, 128, 1, 200, 200, [(SINGLE, 0, 0), (SINGLE, 1, 0), (MIX, 0, 1), (LOWRANK, 0, 0)], 2),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0])
def test_small_every_row(K, case):
    name, L, Hq, Hkv, d, B, T, S, lmap, slots = case
    cfg = base_cfg(name, L, Hq, Hkv, d, B, T, pairs=1)
    inp = make_inputs(cfg, lmap, slots, seed=91)
    out, lse, launches = run(K, cfg, lmap, slots, inp, S)
    lr_layers = sum(1 for k, _, _ in lmap if k == LOWRANK)
    assert launches == len(lmap) + lr_layers          # a projection pre-pass per low-rank layer
    get = oracle_getter(inp)
    rows = np.arange(S)
    worst = scale = 0.0
    for l in range(L):
        for b in range(B):
            for h in range(Hq):
                q = ref.bf16_bits_to_f64(inp["q"][l, b, h, :S])
                o, s = ref.prefill_rows(tuple(lmap), l, b, h, cfg.group, q, rows, get, w=inp.get("w"))
                worst = max(worst, assert_close(out[l, b, h], o, TOL, f"{name} l{l} b{b} h{h}")[0])
                assert_close(lse[l, b, h], s, TOL, f"{name} lse l{l} b{b} h{h}")
                scale = max(scale, float(np.max(np.abs(o))))
    print(f"{name}: worst max|d| {worst:.3e}, max|want| {scale:.3e}")
    assert_scaled(worst, scale, name)


def test_depthweave_shaped_4096(K):
    """The 64K-token model's head layout (32 q / 8 kv heads, d 128) on a 4096-token prefill of
    one layer pair: every layer and head at 32 rows, including the first and last of tiles."""
    c4 = DEPTHWEAVE_DECODE
    S = 4096
    cfg = base_cfg("lr_prefill_4096", 2, c4.q_heads, c4.kv_heads, c4.head_dim, 1, S, pairs=1)
    lmap = [(LOWRANK, 0, 0), (LOWRANK, 0, 0)]
    inp = make_inputs(cfg, lmap, 0, seed=93)
    out, lse, _ = run(K, cfg, lmap, 0, inp, S)
    get = oracle_getter(inp)
    rng = np.random.default_rng(94)
    rows = np.unique(np.concatenate([[0, 1, 63, 64, 127, 128, 255, 256, 2047, 4095], rng.integers(0, S, 22)]))
    worst = scale = 0.0
    for l in range(cfg.layers):
        for h in range(cfg.q_heads):
            q = ref.bf16_bits_to_f64(inp["q"][l, 0, h, rows])
            o, s = ref.prefill_rows(tuple(lmap), l, 0, h, cfg.group, q, rows, get)
            worst = max(worst, assert_close(out[l, 0, h, rows], o, TOL, f"l{l} h{h}")[0])
            scale = max(scale, float(np.max(np.abs(o))))
            assert_close(lse[l, 0, h, rows], s, TOL, f"lse l{l} h{h}")
    print(f"lowrank prefill 4096: worst max|d| {worst:.3e}, max|want| {scale:.3e}")
    assert_scaled(worst, scale, "lowrank prefill 4096")


def test_lowrank_prefill_needs_basis_rank_32(K):
    import torch
    _, h = K.kvshare_create(2, 4, 2, 64, K.KVS_BF16, 1, 64, basis_rank=64)
    try:
        K.kvshare_set_map(h, [(LOWRANK, 0, 0), (LOWRANK, 0, 0)], None)
        q = torch.zeros(2, 1, 4, 64, 64, dtype=torch.bfloat16, device="cuda")
        o = torch.zeros_like(q)
        buf = torch.zeros(1 << 20, dtype=torch.int16, device="cuda")
        cache = K.Cache(batch=1, context=64, coef_k=buf, coef_v=buf, basis_k=buf, basis_v=buf, u_k=buf, u_v=buf,
                        s_k=buf, s_v=buf, r_k=buf, r_v=buf, rank=buf, pairs=1)
        n0 = K.kvshare_launch_count(h)
        assert K.kvshare_prefill(h, cache, q, o, None, seqlen=64, check=False) == K.KVS_EUNSUPPORTED
        assert K.kvshare_launch_count(h) == n0
    finally:
        K.kvshare_destroy(h)
