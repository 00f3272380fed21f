"""GPU parity of kvshare_prefill (tcgen05 causal attention, SINGLE and MIX layers) with the fp64 oracle."""
import numpy as np
import pytest

import oracle.kvshare_ref as ref
import synth.gpu as sgpu
from synth.configs import DEPTHGRAFT_PREFILL, MIX, SINGLE, Config

from gpu_helpers import assert_scaled, assert_close, to_dev

pytestmark = pytest.mark.gpu
TOL = 2e-2


@pytest.fixture(scope="module")
def K():
    from cross_layer_kv_shared_b200 import kvshare
    return kvshare


def pcfg(name, L, lmap, slots, Hq, Hkv, d, B, S, T=None, seed=5):
    return Config(name, "prefill", layers=L, q_heads=Hq, kv_heads=Hkv, head_dim=d, batch=B, context=T or S,
                  dtype="bf16", layer_map=tuple(lmap), slots=slots, seed=seed)


def run_prefill(K, cfg, inp, seqlen=None, dev=None):
    import torch
    S = seqlen or cfg.context
    d = dev or {n: to_dev(a, "bf16") for n, a in inp.items()}
    _, h = K.kvshare_create(cfg.layers, cfg.q_heads, cfg.kv_heads, cfg.head_dim, K.KVS_BF16, cfg.batch, cfg.context)
    try:
        K.kvshare_set_map(h, cfg.layer_map, inp["w"] if inp is not None else cfg.make("w"))
        out = torch.full((cfg.layers, cfg.batch, cfg.q_heads, S, cfg.head_dim), float("nan"),
                         dtype=torch.bfloat16, device="cuda")
        lse = torch.full((cfg.layers, cfg.batch, cfg.q_heads, S), float("nan"), device="cuda")
        cache = K.Cache(batch=cfg.batch, context=cfg.context, k=d["k"], v=d["v"], slots=cfg.slots)
        K.kvshare_prefill(h, cache, d["q"], out, lse, seqlen=S)
        st = K.kvshare_sync_status(h)
        assert st == K.KVS_OK, K.kvshare_status_string(st)
    finally:
        K.kvshare_destroy(h)
    o = out.view(torch.int16).cpu().numpy().view(np.uint16)
    return ref.bf16_bits_to_f64(o), lse.cpu().numpy()


def oracle_prefill(cfg, inp, S, layers=None, batches=None, heads=None, rows=None):
    get = lambda name, index: ref.bf16_bits_to_f64(inp[name][index])  # noqa: E731
    res = {}
    g = cfg.group
    rows = np.arange(S) if rows is None else np.asarray(rows)
    for l in (range(cfg.layers) if layers is None else layers):
        for b in (range(cfg.batch) if batches is None else batches):
            for h in (range(cfg.q_heads) if heads is None else heads):
                q = ref.bf16_bits_to_f64(inp["q"][l, b, h, rows])
                res[(l, b, h)] = ref.prefill_rows(cfg.layer_map, l, b, h, g, q, rows, get, w=inp["w"])
    return res


SMALL = [
    pcfg("pf_single_d128", 2, [(SINGLE, 0, 0), (SINGLE, 1, 0)], 2, 4, 2, 128, 1, 300),
    pcfg("pf_mix_d128", 3, [(SINGLE, 0, 0), (SINGLE, 1, 0), (MIX, 0, 1)], 2, 4, 2, 128, 2, 200),
    # a two-source target reads slots that shallower layers fill (own) in the same pass
    pcfg("pf_d64", 3, [(SINGLE, 1, 0), (SINGLE, 0, 0), (MIX, 1, 0)], 2, 8, 2, 64, 1, 257),
    pcfg("pf_s1", 3, [(SINGLE, 0, 0), (SINGLE, 1, 0), (MIX, 0, 1)], 2, 2, 1, 128, 1, 1),
    pcfg("pf_s128_ctx_longer", 3, [(SINGLE, 0, 0), (SINGLE, 1, 0), (MIX, 1, 0)], 2, 4, 4, 128, 1, 128, T=160),
]


@pytest.mark.parametrize("cfg", SMALL, ids=lambda c: c.name)
def test_small_every_row(K, cfg):
    inp = cfg.make_all()
    S = min(cfg.context, 300) if cfg.name != "pf_s128_ctx_longer" else 128
    inp["q"] = inp["q"][:, :, :, :S].copy()
    out, lse = run_prefill(K, cfg, inp, seqlen=S)
    want = oracle_prefill(cfg, inp, S)
    worst = 0.0
    for (l, b, h), (o, s) in want.items():
        worst = max(worst, assert_close(out[l, b, h], o, TOL, f"out l{l} b{b} h{h}")[0])
        assert_close(lse[l, b, h], s, TOL, f"lse l{l} b{b} h{h}")
    print(f"{cfg.name}: worst {worst:.3e}")


def test_prefill_row_equals_decode_over_prefix(K):
    """Row i of the causal prefill equals a decode step over tokens 0..i (both on the GPU)."""
    import torch
    cfg = SMALL[1]
    inp = cfg.make_all()
    S = cfg.context
    out, lse = run_prefill(K, cfg, inp)
    d = {n: to_dev(a, "bf16") for n, a in inp.items()}
    for i in (0, 63, 64, 127, 199):
        _, h = K.kvshare_create(cfg.layers, cfg.q_heads, cfg.kv_heads, cfg.head_dim, K.KVS_BF16, cfg.batch, S)
        try:
            K.kvshare_set_map(h, cfg.layer_map, inp["w"])
            kp = d["k"][:, :, :, :i + 1].contiguous()
            vp = d["v"][:, :, :, :i + 1].contiguous()
            qd = d["q"][:, :, :, i].contiguous()
            o = torch.empty(cfg.layers, cfg.batch, cfg.q_heads, cfg.head_dim, device="cuda")
            K.kvshare_decode(h, K.Cache(batch=cfg.batch, context=i + 1, k=kp, v=vp, slots=cfg.slots), qd, o)
            assert K.kvshare_sync_status(h) == K.KVS_OK
        finally:
            K.kvshare_destroy(h)
        assert np.max(np.abs(o.cpu().numpy() - out[:, :, :, i])) < 1e-2


def test_full_size_sampled(K):
    import torch
    cfg = DEPTHGRAFT_PREFILL
    dev = {n: sgpu.make_device(cfg, n) for n in cfg.recipe()}
    w = cfg.make("w")
    S = cfg.context
    _, h = K.kvshare_create(cfg.layers, cfg.q_heads, cfg.kv_heads, cfg.head_dim, K.KVS_BF16, cfg.batch, S)
    try:
        K.kvshare_set_map(h, cfg.layer_map, w)
        out = torch.empty((cfg.layers, cfg.batch, cfg.q_heads, S, cfg.head_dim), dtype=torch.bfloat16, device="cuda")
        lse = torch.empty((cfg.layers, cfg.batch, cfg.q_heads, S), device="cuda")
        cache = K.Cache(batch=cfg.batch, context=S, k=dev["k"], v=dev["v"], slots=cfg.slots)
        K.kvshare_prefill(h, cache, dev["q"], out, lse)
        assert K.kvshare_sync_status(h) == K.KVS_OK
    finally:
        K.kvshare_destroy(h)
    # every layer and q head of batch 0 and one seeded batch, at rows {0, 1, 127, 128,
    # 2047, 4095} plus 26 seeded rows
    rng = np.random.default_rng(99)
    rows = np.unique(np.concatenate([[0, 1, 127, 128, 2047, 4095], rng.integers(0, S, 26)]))
    batches = [0, int(rng.integers(1, cfg.batch))]
    import oracle_pool
    units = [(l, b, hh) for l in range(cfg.layers) for b in batches for hh in range(cfg.q_heads)]
    res = oracle_pool.run(oracle_pool.prefill_unit, [(cfg.name, l, b, hh, rows) for (l, b, hh) in units])
    out_h = out.view(torch.int16).cpu().numpy().view(np.uint16)
    lse_h = lse.cpu().numpy()
    worst = scale = 0.0
    for (l, b, hh), (o, s) in zip(units, res):
        got = ref.bf16_bits_to_f64(out_h[l, b, hh][rows])
        worst = max(worst, assert_close(got, o, TOL, f"l{l} b{b} h{hh}")[0])
        scale = max(scale, float(np.max(np.abs(o))))
        assert_close(lse_h[l, b, hh][rows], s, TOL, f"lse l{l} b{b} h{hh}")
    print(f"depthgraft_prefill: worst max|d| {worst:.3e}, max|want| {scale:.3e}")
    assert_scaled(worst, scale, "depthgraft_prefill")
