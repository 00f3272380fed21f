"""GPU parity of kvshare_decode (forms SINGLE and MIX) with the fp64 oracle, through the C ABI.

Tolerances: max|d| <= 1e-4 for fp32 caches, <= 2e-2 for bf16 caches (the stated
bars). Every test also reports the error relative to the output rms.
"""
import numpy as np
import pytest

from synth.configs import CLA2_1P1B, DEPTHGRAFT_DECODE, MIX, SINGLE, TINY_CLA2, Config
import synth.gpu as sgpu

from gpu_helpers import assert_scaled, assert_close, decode_gpu, oracle_decode, to_dev, make_ctx

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-4
TOL_BF16 = 2e-2


@pytest.fixture(scope="module")
def K():
    import torch
    assert torch.cuda.is_available()
    from cross_layer_kv_shared_b200 import kvshare
    return kvshare


def small(name, dtype, L, layer_map, slots, Hq, Hkv, d, B, T, scale=1.0, seed=7):
    return Config(name, "decode", layers=L, q_heads=Hq, kv_heads=Hkv, head_dim=d, batch=B, context=T, dtype=dtype,
                  layer_map=tuple(layer_map), slots=slots, qkv_scale=scale, seed=seed)


CLA_SMALL = small("cla2_small", "bf16", 4, [(SINGLE, l // 2, 0) for l in range(4)], 2, 32, 4, 64, 3, 333, 0.125)
DG_SMALL = small("depthgraft_small", "bf16", 6,
                 [(SINGLE, 0, 0), (SINGLE, 1, 0), (SINGLE, 2, 0), (SINGLE, 3, 0), (MIX, 0, 2), (MIX, 1, 3)],
                 4, 16, 4, 128, 2, 517)


def test_tiny_cla2_f32_every_output(K):
    inp = TINY_CLA2.make_all()
    out, lse, launches = decode_gpu(K, TINY_CLA2, inp)
    want, want_lse = oracle_decode(TINY_CLA2, inp)
    assert_close(out, want, TOL_F32, "out")
    assert_close(lse, want_lse, TOL_F32, "lse")
    assert launches == TINY_CLA2.layers


@pytest.mark.parametrize("cfg", [CLA_SMALL, DG_SMALL], ids=lambda c: c.name)
def test_reduced_bf16_every_output(K, cfg):
    inp = cfg.make_all()
    out, lse, _ = decode_gpu(K, cfg, inp)
    want, want_lse = oracle_decode(cfg, inp)
    _, rel = assert_close(out, want, TOL_BF16, "out")
    assert rel < 2e-2
    assert_close(lse, want_lse, TOL_BF16, "lse")


@pytest.mark.parametrize("dtype,d,g,T,mix", [
    ("bf16", 64, 1, 1, False), ("bf16", 64, 16, 15, False), ("bf16", 128, 4, 16, False),
    ("bf16", 128, 8, 1000, True), ("bf16", 64, 2, 4096, True), ("bf16", 128, 16, 33, True),
    ("bf16", 64, 8, 31, True), ("f32", 128, 4, 77, True), ("f32", 64, 3, 1, False), ("f32", 128, 1, 300, False),
])
def test_edge_shapes(K, dtype, d, g, T, mix):
    Hkv = 2
    lmap = [(SINGLE, 0, 0), (MIX, 0, 1) if mix else (SINGLE, 1, 0)]
    cfg = small(f"edge_{dtype}_{d}_{g}_{T}", dtype, 2, lmap, 2, g * Hkv, Hkv, d, 2, T, seed=11)
    inp = cfg.make_all()
    out, lse, _ = decode_gpu(K, cfg, inp)
    want, want_lse = oracle_decode(cfg, inp)
    tol = TOL_F32 if dtype == "f32" else TOL_BF16
    assert_close(out, want, tol, "out")
    assert_close(lse, want_lse, tol, "lse")


@pytest.mark.parametrize("cfg", [CLA_SMALL, DG_SMALL, TINY_CLA2], ids=lambda c: c.name)
def test_split_count_does_not_change_the_result(K, cfg):
    """fp32 caches agree to fp32 rounding. bf16 caches round each weight p to bf16
    against the split's own running max, so they agree to bf16 precision of the
    weights (relative 2^-8 of the output scale), well inside the 2e-2 bar."""
    inp = cfg.make_all()
    ref_out, ref_lse, _ = decode_gpu(K, cfg, inp, splits=1)
    rel = 1e-5 if cfg.dtype == "f32" else 2.0 ** -8
    for s in (2, 5, 0):
        out, lse, _ = decode_gpu(K, cfg, inp, splits=s)
        assert np.max(np.abs(out - ref_out)) <= rel * np.max(np.abs(ref_out))
        lse_tol = 1e-5 * max(1.0, np.max(np.abs(ref_lse))) if cfg.dtype == "f32" else 2.0 ** -8
        assert np.max(np.abs(lse - ref_lse)) <= lse_tol


@pytest.mark.parametrize("cfg", [CLA_SMALL, DG_SMALL], ids=lambda c: c.name)
@pytest.mark.parametrize("grid", [7, 13, 29, 100])
def test_grids_whose_ranges_straddle_units(K, cfg, grid):
    """CTA ranges that end inside one (batch, kv head) unit and start the next."""
    inp = cfg.make_all()
    out, lse, _ = decode_gpu(K, cfg, inp, grid=grid)
    want, want_lse = oracle_decode(cfg, inp)
    assert_close(out, want, TOL_BF16, "out")
    assert_close(lse, want_lse, TOL_BF16, "lse")


# other sharing topologies the layer table expresses: CLA3 / CLA4 groups reading the
# lowest layer of each group, a single-anchor map (the upper half reads one slot), and
# MQA (one kv head) at group sizes 8 and 16
OTHER_MAPS = [
    small("cla3", "bf16", 6, [(SINGLE, l // 3, 0) for l in range(6)], 2, 8, 2, 64, 2, 257, 0.125),
    small("cla4", "bf16", 8, [(SINGLE, l // 4, 0) for l in range(8)], 2, 16, 4, 128, 1, 300),
    small("single_anchor", "bf16", 6, [(SINGLE, 0, 0), (SINGLE, 1, 0), (SINGLE, 2, 0)] + [(SINGLE, 2, 0)] * 3,
          3, 8, 2, 64, 2, 200, 0.125),
    small("mqa_g8", "bf16", 2, [(SINGLE, 0, 0), (SINGLE, 0, 0)], 1, 8, 1, 128, 2, 333),
    small("mqa_g16", "bf16", 2, [(SINGLE, 0, 0), (MIX, 0, 1)], 2, 16, 1, 64, 1, 129),
]


@pytest.mark.parametrize("cfg", OTHER_MAPS, ids=lambda c: c.name)
def test_other_sharing_maps_every_output(K, cfg):
    inp = cfg.make_all()
    out, lse, launches = decode_gpu(K, cfg, inp)
    want, want_lse = oracle_decode(cfg, inp)
    assert_close(out, want, TOL_BF16, "out")
    assert_close(lse, want_lse, TOL_BF16, "lse")
    assert launches == cfg.layers


@pytest.mark.parametrize("cfg", [CLA_SMALL, DG_SMALL], ids=lambda c: c.name)
def test_kv_overlap_changes_nothing(K, cfg):
    # consecutive layers of one call overlap; with kv_overlap they also fetch K/V early
    inp = cfg.make_all()
    base, base_lse, _ = decode_gpu(K, cfg, inp)
    got, got_lse, _ = decode_gpu(K, cfg, inp, kv_overlap=True)
    assert np.array_equal(base, got) and np.array_equal(base_lse, got_lse)
    want, want_lse = oracle_decode(cfg, inp)
    assert_close(got, want, TOL_BF16, "out")


def test_cla_layers_sharing_a_slot_match_bitwise(K):
    cfg = CLA_SMALL
    inp = cfg.make_all()
    inp["q"] = inp["q"].copy()
    inp["q"][1] = inp["q"][0]              # layer 1 reuses layer 0's slot; same query
    out, lse, _ = decode_gpu(K, cfg, inp)
    assert np.array_equal(out[0], out[1]) and np.array_equal(lse[0], lse[1])


@pytest.mark.parametrize("cfg", [CLA_SMALL, DG_SMALL, TINY_CLA2], ids=lambda c: c.name)
def test_constant_values_give_constant_output(K, cfg):
    inp = cfg.make_all()
    one = np.float32(1.0)
    inp["v"] = (np.full(inp["v"].shape, 0x3F80, np.uint16) if cfg.dtype == "bf16"
                else np.full(inp["v"].shape, one, np.float32))
    out, _, _ = decode_gpu(K, cfg, inp)
    assert np.max(np.abs(out - 1.0)) < 1e-5


def test_mix_weight_endpoints_match_single_source(K):
    base = DG_SMALL
    inp = base.make_all()
    w = inp["w"].copy()
    w[4] = 1.0
    w[5] = 0.0
    inp["w"] = w
    out, _, _ = decode_gpu(K, base, inp, splits=1)
    single = base.replace(layer_map=base.layer_map[:4] + ((SINGLE, 0, 0), (SINGLE, 3, 0)))
    out_s, _, _ = decode_gpu(K, single, inp, splits=1)
    # same values up to the bf16 rounding of the weights p, which the two kernels
    # (different token tiles) take against different running maxima
    assert np.max(np.abs(out[4:] - out_s[4:])) <= 2.0 ** -8 * np.max(np.abs(out_s[4:]))


def test_layer_range_writes_only_its_rows(K):
    cfg = CLA_SMALL
    inp = cfg.make_all()
    out, lse, launches = decode_gpu(K, cfg, inp, layers=(1, 3))
    assert launches == 2
    assert np.all(np.isnan(out[0])) and np.all(np.isnan(out[3]))
    want, _ = oracle_decode(cfg, inp, layers=[1, 2])
    assert_close(out[1:3], want[1:3], TOL_BF16)


@pytest.mark.parametrize("order", ["model", "cold", "reversed"])
def test_decode_host_matches_device_call(K, order):
    # the host-buffer call, with the layers launched in model order, in the bench's cold
    # order or reversed: the same bits as the device call in model order
    import torch
    import bench
    cfg = DG_SMALL
    inp = cfg.make_all()
    out, lse, _ = decode_gpu(K, cfg, inp)
    d = {n: to_dev(a, cfg.dtype) for n, a in inp.items()}
    h = make_ctx(K, cfg)
    try:
        K.kvshare_set_map(h, cfg.layer_map, inp["w"])
        perm = {"model": None, "cold": bench.cold_order(cfg), "reversed": list(range(cfg.layers))[::-1]}[order]
        K.kvshare_set_layer_order(h, perm)
        qh = torch.from_numpy(np.ascontiguousarray(inp["q"]).view(np.int16)).pin_memory()
        oh = torch.full(out.shape, float("nan"), dtype=torch.float32).pin_memory()
        lh = torch.full(lse.shape, float("nan"), dtype=torch.float32).pin_memory()
        cache = K.Cache(batch=cfg.batch, context=cfg.context, k=d["k"], v=d["v"], slots=cfg.slots)
        for _ in range(2):     # a second call reuses the staging buffers
            K.kvshare_decode_host(h, cache, qh, oh, lh)
            assert K.kvshare_sync_status(h) == K.KVS_OK
            assert np.array_equal(oh.numpy(), out) and np.array_equal(lh.numpy(), lse)
        # a partial range in that order writes only its layers
        oh.fill_(float("nan"))
        K.kvshare_decode_host(h, cache, qh, oh, lh, 1, 3)
        assert K.kvshare_sync_status(h) == K.KVS_OK
        assert np.array_equal(oh.numpy()[1:3], out[1:3]) and np.all(np.isnan(oh.numpy()[0]))
    finally:
        K.kvshare_destroy(h)


def test_layer_order_validation(K):
    cfg = DG_SMALL
    h = make_ctx(K, cfg)
    try:
        L = cfg.layers
        assert K.kvshare_set_layer_order(h, [0] * L, check=False) == K.KVS_EINVAL          # repeated
        assert K.kvshare_set_layer_order(h, list(range(1, L + 1)), check=False) == K.KVS_EINVAL   # out of range
        assert K.kvshare_set_layer_order(h, list(range(L))[::-1], check=False) == K.KVS_OK
        assert K.kvshare_set_layer_order(h, None, check=False) == K.KVS_OK
    finally:
        K.kvshare_destroy(h)


# ----------------------------------------------------------------------------- full sizes, sampled
def _device_inputs(cfg):
    return {n: sgpu.make_device(cfg, n) for n in cfg.recipe()}


def _sampled_batches(cfg):
    """Batch 0 plus four seeded batches (all batches when there are at most four)."""
    if cfg.batch <= 4:
        return list(range(cfg.batch))
    rng = np.random.default_rng(cfg.seed)
    return [0] + sorted(int(x) for x in rng.choice(np.arange(1, cfg.batch), 4, replace=False))


@pytest.mark.parametrize("cfg", [CLA2_1P1B, DEPTHGRAFT_DECODE], ids=lambda c: c.name)
def test_full_size_sampled(K, cfg):
    # every layer and kv head (all query heads) of batch 0 and four seeded batches
    layers, batches = list(range(cfg.layers)), _sampled_batches(cfg)
    import torch
    d = _device_inputs(cfg)
    q_host = cfg.make("q")
    # the device generator reproduces the host bits
    assert np.array_equal(d["q"].view(torch.int16).cpu().numpy().view(np.uint16), q_host)
    w = cfg.make("w")
    h = make_ctx(K, cfg)
    try:
        K.kvshare_set_map(h, cfg.layer_map, w)
        out = torch.empty(cfg.layers, cfg.batch, cfg.q_heads, cfg.head_dim, device="cuda")
        lse = torch.empty(cfg.layers, cfg.batch, cfg.q_heads, device="cuda")
        cache = K.Cache(batch=cfg.batch, context=cfg.context, k=d["k"], v=d["v"], slots=cfg.slots)
        K.kvshare_decode(h, cache, d["q"], out, lse)
        assert K.kvshare_sync_status(h) == K.KVS_OK
        # the launch configuration bench.py times: per-layer calls in cold order, early
        # K/V requests across launches, captured once as a CUDA graph and replayed
        import bench
        K.kvshare_set_kv_overlap(h, True)
        out2 = torch.full_like(out, float("nan"))
        lse2 = torch.full_like(lse, float("nan"))
        order = bench.cold_order(cfg)
        for l in order:           # eager pass: attributes and tensor maps set up outside the capture
            K.kvshare_decode(h, cache, d["q"], out2, lse2, l, l + 1)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, capture_error_mode="thread_local"):
            cap = torch.cuda.current_stream()
            for l in order:
                K.kvshare_decode(h, cache, d["q"], out2, lse2, l, l + 1, cap)
        out2.fill_(float("nan"))
        graph.replay()
        graph.replay()
        torch.cuda.synchronize()
        assert K.kvshare_sync_status(h) == K.KVS_OK
        del graph
        assert torch.equal(out, out2) and torch.equal(lse, lse2)
    finally:
        K.kvshare_destroy(h)
    out = out.cpu().numpy()
    lse = lse.cpu().numpy()
    import oracle_pool
    units = [(l, b, j) for l in layers for b in batches for j in range(cfg.kv_heads)]
    res = oracle_pool.run(oracle_pool.decode_unit, [(cfg.name, l, b, j) for (l, b, j) in units])
    want = dict(zip(units, res))
    g = cfg.group
    worst = scale = 0.0
    for (l, b, j), (o, s) in want.items():
        got = out[l, b, j * g:(j + 1) * g]
        worst = max(worst, assert_close(got, o, TOL_BF16, f"l{l} b{b} j{j}")[0])
        scale = max(scale, float(np.max(np.abs(o))))
        assert_close(lse[l, b, j * g:(j + 1) * g], s, TOL_BF16, f"lse l{l} b{b} j{j}")
    print(f"{cfg.name}: worst max|d| {worst:.3e}, max|want| {scale:.3e}")
    assert_scaled(worst, scale, cfg.name)
