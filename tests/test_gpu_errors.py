"""Host validation, unsupported combinations and the bounded device wait (no GPU fault)."""

import numpy as np
import pytest

from synth.configs import MIX, SINGLE, LOWRANK, TINY_CLA2

from gpu_helpers import make_ctx, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def K():
    from cross_layer_kv_shared_b200 import kvshare
    return kvshare


@pytest.fixture()
def setup(K):
    import torch
    cfg = TINY_CLA2
    inp = cfg.make_all()
    d = {n: to_dev(a, cfg.dtype) for n, a in inp.items()}
    h = make_ctx(K, cfg)
    K.kvshare_set_map(h, cfg.layer_map, None)
    out = torch.zeros(cfg.layers, cfg.batch, cfg.q_heads, cfg.head_dim, device="cuda")
    cache = K.Cache(batch=cfg.batch, context=cfg.context, k=d["k"], v=d["v"], slots=cfg.slots)
    yield cfg, h, d, out, cache
    K.kvshare_destroy(h)


def test_set_map_validation(K, setup):
    cfg, h, d, out, cache = setup
    L = cfg.layers
    ok = [(SINGLE, 0, 0)] * L
    assert K.kvshare_set_map(h, ok, None, check=False) == K.KVS_OK
    assert K.kvshare_set_map(h, [(MIX, 0, 1)] + ok[1:], None, check=False) == K.KVS_EINVAL        # no weights
    w = np.full((L, cfg.kv_heads), 0.5, np.float32)
    assert K.kvshare_set_map(h, [(MIX, 0, 0)] + ok[1:], w, check=False) == K.KVS_EINVAL          # src0 == src1
    w[0, 1] = 1.5
    assert K.kvshare_set_map(h, [(MIX, 0, 1)] + ok[1:], w, check=False) == K.KVS_EINVAL          # w > 1
    w[0, 1] = np.nan
    assert K.kvshare_set_map(h, [(MIX, 0, 1)] + ok[1:], w, check=False) == K.KVS_EINVAL          # NaN
    assert K.kvshare_set_map(h, [(7, 0, 0)] + ok[1:], None, check=False) == K.KVS_EINVAL          # kind
    assert K.kvshare_set_map(h, [(SINGLE, -1, 0)] + ok[1:], None, check=False) == K.KVS_EINVAL    # negative
    assert K.kvshare_set_map(h, [(LOWRANK, 0, 0)] + ok[1:], None, check=False) == K.KVS_EUNSUPPORTED  # fp32


def test_decode_validation_launches_nothing(K, setup):
    import torch
    cfg, h, d, out, cache = setup
    n0 = K.kvshare_launch_count(h)
    bad_slot = K.Cache(batch=1, context=cfg.context, k=d["k"], v=d["v"], slots=1)          # map reads slot 1
    assert K.kvshare_decode(h, bad_slot, d["q"], out, check=False) == K.KVS_EINVAL
    big = K.Cache(batch=1, context=cfg.context + 1, k=d["k"], v=d["v"], slots=2)          # > max_context
    assert K.kvshare_decode(h, big, d["q"], out, check=False) == K.KVS_EINVAL
    zero = K.Cache(batch=1, context=0, k=d["k"], v=d["v"], slots=2)
    assert K.kvshare_decode(h, zero, d["q"], out, check=False) == K.KVS_EINVAL
    assert K.kvshare_decode(h, cache, d["q"], out, l0=2, l1=1, check=False) == K.KVS_EINVAL
    assert K.kvshare_decode(h, cache, d["q"], out, l0=0, l1=5, check=False) == K.KVS_EINVAL
    mis = torch.zeros(out.numel() + 4, device="cuda")[1:]                                 # 4-byte offset
    assert K.kvshare_decode(h, cache, d["q"], mis, check=False) == K.KVS_EINVAL
    host_q = d["q"].cpu()
    assert K.kvshare_decode(h, cache, host_q, out, check=False) == K.KVS_EINVAL            # host pointer
    nokv = K.Cache(batch=1, context=cfg.context, k=None, v=d["v"], slots=2)
    assert K.kvshare_decode(h, nokv, d["q"], out, check=False) == K.KVS_EINVAL
    assert K.kvshare_launch_count(h) == n0
    assert K.kvshare_decode(h, cache, d["q"], out, check=False) == K.KVS_OK
    assert K.kvshare_launch_count(h) == n0 + cfg.layers
    assert K.kvshare_sync_status(h) == K.KVS_OK


def test_map_required_before_decode(K):
    import torch
    cfg = TINY_CLA2
    h = make_ctx(K, cfg)
    try:
        inp = cfg.make_all()
        d = {n: to_dev(a, cfg.dtype) for n, a in inp.items()}
        out = torch.zeros(cfg.layers, cfg.batch, cfg.q_heads, cfg.head_dim, device="cuda")
        cache = K.Cache(batch=1, context=cfg.context, k=d["k"], v=d["v"], slots=2)
        assert K.kvshare_decode(h, cache, d["q"], out, check=False) == K.KVS_EINVAL
    finally:
        K.kvshare_destroy(h)


def test_bounded_wait_reports_timeout_and_context_stays_usable(K, setup):
    cfg, h, d, out, cache = setup
    K.kvshare_debug_stall_next(h, True)
    assert K.kvshare_decode(h, cache, d["q"], out, l0=0, l1=1, check=False) == K.KVS_OK
    assert K.kvshare_sync_status(h) == K.KVS_ETIMEOUT
    # the hook clears itself, the status word was cleared, and the context still works
    assert K.kvshare_decode(h, cache, d["q"], out, check=False) == K.KVS_OK
    assert K.kvshare_sync_status(h) == K.KVS_OK


def test_bounded_wait_in_the_bf16_kernel(K):
    import torch
    cfg = TINY_CLA2.replace(dtype="bf16")
    inp = cfg.make_all()
    d = {n: to_dev(a, cfg.dtype) for n, a in inp.items()}
    h = make_ctx(K, cfg)
    try:
        K.kvshare_set_map(h, cfg.layer_map, None)
        out = torch.zeros(cfg.layers, cfg.batch, cfg.q_heads, cfg.head_dim, device="cuda")
        cache = K.Cache(batch=1, context=cfg.context, k=d["k"], v=d["v"], slots=2)
        K.kvshare_debug_stall_next(h, True)
        K.kvshare_decode(h, cache, d["q"], out)
        assert K.kvshare_sync_status(h) == K.KVS_ETIMEOUT
        K.kvshare_decode(h, cache, d["q"], out)
        assert K.kvshare_sync_status(h) == K.KVS_OK
    finally:
        K.kvshare_destroy(h)


def test_prefill_rejects_fp32_with_unsupported(K, setup):
    # the fp32 tiny workload: prefill runs on bf16 operands only
    cfg, h, d, out, cache = setup
    n0 = K.kvshare_launch_count(h)
    st = K.kvshare_prefill(h, cache, d["q"], out, None, 0, 1, seqlen=1, check=False)
    assert st == K.KVS_EUNSUPPORTED
    assert K.kvshare_launch_count(h) == n0


def prefill_ctx(K, layer_map, L=3, Hq=4, Hkv=2, d=64, T=32, w=None):
    import torch
    _, h = K.kvshare_create(L, Hq, Hkv, d, K.KVS_BF16, 1, T)
    w = np.full((L, Hkv), 0.5, np.float32) if w is None else w
    q = torch.zeros(L, 1, Hq, T, d, dtype=torch.bfloat16, device="cuda")
    o = torch.zeros_like(q)
    kv = torch.zeros(3, 1, Hkv, T, d, dtype=torch.bfloat16, device="cuda")
    cache = K.Cache(batch=1, context=T, k=kv, v=kv, slots=3)
    return h, q, o, cache, w


def test_prefill_lowrank_layer_needs_the_lowrank_arrays(K):
    # a low-rank layer is prefilled in the absorbed form; without its cache arrays the
    # call is rejected before any launch
    h, q, o, cache, w = prefill_ctx(K, None)
    try:
        K.kvshare_set_map(h, [(SINGLE, 0, 0), (SINGLE, 1, 0), (LOWRANK, 0, 0)], None)
        n0 = K.kvshare_launch_count(h)
        cache.pairs = 1
        st = K.kvshare_prefill(h, cache, q, o, None, 0, 3, seqlen=32, check=False)
        assert st == K.KVS_EINVAL
        assert K.kvshare_launch_count(h) == n0
    finally:
        K.kvshare_destroy(h)


@pytest.mark.parametrize("layer_map,ok", [
    ([(SINGLE, 0, 0), (SINGLE, 1, 0), (MIX, 0, 1)], True),      # both sources owned by shallower layers
    ([(SINGLE, 0, 0), (MIX, 0, 1), (SINGLE, 1, 0)], False),     # slot 1 is filled deeper than the target
    ([(SINGLE, 0, 0), (SINGLE, 0, 0), (MIX, 0, 2)], False),     # slot 2 has no owner at all
    ([(MIX, 0, 1), (SINGLE, 0, 0), (SINGLE, 1, 0)], False),     # both sources deeper
], ids=["owned", "deeper_source", "unowned_slot", "both_deeper"])
def test_prefill_mix_sources_must_be_owned_by_shallower_layers(K, layer_map, ok):
    h, q, o, cache, w = prefill_ctx(K, None)
    try:
        K.kvshare_set_map(h, layer_map, w)
        n0 = K.kvshare_launch_count(h)
        mix_l = [l for l, e in enumerate(layer_map) if e[0] == MIX][0]
        # the rule covers the map, so a call over the target layer alone is judged the same
        st = K.kvshare_prefill(h, cache, q, o, None, mix_l, mix_l + 1, seqlen=32, check=False)
        if ok:
            assert st == K.KVS_OK
            assert K.kvshare_launch_count(h) == n0 + 1
            assert K.kvshare_sync_status(h) == K.KVS_OK
        else:
            assert st == K.KVS_EINVAL
            assert K.kvshare_launch_count(h) == n0
    finally:
        K.kvshare_destroy(h)
