"""kvshare_decode_layer_noalloc: the decode entry point for callers that cannot allocate.

Some callers cannot call cudaMalloc: work recorded into a capture they do not
own, plug-ins of a framework whose allocator must hand out all device memory,
or processes whose footprint may not grow after start-up. For them the library
offers one decode layer whose scratch (split partials, arrival counters, status
word) lives in a fixed device array inside the library instead of a context
workspace. These checks call it through the C ABI and compare it with the fp64
oracle, twice in a row, since every call reuses the array the previous one
left; they also compare it with kvshare_decode, which runs the same kernel. The
file sorts last so a run that stops at the first failure has already run every
other test; it also passes on its own in a fresh process (the first call looks
up the array's address).
"""
import numpy as np
import pytest

import oracle.kvshare_ref as ref
from synth.configs import MIX, SINGLE, Config

pytestmark = pytest.mark.gpu
TOL = 2e-2


def run_case(cfg):
    import torch
    from cross_layer_kv_shared_b200 import kvshare as K

    inp = cfg.make_all()
    to_dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16) if a.dtype == np.uint16 else a).cuda()  # noqa: E731
    q, k, v = to_dev(inp["q"]), to_dev(inp["k"]), to_dev(inp["v"])
    w_all = inp["w"]
    get = lambda name, index: ref.bf16_bits_to_f64(inp[name][index])  # noqa: E731
    want, want_lse = ref.decode(cfg.layer_map, ref.bf16_bits_to_f64(inp["q"]), get, w=w_all)
    rms = float(np.sqrt(np.mean(want ** 2)))

    # the context entry point on the same inputs: the same kernel, so the same bits
    _, h = K.kvshare_create(cfg.layers, cfg.q_heads, cfg.kv_heads, cfg.head_dim, K.KVS_BF16, cfg.batch, cfg.context)
    try:
        K.kvshare_set_map(h, cfg.layer_map, w_all)
        ctx_out = torch.empty(cfg.layers, cfg.batch, cfg.q_heads, cfg.head_dim, device="cuda")
        ctx_lse = torch.empty(cfg.layers, cfg.batch, cfg.q_heads, device="cuda")
        K.kvshare_decode(h, K.Cache(batch=cfg.batch, context=cfg.context, k=k, v=v, slots=cfg.slots), q,
                         ctx_out, ctx_lse)
        assert K.kvshare_sync_status(h) == K.KVS_OK
    finally:
        K.kvshare_destroy(h)

    for call in range(2):
        got = torch.full_like(ctx_out, float("nan"))
        got_lse = torch.full_like(ctx_lse, float("nan"))
        for l, (kind, s0, s1) in enumerate(cfg.layer_map):
            w_dev = torch.from_numpy(np.ascontiguousarray(w_all[l])).cuda() if kind == MIX else None
            K.kvshare_decode_layer_noalloc(q[l], k, v, w_dev, got[l], got_lse[l], cfg.batch, cfg.q_heads,
                                           cfg.kv_heads, cfg.head_dim, cfg.context, cfg.slots, s0,
                                           s1 if kind == MIX else -1)
        torch.cuda.synchronize()
        o, s = got.cpu().numpy(), got_lse.cpu().numpy()
        assert np.all(np.isfinite(o)) and np.all(np.isfinite(s)), f"call {call}"
        err = float(np.max(np.abs(o - want)))
        assert err <= TOL and err <= TOL * rms, f"call {call}: max|d| {err:.3e}, rms {rms:.3e}"
        assert float(np.max(np.abs(s - want_lse))) <= TOL, f"call {call}"
        assert torch.equal(got, ctx_out) and torch.equal(got_lse, ctx_lse), f"call {call}"


def test_no_alloc_matches_the_oracle_on_two_calls_in_a_row():
    cfg = Config("noalloc_check", "decode", layers=2, q_heads=16, kv_heads=4, head_dim=128, batch=2, context=517,
                 dtype="bf16", layer_map=((SINGLE, 0, 0), (MIX, 0, 1)), slots=2, seed=77)
    run_case(cfg)


def test_no_alloc_largest_partial_footprint():
    # 74 units of a 16-head group at d = 128, two CTAs per unit on 148 SMs: 222 partial
    # slots of 16 x 132 floats, the most the default grid writes (1.9 of the 2 MiB)
    cfg = Config("noalloc_full", "decode", layers=2, q_heads=32, kv_heads=2, head_dim=128, batch=37, context=300,
                 dtype="bf16", layer_map=((SINGLE, 0, 0), (MIX, 1, 0)), slots=2, seed=78)
    run_case(cfg)


def test_no_alloc_rejects_more_units_than_its_array_holds():
    import torch
    from cross_layer_kv_shared_b200 import kvshare as K

    buf = torch.zeros(1024, device="cuda")
    st = K.kvshare_decode_layer_noalloc(buf, buf, buf, None, buf, None, 4097, 8, 1, 64, 16, 1, 0, -1, check=False)
    assert st == K.KVS_EINVAL
    host = torch.zeros(1024).pin_memory()
    st = K.kvshare_decode_layer_noalloc(host, buf, buf, None, buf, None, 1, 8, 1, 64, 16, 1, 0, -1, check=False)
    assert st == K.KVS_EINVAL
