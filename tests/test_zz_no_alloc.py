"""kvshare_decode_layer_noalloc: the decode entry point for callers that cannot allocate.

Some callers cannot call cudaMalloc (work inside a capture or a framework whose
allocator owns all device memory). For them the library offers one decode
layer whose scratch lives in a fixed device array instead of a context
workspace. These checks call it through the C ABI and compare it with
kvshare_decode on the same inputs, twice in a row, since every call reuses the
array left by the previous one. The file sorts last so a run that stops at the
first failure has already run every other test; it also passes on its own in a
fresh process (the first call sets up the array's address).
"""
import numpy as np
import pytest

from synth.configs import MIX, SINGLE, Config

pytestmark = pytest.mark.gpu
TOL = 2e-2


def test_no_alloc_matches_the_context_decode_on_two_calls_in_a_row():
    import torch
    from cross_layer_kv_shared_b200 import kvshare as K

    cfg = Config("noalloc_check", "decode", layers=2, q_heads=16, kv_heads=4, head_dim=128, batch=2, context=517,
                 dtype="bf16", layer_map=((SINGLE, 0, 0), (MIX, 0, 1)), slots=2, seed=77)
    inp = cfg.make_all()
    to_dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16) if a.dtype == np.uint16 else a).cuda()  # noqa: E731
    q, k, v = to_dev(inp["q"]), to_dev(inp["k"]), to_dev(inp["v"])
    w_all = inp["w"]

    # the existing entry point (context workspace)
    _, h = K.kvshare_create(cfg.layers, cfg.q_heads, cfg.kv_heads, cfg.head_dim, K.KVS_BF16, cfg.batch, cfg.context)
    try:
        K.kvshare_set_map(h, cfg.layer_map, w_all)
        want = torch.empty(cfg.layers, cfg.batch, cfg.q_heads, cfg.head_dim, device="cuda")
        want_lse = torch.empty(cfg.layers, cfg.batch, cfg.q_heads, device="cuda")
        K.kvshare_decode(h, K.Cache(batch=cfg.batch, context=cfg.context, k=k, v=v, slots=cfg.slots), q, want, want_lse)
        assert K.kvshare_sync_status(h) == K.KVS_OK
    finally:
        K.kvshare_destroy(h)

    w_dev = torch.from_numpy(np.ascontiguousarray(w_all[1])).cuda()   # weights of the mixing layer
    for call in range(2):
        got = torch.full_like(want, float("nan"))
        got_lse = torch.full_like(want_lse, float("nan"))
        for l, (kind, s0, s1) in enumerate(cfg.layer_map):
            K.kvshare_decode_layer_noalloc(q[l], k, v, w_dev if kind == MIX else None, got[l], got_lse[l],
                                           cfg.batch, cfg.q_heads, cfg.kv_heads, cfg.head_dim, cfg.context,
                                           cfg.slots, s0, s1 if kind == MIX else -1)
        torch.cuda.synchronize()
        assert torch.isfinite(got).all() and torch.isfinite(got_lse).all(), f"call {call}"
        assert float((got - want).abs().max()) <= TOL, f"call {call}"
        assert float((got_lse - want_lse).abs().max()) <= TOL, f"call {call}"


def test_no_alloc_rejects_more_units_than_its_array_holds():
    import torch
    from cross_layer_kv_shared_b200 import kvshare as K

    buf = torch.zeros(1024, device="cuda")
    st = K.kvshare_decode_layer_noalloc(buf, buf, buf, None, buf, None, 4097, 8, 1, 64, 16, 1, 0, -1, check=False)
    assert st == K.KVS_EINVAL
