"""GPU parity of kvshare_append_lowrank (the write side of the low-rank form for a new token).

The shared coefficients, residual codes, scales and ranks the kernel writes are
compared bit for bit with oracle/encode_ref.py (the same fp32 sequence on both
sides); everything else in the cache must be left as it was; a decode over the
grown sequences then matches the fp64 oracle on the cache the oracle's own encode
produced.
"""
import numpy as np
import pytest

import oracle.encode_ref as er
import oracle.kvshare_ref as ref
import oracle.quant_ref as qr
from synth.configs import Config, depthweave_map

import code_layout as cl
from gpu_helpers import assert_close, to_dev

pytestmark = pytest.mark.gpu
TOL = 2e-2


@pytest.fixture(scope="module")
def K():
    from cross_layer_kv_shared_b200 import kvshare
    return kvshare


def layers_of_pair(cfg, p):
    ls = [l for l, (kind, s0, _) in enumerate(cfg.layer_map) if s0 == p]
    return ls[0], ls[-1]


def host_state(d, packed):
    """The device state on the host; the group-packed codes as dense [..., T, 16] by the stored ranks."""
    rank, ck, cv, sk, sv = packed
    r = rank.cpu().numpy().copy()
    return {"coef_k": d["coef_k"].cpu().numpy().view(np.uint16).copy(),
            "coef_v": d["coef_v"].cpu().numpy().view(np.uint16).copy(),
            "u_k": cl.unpack(ck.cpu().numpy(), r), "u_v": cl.unpack(cv.cpu().numpy(), r),
            "s_k": sk.cpu().numpy().view(np.uint16).copy(), "s_v": sv.cpu().numpy().view(np.uint16).copy(),
            "rank": r}


def oracle_append(cfg, state, inp, k_new, v_new, score, pos):
    """The oracle's encode of the new token written into a copy of the host state."""
    st = {k: v.copy() for k, v in state.items()}
    B, Hkv = cfg.batch, cfg.kv_heads
    for p in range(cfg.pairs):
        la, lb = layers_of_pair(cfg, p)
        for b in range(B):
            t = int(pos[b])
            if not 0 <= t < cfg.context:
                continue
            ra = int(qr.route_rank(score[la, b]))
            rb = int(qr.route_rank(score[lb, b]))
            for j in range(Hkv):
                for side, new in (("k", k_new), ("v", v_new)):
                    basis = er.bf16_bits_to_f32(inp["basis_" + side][p, j])
                    res = er.encode_pair(er.bf16_bits_to_f32(new[la, b, j]), er.bf16_bits_to_f32(new[lb, b, j]),
                                         basis, er.bf16_bits_to_f32(inp["r_" + side][la, j]),
                                         er.bf16_bits_to_f32(inp["r_" + side][lb, j]), ra, rb)
                    cb, _, c0, s0, _, c1, s1 = res
                    st["coef_" + side][p, b, j, t] = cb
                    st["u_" + side][la, b, j, t] = c0
                    st["s_" + side][la, b, j, t] = s0
                    st["u_" + side][lb, b, j, t] = c1
                    st["s_" + side][lb, b, j, t] = s1
            st["rank"][la, b, t] = ra
            st["rank"][lb, b, t] = rb
    return st


def make_case(seed, L=4, Hq=8, Hkv=2, d=128, B=3, T=64, Rb=32):
    cfg = Config("append", "decode", layers=L, q_heads=Hq, kv_heads=Hkv, head_dim=d, batch=B, context=T,
                 dtype="bf16", layer_map=depthweave_map(L), pairs=(L + 1) // 2, basis_rank=Rb, seed=seed)
    rng = np.random.default_rng(seed)
    new = lambda: er.f32_to_bf16_bits(rng.standard_normal((L, B, Hkv, d)).astype(np.float32))  # noqa: E731
    return cfg, new, rng


@pytest.mark.parametrize("shape", [dict(), dict(d=64, Hq=16, Hkv=1, Rb=32), dict(L=3, B=2, Hkv=4, Hq=16)],
                         ids=["d128", "d64_g16", "odd_layers"])
def test_append_is_bit_exact_and_decodes(K, shape):
    import torch
    from test_gpu_lowrank import pack_gpu
    cfg, new, rng = make_case(81, **shape)
    inp = cfg.make_all()
    d = {n: to_dev(a, "bf16") for n, a in inp.items()}
    _, h = K.kvshare_create(cfg.layers, cfg.q_heads, cfg.kv_heads, cfg.head_dim, K.KVS_BF16, cfg.batch,
                            cfg.context, basis_rank=cfg.basis_rank)
    try:
        K.kvshare_set_map(h, cfg.layer_map, None)
        packed = pack_gpu(K, h, cfg, d["score"], d["u_k"], d["u_v"])
        cache = K.Cache(batch=cfg.batch, context=cfg.context, coef_k=d["coef_k"], coef_v=d["coef_v"],
                        basis_k=d["basis_k"], basis_v=d["basis_v"], u_k=packed[1], u_v=packed[2], s_k=packed[3],
                        s_v=packed[4], r_k=d["r_k"], r_v=d["r_v"], rank=packed[0], pairs=cfg.pairs)
        state = host_state(d, packed)
        pos = np.array([10, cfg.context - 1, 0][:cfg.batch], np.int32)
        for step in range(2):                 # two appends in a row, the second one token later
            k_new, v_new = new(), new()
            score = rng.choice(np.array([0.1, 0.75, 0.95], np.float32), size=(cfg.layers, cfg.batch))
            n0 = K.kvshare_launch_count(h)
            K.kvshare_append_lowrank(h, cache, to_dev(k_new, "bf16"), to_dev(v_new, "bf16"),
                                     torch.from_numpy(score).cuda(), torch.from_numpy(pos).cuda())
            assert K.kvshare_sync_status(h) == K.KVS_OK
            assert K.kvshare_launch_count(h) == n0 + 1
            want = oracle_append(cfg, state, inp, k_new, v_new, score, pos)
            got = host_state(d, packed)
            for name in want:
                if name in ("u_k", "u_v"):
                    # codes of the tokens up to the append (later tokens of a code group
                    # move with the appended token's length: past the sequence, undefined)
                    for b in range(cfg.batch):
                        n = int(pos[b]) + 1
                        assert np.array_equal(got[name][:, b, :, :n], want[name][:, b, :, :n]), (step, name, b)
                else:
                    assert np.array_equal(got[name], want[name]), (step, name)
            state = want
            last = pos
            pos = np.minimum(pos + 1, cfg.context - 1)
        # decode over each sequence's tokens up to the last append (a token after it in
        # the same code group moved with the appended token's code length)
        lens = last + 1
        out = torch.empty(cfg.layers, cfg.batch, cfg.q_heads, cfg.head_dim, device="cuda")
        lse = torch.empty(cfg.layers, cfg.batch, cfg.q_heads, device="cuda")
        cache.lengths = torch.from_numpy(lens.astype(np.int32)).cuda()
        K.kvshare_decode(h, cache, d["q"], out, lse)
        assert K.kvshare_sync_status(h) == K.KVS_OK
    finally:
        K.kvshare_destroy(h)
    arrs = {"coef_k": ref.bf16_bits_to_f64(state["coef_k"]), "coef_v": ref.bf16_bits_to_f64(state["coef_v"]),
            "basis_k": ref.bf16_bits_to_f64(inp["basis_k"]), "basis_v": ref.bf16_bits_to_f64(inp["basis_v"]),
            "u_k": state["u_k"].astype(np.float64), "u_v": state["u_v"].astype(np.float64),
            "s_k": ref.f16_bits_to_f64(state["s_k"]), "s_v": ref.f16_bits_to_f64(state["s_v"]),
            "r_k": ref.bf16_bits_to_f64(inp["r_k"]), "r_v": ref.bf16_bits_to_f64(inp["r_v"]), "rank": state["rank"]}
    o, l = ref.decode(cfg.layer_map, ref.bf16_bits_to_f64(inp["q"]), lambda n, i: arrs[n][i], lengths=lens)
    _, rel = assert_close(out.cpu().numpy(), o, TOL, "decode after append")
    assert rel < 2e-2
    assert_close(lse.cpu().numpy(), l, TOL, "lse after append")


def test_append_rejects_positions_outside_the_store(K):
    import torch
    from test_gpu_lowrank import pack_gpu
    cfg, new, rng = make_case(82, B=2)
    inp = cfg.make_all()
    d = {n: to_dev(a, "bf16") for n, a in inp.items()}
    _, h = K.kvshare_create(cfg.layers, cfg.q_heads, cfg.kv_heads, cfg.head_dim, K.KVS_BF16, cfg.batch, cfg.context)
    try:
        K.kvshare_set_map(h, cfg.layer_map, None)
        packed = pack_gpu(K, h, cfg, d["score"], d["u_k"], d["u_v"])
        cache = K.Cache(batch=cfg.batch, context=cfg.context, coef_k=d["coef_k"], coef_v=d["coef_v"],
                        basis_k=d["basis_k"], basis_v=d["basis_v"], u_k=packed[1], u_v=packed[2], s_k=packed[3],
                        s_v=packed[4], r_k=d["r_k"], r_v=d["r_v"], rank=packed[0], pairs=cfg.pairs)
        before = host_state(d, packed)
        score = torch.full((cfg.layers, cfg.batch), 0.95, device="cuda")
        pos = torch.tensor([cfg.context, -1], dtype=torch.int32, device="cuda")
        K.kvshare_append_lowrank(h, cache, to_dev(new(), "bf16"), to_dev(new(), "bf16"), score, pos)
        assert K.kvshare_sync_status(h) == K.KVS_EINVAL
        after = host_state(d, packed)
        for name in before:
            assert np.array_equal(before[name], after[name]), name
        # validation before any launch: a host pointer, and a layer table without low-rank layers
        n0 = K.kvshare_launch_count(h)
        st = K.kvshare_append_lowrank(h, cache, to_dev(new(), "bf16"), to_dev(new(), "bf16"), score, pos.cpu(),
                                      check=False)
        assert st == K.KVS_EINVAL
        K.kvshare_set_map(h, [(0, 0, 0)] * cfg.layers, None)
        st = K.kvshare_append_lowrank(h, cache, to_dev(new(), "bf16"), to_dev(new(), "bf16"), score, pos,
                                      check=False)
        assert st == K.KVS_EINVAL
        assert K.kvshare_launch_count(h) == n0
    finally:
        K.kvshare_destroy(h)
