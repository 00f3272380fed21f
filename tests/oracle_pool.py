"""Oracle units computed in a process pool, for the full-size sampled parity tests.

Each worker regenerates, on the host, only the seeded input slices one unit needs
(synth's counter-based generator, so any slice is reproducible on its own) and
evaluates the fp64 oracle on them. The pool is started with the `spawn` method,
so it is safe to create after CUDA has been initialised in the parent.
"""
import concurrent.futures as cf
import multiprocessing as mp
import os

import numpy as np


def _pool(n_jobs):
    workers = max(1, min(n_jobs, os.cpu_count() or 1, 32))
    return cf.ProcessPoolExecutor(max_workers=workers, mp_context=mp.get_context("spawn"))


def run(fn, args_list):
    """fn(*args) for every args tuple, in a spawn pool; results in input order."""
    if not args_list:
        return []
    with _pool(len(args_list)) as ex:
        return list(ex.map(fn, *zip(*args_list), chunksize=1))


# ---------------------------------------------------------------- decode, forms SINGLE / MIX
def decode_unit(cfg_name, l, b, j):
    """(o [g][d], lse [g]) of layer l, batch b, kv head j of a named workload."""
    from oracle import kvshare_ref as ref
    from synth.configs import BY_NAME
    cfg = BY_NAME[cfg_name]
    w = cfg.make("w")
    g = cfg.group
    q = ref.to_f64(cfg.make("q", (l, b))[j * g:(j + 1) * g], cfg.dtype)
    get = lambda name, index: ref.to_f64(cfg.make(name, index), cfg.dtype)  # noqa: E731
    return ref.decode_head_group(cfg.layer_map, l, b, j, q, get, w=w)


# ---------------------------------------------------------------- decode, low-rank form
def lowrank_unit(cfg_name, l, j):
    """Low-rank decode of layer l, kv head j at batch 0, with the packer rule run on the
    host: returns (o [g][d], lse [g], rank [T], codes_k [T][16], codes_v [T][16],
    scale_k bits [T], scale_v bits [T])."""
    from oracle import kvshare_ref as ref
    from oracle import quant_ref as qr
    from synth.configs import BY_NAME
    cfg = BY_NAME[cfg_name]
    p = l // 2
    g = cfg.group
    score = cfg.make("score", (l, 0))
    r = qr.route_rank(score)
    codes_k, sck = qr.quantize(cfg.make("u_k", (l, 0, j)), r)
    codes_v, scv = qr.quantize(cfg.make("u_v", (l, 0, j)), r)
    kv = []
    for s, codes, sc in (("k", codes_k, sck), ("v", codes_v, scv)):
        kv.append(ref.kv_lowrank(ref.bf16_bits_to_f64(cfg.make("coef_" + s, (p, 0, j))),
                                 ref.bf16_bits_to_f64(cfg.make("basis_" + s, (p, j))),
                                 ref.f16_bits_to_f64(sc), codes.astype(np.float64),
                                 ref.bf16_bits_to_f64(cfg.make("r_" + s, (l, j))), r))
    q = ref.bf16_bits_to_f64(cfg.make("q", (l, 0))[j * g:(j + 1) * g])
    o, lse, _ = ref.attend(q, kv[0], kv[1], 1 / np.sqrt(cfg.head_dim))
    return o, lse, r, codes_k, codes_v, sck, scv


def lowrank_stats_unit(cfg_name, l, j):
    """Attention statistics of layer l, kv head j at batch 0 of a named low-rank workload
    (codes and scales from the host packer): (mass [T], entropy [g], peak [g])."""
    from oracle import kvshare_ref as ref
    from oracle import quant_ref as qr
    from oracle import router_ref as rr
    from synth.configs import BY_NAME
    cfg = BY_NAME[cfg_name]
    p = l // 2
    g = cfg.group
    r = qr.route_rank(cfg.make("score", (l, 0)))
    kv = []
    for s in ("k", "v"):
        codes, sc = qr.quantize(cfg.make("u_" + s, (l, 0, j)), r)
        kv.append(ref.kv_lowrank(ref.bf16_bits_to_f64(cfg.make("coef_" + s, (p, 0, j))),
                                 ref.bf16_bits_to_f64(cfg.make("basis_" + s, (p, j))),
                                 ref.f16_bits_to_f64(sc), codes.astype(np.float64),
                                 ref.bf16_bits_to_f64(cfg.make("r_" + s, (l, j))), r))
    q = ref.bf16_bits_to_f64(cfg.make("q", (l, 0))[j * g:(j + 1) * g])
    _, _, pw = ref.attend(q, kv[0], kv[1], 1 / np.sqrt(cfg.head_dim))
    ent, peak = rr.attention_stats(pw)
    return rr.kv_mass(pw, g)[0], ent, peak


# ---------------------------------------------------------------- causal prefill
def prefill_unit(cfg_name, l, b, h, rows):
    """(o [n][d], lse [n]) of prefill layer l, batch b, q head h at the given rows."""
    from oracle import kvshare_ref as ref
    from synth.configs import BY_NAME
    cfg = BY_NAME[cfg_name]
    rows = np.asarray(rows)
    q = ref.bf16_bits_to_f64(cfg.make("q", (l, b, h)))[rows]
    get = lambda name, index: ref.bf16_bits_to_f64(cfg.make(name, index))  # noqa: E731
    return ref.prefill_rows(cfg.layer_map, l, b, h, cfg.group, q, rows, get, w=cfg.make("w"))
