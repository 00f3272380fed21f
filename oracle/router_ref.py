"""Attention statistics of one decode step and the online rank router (test infrastructure).

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may use this.

The pages give the router's inputs and purpose but not its formula
("DepthWeave-KV: Smarter KV Cache Compression by Sharing Across Layers and
Adapting Per Token", Core Mechanism, second component: the router reads
attention statistics, entropy and peak scores, gives retrieval-critical tokens a
higher-rank residual, and runs online during generation; Key Concepts,
Token-Conditional Depth Routing: low entropy means focused attention, the
decision is made per token and per generation step). Readings evaluated here,
all from the softmax weights p of ``kvshare_ref.attend``:

* per query head h: entropy H_h = -sum_t p_{h,t} ln p_{h,t} (nats, 0 ln 0 = 0) and
  peak P_h = max_t p_{h,t}: how focused that head's attention is;
* per kv head j and cached token t: the attention mass the token receives from
  the g query heads that read kv head j, A_{j,t} = sum_{h in group j} p_{h,t}
  (sums to g over t);
* the router score of token t, shared by all kv heads and by K and V like its
  rank: the token's share of all Hq heads' attention against a uniform share,
  x = T * (sum_j A_{j,t}) / Hq, mapped monotonically into [0, 1) by
  score = x / (1 + x). A token at the uniform share scores 0.5 and keeps rank 0;
  the rank rule of ``quant_ref.route_rank`` (0.7 / 0.9) gives rank 8 from 7/3
  times the uniform share and rank 16 from 9 times. The map is evaluated in fp32
  in the stated order (sum over j from 0 up, then the product with T, the
  division by Hq, the addition of one and the final division, each correctly
  rounded), so a score computed from the same fp32 masses decides the same rank.

Statistics are fp64 from the fp64 weights; only ``route_score`` is fp32.
"""
from __future__ import annotations

import numpy as np


def attention_stats(p):
    """Entropy (nats) and peak of each row of softmax weights p [n, T]."""
    p = np.atleast_2d(np.asarray(p, dtype=np.float64))
    with np.errstate(divide="ignore", invalid="ignore"):
        terms = np.where(p > 0.0, -p * np.log(p), 0.0)
    return np.sum(terms, axis=1), np.max(p, axis=1)


def kv_mass(p, g: int):
    """Attention mass per kv head and token: p [Hq, T] (contiguous groups of g) -> [Hq // g, T]."""
    p = np.asarray(p, dtype=np.float64)
    Hq, T = p.shape
    return p.reshape(Hq // g, g, T).sum(axis=1)


def route_score(mass, context: int, num_q_heads: int):
    """fp32 router score per token: x = (T * sum_j mass_j) / Hq, score = x / (1 + x)."""
    m = np.asarray(mass, dtype=np.float32)
    total = m[0].copy()
    for j in range(1, m.shape[0]):
        total = (total + m[j]).astype(np.float32)
    x = (np.float32(context) * total).astype(np.float32)
    x = (x / np.float32(num_q_heads)).astype(np.float32)
    return (x / (np.float32(1.0) + x).astype(np.float32)).astype(np.float32)


def decode_stats(layer_map, q, get, w=None, scale=None, layers=None, batches=None, kv_heads=None,
                 lengths=None):
    """Statistics of a full decode step.

    q [L][B][Hq][d] fp64 -> mass [L][B][Hkv][T], entropy [L][B][Hq], peak [L][B][Hq];
    ``get``, ``w`` and ``lengths`` as in ``kvshare_ref.decode``. Tokens at or past a
    sequence's length receive no mass; a sequence with no tokens has entropy 0 and
    peak 0. Rows not computed are NaN.
    """
    from . import kvshare_ref as ref
    q = np.asarray(q, dtype=np.float64)
    L, B, Hq, d = q.shape
    sc = 1.0 / np.sqrt(d) if scale is None else scale
    mass = ent = peak = None
    for l in (range(L) if layers is None else layers):
        for b in (range(B) if batches is None else batches):
            Hkv = kv_heads or ref._kv_heads(get, layer_map, l)
            g = Hq // Hkv
            for j in range(Hkv):
                K, V = ref.layer_kv(layer_map, l, b, j, get, w)
                if mass is None:
                    T = K.shape[0]
                    mass = np.full((L, B, Hkv, T), np.nan)
                    ent = np.full((L, B, Hq), np.nan)
                    peak = np.full((L, B, Hq), np.nan)
                n = K.shape[0] if lengths is None else int(lengths[b])
                mass[l, b, j] = 0.0
                if n == 0:
                    ent[l, b, j * g:(j + 1) * g] = 0.0
                    peak[l, b, j * g:(j + 1) * g] = 0.0
                    continue
                _, _, p = ref.attend(q[l, b, j * g:(j + 1) * g], K[:n], V[:n], sc)
                e, pk = attention_stats(p)
                ent[l, b, j * g:(j + 1) * g] = e
                peak[l, b, j * g:(j + 1) * g] = pk
                mass[l, b, j, :n] = kv_mass(p, g)[0]
    return mass, ent, peak
