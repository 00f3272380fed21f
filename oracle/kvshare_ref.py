"""fp64 definition of attention over a cross-layer shared KV cache (test infrastructure).

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may use this.

What the method computes, and where the pages say so:

* A layer either computes its own K/V or reads another layer's ("Reducing
  Transformer Key-Value Cache Size with Cross-Layer Attention", Methodology:
  some layers compute new KV, the others reuse it; sharing factors CLA2/3/4).
  Query heads share kv heads within a layer (same page, Abstract: MQA/GQA).
* A deep target layer's K/V is rebuilt from a stride-aligned shallow/middle
  source pair ("DepthGraft: Structural Regularization through Hierarchical
  Cross-Layer KV Reconstruction", Abstract). The pages give no operator; the
  reading used here is a convex mix per (target layer, kv head):
  K = w*K_s1 + (1-w)*K_s2, and the same w for V.
* A layer pair shares a low-rank channel basis and each layer adds its own
  low-rank, quantised residual at a per-token rank a router picks
  ("DepthWeave-KV: Smarter KV Cache Compression by Sharing Across Layers and
  Adapting Per Token", Core Mechanism and Framework Shift). Reading used here:
  K_t = sum_i C[t,i] B[i,:] + s_t * sum_{i < r_t} U[t,i] R[i,:], separate
  B/R/C/U/s for K and V, coefficients shared by the two layers of a pair,
  residual per layer, rank per (layer, batch, token).
* Attention itself is standard softmax attention over the rebuilt K/V with
  scale 1/sqrt(d); decode sees every cached token, causal prefill row i sees
  tokens 0..i.

Everything is evaluated in fp64 from the stored bits (bf16, fp16 and int8
convert to fp64 exactly), with no blocking, splitting or reordering.
"""
from __future__ import annotations

import numpy as np

SINGLE, MIX, LOWRANK = 0, 1, 2


# ----------------------------------------------------------------------------- storage decoding
def bf16_bits_to_f64(bits) -> np.ndarray:
    """bf16 bit patterns (uint16) -> exact fp64 values."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def f16_bits_to_f64(bits) -> np.ndarray:
    """IEEE half bit patterns (uint16) -> exact fp64 values."""
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def to_f64(x, dtype: str) -> np.ndarray:
    """Stored tensor -> fp64: 'bf16' holds uint16 bit patterns, 'f32' float32 values."""
    if dtype == "bf16":
        return bf16_bits_to_f64(x)
    return np.asarray(x, dtype=np.float64)


# ----------------------------------------------------------------------------- layer map
def resolve(layer_map, l: int):
    """Layer-to-source table lookup: (kind, src0, src1) of layer ``l``.

    SINGLE reads store slot src0; MIX reads slots src0 and src1; LOWRANK reads
    basis pair src0 and the layer's own residual (index l).
    """
    kind, s0, s1 = layer_map[l]
    return int(kind), int(s0), int(s1)


# ----------------------------------------------------------------------------- reconstruction
def kv_single(K_src: np.ndarray) -> np.ndarray:
    """Form (a): the layer attends over the source slot's K (or V) unchanged."""
    return np.asarray(K_src, dtype=np.float64)


def kv_mix(w: float, K1: np.ndarray, K2: np.ndarray) -> np.ndarray:
    """Form (b): convex mix of the two sources, w*K1 + (1-w)*K2."""
    w = float(w)
    return w * np.asarray(K1, dtype=np.float64) + (1.0 - w) * np.asarray(K2, dtype=np.float64)


def kv_lowrank(C: np.ndarray, Bas: np.ndarray, s: np.ndarray, U: np.ndarray,
               R: np.ndarray, r: np.ndarray) -> np.ndarray:
    """Form (c): shared-basis part plus the layer's scaled low-rank residual at rank r_t.

    C [T, Rb] coefficients, Bas [Rb, d] basis, s [T] per-token scale,
    U [T, Rm] residual codes, R [Rm, d] residual factor, r [T] per-token rank.
    Row t = sum_i C[t,i] Bas[i] + s[t] * sum_{i < r[t]} U[t,i] R[i].
    """
    C = np.asarray(C, dtype=np.float64)
    U = np.asarray(U, dtype=np.float64)
    Rm = U.shape[1]
    keep = np.arange(Rm)[None, :] < np.asarray(r, dtype=np.int64)[:, None]
    Um = np.where(keep, U, 0.0) * np.asarray(s, dtype=np.float64)[:, None]
    return C @ np.asarray(Bas, dtype=np.float64) + Um @ np.asarray(R, dtype=np.float64)


# ----------------------------------------------------------------------------- attention
def attend(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float, visible=None):
    """Softmax attention of query rows q [n, d] over K, V [T, d].

    z = (q . K_t) * scale;  p = exp(z - max z) / sum exp(z - max z);
    o = sum_t p_t V_t;  lse = max z + ln sum exp(z - max z).
    ``visible`` (optional) is the number of visible tokens per row (causal rows
    pass i+1); tokens at or after it get no weight.
    Returns (o [n, d], lse [n], p [n, T]).
    """
    q = np.atleast_2d(np.asarray(q, dtype=np.float64))
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    z = (q @ K.T) * float(scale)
    if visible is not None:
        vis = np.asarray(visible, dtype=np.int64).reshape(-1, 1)
        z = np.where(np.arange(K.shape[0])[None, :] < vis, z, -np.inf)
    m = np.max(z, axis=1, keepdims=True)
    e = np.exp(z - m)
    den = np.sum(e, axis=1, keepdims=True)
    p = e / den
    o = p @ V
    lse = (m + np.log(den))[:, 0]
    return o, lse, p


def layer_kv(layer_map, l: int, b: int, j: int, get, w=None):
    """Rebuilt (K, V) [T, d] of layer l, batch b, kv head j.

    ``get(name, index)`` returns the stored tensor ``name`` indexed by the tuple
    ``index`` (the test's seeded generator or a dict of arrays); names follow the
    cache fields: k, v, coef_k, coef_v, basis_k, basis_v, u_k, u_v, s_k, s_v,
    r_k, r_v, rank, with dtype tags resolved by ``get``.
    """
    kind, s0, s1 = resolve(layer_map, l)
    if kind == SINGLE:
        return kv_single(get("k", (s0, b, j))), kv_single(get("v", (s0, b, j)))
    if kind == MIX:
        wj = float(w[l][j])
        return (kv_mix(wj, get("k", (s0, b, j)), get("k", (s1, b, j))),
                kv_mix(wj, get("v", (s0, b, j)), get("v", (s1, b, j))))
    if kind == LOWRANK:
        r = get("rank", (l, b))
        K = kv_lowrank(get("coef_k", (s0, b, j)), get("basis_k", (s0, j)), get("s_k", (l, b, j)),
                       get("u_k", (l, b, j)), get("r_k", (l, j)), r)
        V = kv_lowrank(get("coef_v", (s0, b, j)), get("basis_v", (s0, j)), get("s_v", (l, b, j)),
                       get("u_v", (l, b, j)), get("r_v", (l, j)), r)
        return K, V
    raise ValueError(f"unknown layer kind {kind}")


def decode_head_group(layer_map, l, b, j, q_group, get, w=None, scale=None, length=None):
    """Decode outputs of the q heads of kv head j: q_group [g, d] -> (o [g, d], lse [g]).

    ``length`` (optional) is the sequence's own token count: only cached tokens
    0 .. length-1 are attended to. A sequence with no tokens has an empty softmax:
    its outputs are 0 and its lse is -inf.
    """
    K, V = layer_kv(layer_map, l, b, j, get, w)
    if length is not None:
        K, V = K[:int(length)], V[:int(length)]
    q_group = np.atleast_2d(q_group)
    if K.shape[0] == 0:
        return np.zeros((q_group.shape[0], V.shape[1])), np.full(q_group.shape[0], -np.inf)
    d = K.shape[1]
    sc = 1.0 / np.sqrt(d) if scale is None else scale
    o, lse, _ = attend(q_group, K, V, sc)
    return o, lse


def decode(layer_map, q, get, w=None, scale=None, layers=None, batches=None, lengths=None):
    """Full decode step: q [L][B][Hq][d] (fp64) -> out [L][B][Hq][d], lse [L][B][Hq].

    Query head h reads kv head h // g (contiguous GQA groups). ``lengths`` [B]
    (optional) gives each sequence's own token count; without it every sequence
    attends to all cached tokens.
    """
    q = np.asarray(q, dtype=np.float64)
    L, B, Hq, d = q.shape
    out = np.full((L, B, Hq, d), np.nan)
    lse = np.full((L, B, Hq), np.nan)
    Hkv = None
    for l in (range(L) if layers is None else layers):
        for b in (range(B) if batches is None else batches):
            if Hkv is None:
                Hkv = _kv_heads(get, layer_map, l)
            g = Hq // Hkv
            for j in range(Hkv):
                o, s = decode_head_group(layer_map, l, b, j, q[l, b, j * g:(j + 1) * g], get, w, scale,
                                         None if lengths is None else lengths[b])
                out[l, b, j * g:(j + 1) * g] = o
                lse[l, b, j * g:(j + 1) * g] = s
    return out, lse


def _kv_heads(get, layer_map, l):
    kind, s0, _ = resolve(layer_map, l)
    if kind == LOWRANK:
        return int(np.asarray(get("basis_k", (s0,))).shape[0])
    return int(np.asarray(get("k", (s0, 0))).shape[0])


def prefill_rows(layer_map, l, b, h, g, q_rows, rows, get, w=None, scale=None):
    """Causal prefill outputs of query head h at the given positions.

    q_rows [n, d] are the queries at positions ``rows``; position i sees tokens
    0..i of the layer's rebuilt K/V. Returns (o [n, d], lse [n]).
    """
    K, V = layer_kv(layer_map, l, b, h // g, get, w)
    d = K.shape[1]
    sc = 1.0 / np.sqrt(d) if scale is None else scale
    o, lse, _ = attend(q_rows, K, V, sc, visible=np.asarray(rows) + 1)
    return o, lse


# ----------------------------------------------------------------------------- stored bytes
def stored_bytes(layer_map, batch, kv_heads, context, head_dim, elem_bytes=2,
                 basis_rank=32, ranks=None):
    """Bytes a cache stores for this layer table (one step, all layers).

    Forms (a)/(b): one K and one V store per distinct SINGLE source slot.
    Form (c): per pair, coefficients C_K, C_V [T, Rb] and bases [Rb, d]; per
    layer, codes of r_t bytes per token and kv head for K and V, an fp16 scale
    for K and V when r_t > 0, the residual factors R_K, R_V [Rm=16, d], and a
    one-byte rank per token. ``ranks`` [L][B][T] gives r_t.
    """
    slots = set()
    pairs = set()
    total = 0
    for l, (kind, s0, s1) in enumerate(layer_map):
        if kind == SINGLE:
            slots.add(s0)
        elif kind == MIX:
            slots.add(s0)
            slots.add(s1)
        else:
            pairs.add(s0)
            r = np.asarray(ranks[l], dtype=np.int64)            # [B, T]
            total += 2 * kv_heads * int(r.sum())                # codes K and V
            total += 2 * 2 * kv_heads * int((r > 0).sum())      # fp16 scales K and V
            total += 2 * 16 * head_dim * kv_heads * elem_bytes  # R_K, R_V
            total += batch * context                            # rank bytes
    total += len(slots) * 2 * batch * kv_heads * context * head_dim * elem_bytes
    total += len(pairs) * 2 * (batch * kv_heads * context * basis_rank * elem_bytes
                               + kv_heads * basis_rank * head_dim * elem_bytes)
    return total


def full_cache_bytes(layers, batch, kv_heads, context, head_dim, elem_bytes=2):
    """Bytes of an unshared cache: every layer stores its own K and V."""
    return layers * 2 * batch * kv_heads * context * head_dim * elem_bytes
