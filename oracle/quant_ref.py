"""Write side of the low-rank form: rank routing and int8 residual codes (test infrastructure).

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may use this.

The pages say the per-layer residual is low-rank and quantised ("DepthWeave-KV:
Smarter KV Cache Compression by Sharing Across Layers and Adapting Per Token",
Core Mechanism diagram: residual "low-rank, quantized"; Framework Shift:
"per-layer residual (small, quantized)" and "per-token rank (router
allocates)"), and that a router gives instruction and retrieval-critical tokens a
higher rank (Core Mechanism, second component). They fix neither the router's
score nor the quantiser. The readings evaluated here:

* rank: a per-token router score s in [0, 1) maps to r = 0 if s < 0.7,
  8 if s < 0.9, else 16 (fp32 comparisons).
* symmetric int8 with a per-token fp16 scale over the first r slots:
  amax = max_{i<r} |u_i|;  scale = fp16_rne(min(amax / 127, 65504)) (the
  division in fp32);  code_i = clamp(rint(u_i / scale), -127, 127) for i < r,
  with the division in fp32 and rint rounding half to even; code_i = 0 for
  i >= r; a zero scale gives all-zero codes.

All arithmetic is fp32 with correctly rounded IEEE operations, so the integer
results are unique and the GPU must reproduce them bit for bit.
"""
from __future__ import annotations

import numpy as np

ROUTE_LOW = np.float32(0.7)
ROUTE_HIGH = np.float32(0.9)
RANK_LOW, RANK_MID, RANK_HIGH = 0, 8, 16
CODE_MAX = np.float32(127.0)
F16_MAX = np.float32(65504.0)


def route_rank(score) -> np.ndarray:
    """Per-token rank from the router score (uint8 in {0, 8, 16})."""
    s = np.asarray(score, dtype=np.float32)
    return np.where(s < ROUTE_LOW, RANK_LOW, np.where(s < ROUTE_HIGH, RANK_MID, RANK_HIGH)).astype(np.uint8)


def quantize(u, rank):
    """int8 codes and fp16 scale bits of residual rows u [..., Rm] at per-row rank [...].

    Returns (codes int8 [..., Rm], scale uint16 [...]) following the rule in the
    module docstring.
    """
    u = np.asarray(u, dtype=np.float32)
    Rm = u.shape[-1]
    r = np.asarray(rank, dtype=np.int64)[..., None]
    keep = np.arange(Rm) < r
    mag = np.where(keep, np.abs(u), np.float32(0.0)).astype(np.float32)
    amax = np.max(mag, axis=-1)                                   # fp32, exact
    s32 = np.minimum(amax / CODE_MAX, F16_MAX).astype(np.float32)  # fp32 division
    s16 = s32.astype(np.float16)                                  # round to nearest even
    sf = s16.astype(np.float32)[..., None]
    with np.errstate(divide="ignore", invalid="ignore"):
        x = (u / np.where(sf > 0, sf, np.float32(1.0))).astype(np.float32)
    c = np.clip(np.rint(x), -CODE_MAX, CODE_MAX)
    c = np.where(keep & (sf > 0), c, np.float32(0.0))
    return c.astype(np.int8), s16.view(np.uint16)


def pack_residual(score, u_k, u_v):
    """Route, then quantise the K and V residuals of every token.

    score [L][B][T] f32; u_k, u_v [L][B][Hkv][T][Rm] f32.
    Returns rank [L][B][T] u8, codes_k, codes_v [L][B][Hkv][T][Rm] i8,
    scale_k, scale_v [L][B][Hkv][T] fp16 bits (u16). The rank is shared by all
    kv heads and by K and V of a token.
    """
    rank = route_rank(score)
    rb = rank[:, :, None, :]
    ck, sk = quantize(u_k, rb)
    cv, sv = quantize(u_v, rb)
    return rank, ck, cv, sk, sv
