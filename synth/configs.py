"""Workload presets and their seeded tensors.

Six presets follow the workloads the pages describe, at the sizes the build is
measured on:

* ``tiny_cla2_f32``   - CLA2 (adjacent-layer sharing, sharing factor 2), fp32, tiny.
  Cross-Layer Attention page, "Methodology" (sharing factors CLA2/3/4).
* ``cla2_1p1b``       - CLA2 on a 1.1B-shaped GQA model (22 layers, 32/4 heads, d 64).
* ``depthgraft_decode`` / ``depthgraft_prefill`` - layers 0..15 own K/V; target layer
  16+j reads the stride-aligned pair (j, 8+j). DepthGraft page, "Abstract".
* ``depthweave_decode`` - 16 layer pairs sharing a rank-32 basis, per-layer int8
  low-rank residual with per-token rank. DepthWeave-KV page, "Core Mechanism".
* ``depthweave_prefill`` - the same model's causal prefill of 4096 tokens.

Everything here is data: shapes, layer tables and the (seed, tensor id, scale)
recipe of every input. No attention, mixing or quantisation arithmetic.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass
from typing import Optional, Tuple

import numpy as np

from . import philox

# layer kinds (match the values of the C enum in include/kvshare.h)
SINGLE, MIX, LOWRANK = 0, 1, 2

# tensor ids: the second Philox key word
T_Q, T_K, T_V, T_W = 1, 2, 3, 4
T_BASIS_K, T_BASIS_V, T_COEF_K, T_COEF_V = 5, 6, 7, 8
T_U_K, T_U_V, T_R_K, T_R_V, T_SCORE = 9, 10, 11, 12, 13

SEED0 = 20261202


@dataclass(frozen=True)
class Config:
    name: str
    mode: str                    # 'decode' or 'prefill'
    layers: int
    q_heads: int
    kv_heads: int
    head_dim: int
    batch: int
    context: int                 # cached tokens T (decode) or sequence S (prefill)
    dtype: str                   # 'f32' or 'bf16' (q, k, v storage)
    layer_map: Tuple[Tuple[int, int, int], ...]   # (kind, src0, src1) per layer
    slots: int = 0               # K/V store slots (forms a, b)
    pairs: int = 0               # basis pairs (form c)
    qkv_scale: float = 1.0
    basis_rank: int = 32
    max_resid_rank: int = 16
    seed: int = SEED0

    @property
    def group(self) -> int:
        return self.q_heads // self.kv_heads

    def replace(self, **kw) -> "Config":
        return dataclasses.replace(self, **kw)

    # ---- shapes -------------------------------------------------------------
    def q_shape(self):
        if self.mode == "prefill":
            return (self.layers, self.batch, self.q_heads, self.context, self.head_dim)
        return (self.layers, self.batch, self.q_heads, self.head_dim)

    def kv_shape(self):
        return (self.slots, self.batch, self.kv_heads, self.context, self.head_dim)

    def w_shape(self):
        return (self.layers, self.kv_heads)

    def basis_shape(self):
        return (self.pairs, self.kv_heads, self.basis_rank, self.head_dim)

    def coef_shape(self):
        return (self.pairs, self.batch, self.kv_heads, self.context, self.basis_rank)

    def u_shape(self):
        return (self.layers, self.batch, self.kv_heads, self.context, self.max_resid_rank)

    def r_shape(self):
        return (self.layers, self.kv_heads, self.max_resid_rank, self.head_dim)

    def score_shape(self):
        return (self.layers, self.batch, self.context)

    @property
    def lowrank(self) -> bool:
        return any(k == LOWRANK for k, _, _ in self.layer_map)

    @property
    def has_mix(self) -> bool:
        return any(k == MIX for k, _, _ in self.layer_map)

    # ---- input recipe: name -> (shape, tensor id, scale, storage) -------------
    def recipe(self):
        r = {"q": (self.q_shape(), T_Q, self.qkv_scale, self.dtype, "normal")}
        if not self.lowrank:
            r["k"] = (self.kv_shape(), T_K, self.qkv_scale, self.dtype, "normal")
            r["v"] = (self.kv_shape(), T_V, self.qkv_scale, self.dtype, "normal")
            r["w"] = (self.w_shape(), T_W, 1.0, "f32", "uniform")
        else:
            sb = 1.0 / np.sqrt(float(self.basis_rank))
            sr = 1.0 / np.sqrt(float(self.max_resid_rank))
            r["basis_k"] = (self.basis_shape(), T_BASIS_K, sb, "bf16", "normal")
            r["basis_v"] = (self.basis_shape(), T_BASIS_V, sb, "bf16", "normal")
            r["coef_k"] = (self.coef_shape(), T_COEF_K, sb, "bf16", "normal")
            r["coef_v"] = (self.coef_shape(), T_COEF_V, sb, "bf16", "normal")
            r["u_k"] = (self.u_shape(), T_U_K, sr, "f32", "normal")
            r["u_v"] = (self.u_shape(), T_U_V, sr, "f32", "normal")
            r["r_k"] = (self.r_shape(), T_R_K, sr, "bf16", "normal")
            r["r_v"] = (self.r_shape(), T_R_V, sr, "bf16", "normal")
            r["score"] = (self.score_shape(), T_SCORE, 1.0, "f32", "uniform")
        return r

    def make(self, name: str, index: Optional[tuple] = None):
        """Draw input ``name`` (whole tensor, or ``full[index]``) on the CPU."""
        shape, tid, scale, dt, dist = self.recipe()[name]
        if dist == "uniform":
            if index is None:
                return philox.uniform_f32(shape, self.seed, tid)
            return philox.uniform_slice(shape, index, self.seed, tid)
        if index is None:
            return philox.normal(shape, self.seed, tid, scale, dt)
        return philox.normal_slice(shape, index, self.seed, tid, scale, dt)

    def make_all(self):
        return {n: self.make(n) for n in self.recipe()}


def cla_map(layers: int, factor: int = 2):
    """Adjacent sharing: a group of ``factor`` consecutive layers reads the lowest one's store."""
    return tuple((SINGLE, l // factor, 0) for l in range(layers))


def depthgraft_map(own: int = 16, stride: int = 8, targets: int = 8):
    """Layers 0..own-1 own a store; target own+j mixes stores (j, stride+j)."""
    m = [(SINGLE, l, 0) for l in range(own)]
    m += [(MIX, j, stride + j) for j in range(targets)]
    return tuple(m)


def depthweave_map(layers: int):
    return tuple((LOWRANK, l // 2, 0) for l in range(layers))


TINY_CLA2 = Config("tiny_cla2_f32", "decode", layers=4, q_heads=4, kv_heads=2, head_dim=64,
                   batch=1, context=128, dtype="f32", layer_map=cla_map(4), slots=2,
                   seed=SEED0 + 0)
CLA2_1P1B = Config("cla2_1p1b", "decode", layers=22, q_heads=32, kv_heads=4, head_dim=64,
                   batch=32, context=2048, dtype="bf16", layer_map=cla_map(22), slots=11,
                   qkv_scale=1.0 / 8.0, seed=SEED0 + 1)
DEPTHGRAFT_DECODE = Config("depthgraft_decode", "decode", layers=24, q_heads=16, kv_heads=4,
                           head_dim=128, batch=16, context=8192, dtype="bf16",
                           layer_map=depthgraft_map(), slots=16, seed=SEED0 + 2)
DEPTHGRAFT_PREFILL = Config("depthgraft_prefill", "prefill", layers=24, q_heads=16, kv_heads=4,
                            head_dim=128, batch=4, context=4096, dtype="bf16",
                            layer_map=depthgraft_map(), slots=16, seed=SEED0 + 3)
DEPTHWEAVE_DECODE = Config("depthweave_decode", "decode", layers=32, q_heads=32, kv_heads=8,
                           head_dim=128, batch=1, context=65536, dtype="bf16",
                           layer_map=depthweave_map(32), pairs=16, seed=SEED0 + 4)

# causal prefill of the DepthWeave model's first 4096 tokens (its head layout, 16 layer pairs)
DEPTHWEAVE_PREFILL = Config("depthweave_prefill", "prefill", layers=32, q_heads=32, kv_heads=8,
                            head_dim=128, batch=1, context=4096, dtype="bf16",
                            layer_map=depthweave_map(32), pairs=16, seed=SEED0 + 5)

PRESETS = [TINY_CLA2, CLA2_1P1B, DEPTHGRAFT_DECODE, DEPTHGRAFT_PREFILL, DEPTHWEAVE_DECODE, DEPTHWEAVE_PREFILL]
BY_NAME = {c.name: c for c in PRESETS}
