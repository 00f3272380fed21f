"""Write side of the low-rank form for one new token (test infrastructure).

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may use this.

A layer pair shares a low-rank channel basis and each layer keeps a light
per-layer residual for what the basis misses ("DepthWeave-KV: Smarter KV Cache
Compression by Sharing Across Layers and Adapting Per Token", Core Mechanism,
first component, and its diagram: the shared basis B plus a residual R_i per
layer, low-rank and quantised). The pages do not say how a token's coefficients
and residual are found; the readings evaluated here, for a token with key (or
value) vectors k_0, k_1 in the two layers of the pair, bases rows B [Rb][d] and
each layer's residual factor rows R_a [16][d]:

* coefficients, shared by the two layers: the least-squares fit of both layers'
  vectors in the shared basis when its rows are orthonormal, i.e. the projection
  of their mean, c = B (k_0 + k_1) / 2, stored as bf16 (round to nearest even);
* residual of layer a against what the stored coefficients rebuild:
  e_a = k_a - B^T c_stored;
* the layer's low-rank residual coordinates u_a = R_a e_a (16 values), which
  the existing quantiser (``quant_ref.quantize``) turns into int8 codes and an
  fp16 scale at the token's rank.

Because the codes are integers decided by floating point, every step is fp32 in
a stated order, each operation correctly rounded, with no fused multiply-add:
m_i = (k_0,i + k_1,i) * 0.5; a dot product accumulates its terms from index 0
up as acc = acc + (x_i * y_i), starting from the first product. ``fit_pair_basis``
builds orthonormal rows from a calibration window with numpy's SVD; it serves the
tests that need a basis with the structure the method assumes.
"""
from __future__ import annotations

import numpy as np

from . import quant_ref


def _f32(x):
    return np.asarray(x, dtype=np.float32)


def dot_rows_f32(A, x):
    """fp32 dot products of each row of A with x, accumulated from index 0 up with the
    product and the sum each rounded: A [n][d], x [d] -> [n]."""
    A = _f32(A)
    x = _f32(x)
    acc = (A[:, 0] * x[0]).astype(np.float32)
    for i in range(1, A.shape[1]):
        acc = (acc + (A[:, i] * x[i]).astype(np.float32)).astype(np.float32)
    return acc


def combine_rows_f32(c, A):
    """fp32 sum_r c_r A[r][:], accumulated from r = 0 up, each product and sum rounded."""
    c = _f32(c)
    A = _f32(A)
    acc = (c[0] * A[0]).astype(np.float32)
    for r in range(1, A.shape[0]):
        acc = (acc + (c[r] * A[r]).astype(np.float32)).astype(np.float32)
    return acc


def f32_to_bf16_bits(x):
    """Round fp32 values to bf16 (nearest, ties to even); NaN is not expected here."""
    b = _f32(x).view(np.uint32).astype(np.uint64)
    lsb = (b >> 16) & 1
    return ((b + 0x7FFF + lsb) >> 16).astype(np.uint16)


def bf16_bits_to_f32(bits):
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def encode_pair(k0, k1, basis, r0, r1, rank0, rank1):
    """One token of one kv head of a layer pair.

    k0, k1 [d]: the token's vectors in the pair's two layers (fp32 values, bf16 in
    the cache's use); basis [Rb][d]; r0, r1 [16][d] the layers' residual factors;
    rank0, rank1 the token's residual rank in each layer.
    Returns (coef bf16 bits [Rb], u0 [16] fp32, codes0 int8 [16], scale0 fp16 bits,
    u1, codes1, scale1).
    """
    k0 = _f32(k0)
    k1 = _f32(k1)
    m = ((k0 + k1).astype(np.float32) * np.float32(0.5)).astype(np.float32)
    c = dot_rows_f32(basis, m)
    cb = f32_to_bf16_bits(c)
    rebuilt = combine_rows_f32(bf16_bits_to_f32(cb), basis)
    out = [cb]
    for k, R, rank in ((k0, r0, rank0), (k1, r1, rank1)):
        e = (k - rebuilt).astype(np.float32)
        u = dot_rows_f32(R, e)
        codes, scale = quant_ref.quantize(u[None, :], np.array([rank]))
        out += [u, codes[0], scale[0]]
    return tuple(out)


def fit_pair_basis(K0, K1, rank: int):
    """Orthonormal rows spanning the top-``rank`` right singular subspace of the stacked
    calibration window [K0; K1] (n x d each), rows in descending singular value order."""
    X = np.concatenate([np.asarray(K0, np.float64), np.asarray(K1, np.float64)], axis=0)
    _, _, vt = np.linalg.svd(X, full_matrices=False)
    return vt[:rank]
