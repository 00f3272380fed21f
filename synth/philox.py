"""Counter-based seeded generator for the synthetic workloads (numpy side).

This module only makes random numbers. It holds none of the attention, mixing,
reconstruction or quantisation arithmetic, so both the fp64 oracle tests and the
CUDA tests/bench can draw their inputs from it.

Definition (the CUDA twin in ``synth/csrc/synth_gen.cu`` implements the same
bits; the two share no code):

* Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as easy
  as 1, 2, 3", SC'11): 10 rounds of the 4x32 Philox S-box with multipliers
  0xD2511F53 / 0xCD9E8D57 and Weyl key increments 0x9E3779B9 / 0xBB67AE85.
* Stream layout: element ``i`` of a tensor drawn with (seed, tensor id) uses
  word ``i & 3`` of the block produced for counter ``(i >> 2)`` (low 32 bits,
  high 32 bits, 0, 0) under key ``(seed, tensor id)``.
* Uniform on [0, 1): ``(word >> 8) * 2**-24`` (exact in fp32).
* Normal: Box-Muller on the word pair (w0, w1) of the element's half-block
  (words 0,1 for elements 0,1 of the block; words 2,3 for elements 2,3):
  ``u = (w0 + 1) * 2**-32`` in (0, 1], ``theta = 2*pi*w1 * 2**-32``,
  ``z = sqrt(-2 ln u) * (cos theta | sin theta)`` (cos for even elements, sin
  for odd).  ``ln``, ``cos`` and ``sin`` are evaluated by the power series
  below in fp64 with one IEEE operation at a time (no fused multiply-add), so
  that the CPU and the GPU produce identical bits:

  - ``ln(n * 2**-32)`` for integer ``n`` in [1, 2**32]: ``n = m * 2**e`` with
    m in [1, 2); if m > sqrt(2) then m /= 2, e += 1;
    ``ln m = 2 atanh(y)``, ``y = (m-1)/(m+1)``, atanh by its Taylor series
    ``y * sum_k y**(2k) / (2k+1)`` (k < 13, Horner);
    ``ln = (e - 32) * ln2 + ln m``.
  - theta = quadrant * pi/2 + phi, quadrant = w1 >> 30,
    phi = (w1 & (2**30-1)) * 2**-30 * (pi/2) in [0, pi/2);
    sin/cos phi by their Taylor series (k < 14, Horner on phi**2 with
    coefficients 1/(2k+1)! and 1/(2k)! built by repeated division), then
    rotated by the quadrant with exact sign flips.
* Storage rounding: the fp64 value times the tensor's scale is rounded to fp32
  (round to nearest even), then, for bf16 tensors, to bf16 by round to nearest
  even on the fp32 bit pattern.
"""
from __future__ import annotations

import numpy as np

_M0 = np.uint64(0xD2511F53)
_M1 = np.uint64(0xCD9E8D57)
_W0 = 0x9E3779B9
_W1 = 0xBB67AE85
_MASK32 = np.uint64(0xFFFFFFFF)

LN2 = 0.6931471805599453          # ln 2 rounded to double
HALF_PI = 1.5707963267948966      # pi/2 rounded to double
SQRT2 = 1.4142135623730951        # sqrt(2) rounded to double
_ATANH_TERMS = 13
_TRIG_TERMS = 14


def philox4x32_10(c0, c1, c2, c3, k0, k1):
    """Philox4x32-10 on uint64 arrays that hold 32-bit words; returns 4 word arrays."""
    c0 = np.asarray(c0, dtype=np.uint64)
    c1 = np.asarray(c1, dtype=np.uint64)
    c2 = np.asarray(c2, dtype=np.uint64)
    c3 = np.asarray(c3, dtype=np.uint64)
    k0 = int(k0) & 0xFFFFFFFF
    k1 = int(k1) & 0xFFFFFFFF
    for _ in range(10):
        p0 = _M0 * c0
        p1 = _M1 * c2
        hi0, lo0 = p0 >> np.uint64(32), p0 & _MASK32
        hi1, lo1 = p1 >> np.uint64(32), p1 & _MASK32
        c0, c1, c2, c3 = (hi1 ^ c1 ^ np.uint64(k0)), lo1, (hi0 ^ c3 ^ np.uint64(k1)), lo0
        k0 = (k0 + _W0) & 0xFFFFFFFF
        k1 = (k1 + _W1) & 0xFFFFFFFF
    return c0, c1, c2, c3


def raw_words(n: int, offset: int, seed: int, stream: int) -> np.ndarray:
    """The 32-bit word of elements [offset, offset+n) (uint64 array)."""
    idx = np.arange(offset, offset + n, dtype=np.uint64)
    return _words_for(idx, seed, stream)[0]


def _words_for(idx: np.ndarray, seed: int, stream: int):
    blk = idx >> np.uint64(2)
    lane = (idx & np.uint64(3)).astype(np.int64)
    w = philox4x32_10(blk & _MASK32, blk >> np.uint64(32), np.zeros_like(blk), np.zeros_like(blk),
                      seed, stream)
    words = np.stack(w, axis=-1)                       # [n, 4]
    rows = np.arange(idx.shape[0])
    own = words[rows, lane]
    pair0 = words[rows, (lane & 2)]                    # w0 of the Box-Muller pair
    pair1 = words[rows, (lane & 2) + 1]                # w1 of the Box-Muller pair
    return own, pair0, pair1, lane


def _coeffs():
    # 1/(2k+1) for atanh; 1/(2k+1)! and 1/(2k)! by repeated division (same order on GPU)
    at = [1.0 / float(2 * k + 1) for k in range(_ATANH_TERMS)]
    s = [1.0]
    c = [1.0]
    for k in range(1, _TRIG_TERMS):
        s.append(s[-1] / float((2 * k) * (2 * k + 1)))
        c.append(c[-1] / float((2 * k - 1) * (2 * k)))
    return at, s, c


_AT, _SIN_C, _COS_C = _coeffs()


def series_log_u32(w0: np.ndarray) -> np.ndarray:
    """ln((w0 + 1) * 2**-32) by the atanh series (fp64, one IEEE op at a time)."""
    n = w0.astype(np.uint64) + np.uint64(1)            # 1 .. 2**32
    # e = floor(log2 n), exact from the bit length
    e = np.zeros(n.shape, dtype=np.int64)
    t = n.copy()
    for sh in (32, 16, 8, 4, 2, 1):
        big = t >= (np.uint64(1) << np.uint64(sh))
        e = np.where(big, e + sh, e)
        t = np.where(big, t >> np.uint64(sh), t)
    m = n.astype(np.float64) / np.exp2(e.astype(np.float64))   # exact: power-of-two divide
    hi = m > SQRT2
    m = np.where(hi, m * 0.5, m)
    e = np.where(hi, e + 1, e)
    y = (m - 1.0) / (m + 1.0)
    y2 = y * y
    acc = np.full(y.shape, _AT[_ATANH_TERMS - 1])
    for k in range(_ATANH_TERMS - 2, -1, -1):
        acc = acc * y2
        acc = acc + _AT[k]
    lnm = (2.0 * y) * acc
    return (e - 32).astype(np.float64) * LN2 + lnm


def series_sincos_u32(w1: np.ndarray):
    """(cos, sin) of 2*pi*w1*2**-32 by quadrant reduction and Taylor series."""
    w1 = w1.astype(np.uint64)
    quad = (w1 >> np.uint64(30)).astype(np.int64)
    frac = (w1 & np.uint64(0x3FFFFFFF)).astype(np.float64) * (2.0 ** -30)
    phi = frac * HALF_PI
    p2 = phi * phi
    sa = np.full(phi.shape, ((-1.0) ** (_TRIG_TERMS - 1)) * _SIN_C[_TRIG_TERMS - 1])
    ca = np.full(phi.shape, ((-1.0) ** (_TRIG_TERMS - 1)) * _COS_C[_TRIG_TERMS - 1])
    for k in range(_TRIG_TERMS - 2, -1, -1):
        sgn = 1.0 if k % 2 == 0 else -1.0
        sa = sa * p2
        sa = sa + sgn * _SIN_C[k]
        ca = ca * p2
        ca = ca + sgn * _COS_C[k]
    s = phi * sa
    c = ca
    cos_t = np.select([quad == 0, quad == 1, quad == 2], [c, -s, -c], s)
    sin_t = np.select([quad == 0, quad == 1, quad == 2], [s, c, -s], -c)
    return cos_t, sin_t


def normal_f64(n: int, offset: int, seed: int, stream: int) -> np.ndarray:
    """Standard normal deviates (fp64) of elements [offset, offset+n)."""
    idx = np.arange(offset, offset + n, dtype=np.uint64)
    return normal_f64_at(idx, seed, stream)


def normal_f64_at(idx: np.ndarray, seed: int, stream: int) -> np.ndarray:
    idx = np.asarray(idx, dtype=np.uint64)
    if idx.size == 0:
        return np.zeros(0)
    blk = idx >> np.uint64(2)
    b0, b1 = int(blk.min()), int(blk.max())
    if 4 * (b1 - b0 + 1) <= 2 * idx.size + 64:
        # dense request: one Philox call and one Box-Muller pair per block/pair
        z = _normal_blocks(b0, b1 - b0 + 1, seed, stream)          # [nblk, 4]
        return z[(blk - np.uint64(b0)).astype(np.int64), (idx & np.uint64(3)).astype(np.int64)]
    _, w0, w1, lane = _words_for(idx, seed, stream)
    r = np.sqrt(-2.0 * series_log_u32(w0))
    cos_t, sin_t = series_sincos_u32(w1)
    return np.where((lane & 1) == 0, r * cos_t, r * sin_t)


def _normal_blocks(first_blk: int, nblk: int, seed: int, stream: int) -> np.ndarray:
    """Normals of all 4 elements of blocks [first_blk, first_blk + nblk): array [nblk, 4]."""
    blk = np.arange(first_blk, first_blk + nblk, dtype=np.uint64)
    w = philox4x32_10(blk & _MASK32, blk >> np.uint64(32), np.zeros_like(blk), np.zeros_like(blk), seed, stream)
    out = np.empty((nblk, 4))
    for p in range(2):
        r = np.sqrt(-2.0 * series_log_u32(w[2 * p]))
        cos_t, sin_t = series_sincos_u32(w[2 * p + 1])
        out[:, 2 * p] = r * cos_t
        out[:, 2 * p + 1] = r * sin_t
    return out


def f32_bits_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest even) and return the 16-bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return r.astype(np.uint16)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def normal(shape, seed: int, stream: int, scale: float = 1.0, dtype: str = "bf16", offset: int = 0):
    """A tensor of N(0,1)*scale in its storage type: 'f32' -> float32, 'bf16' -> uint16 bits."""
    n = int(np.prod(shape))
    z = normal_f64(n, offset, seed, stream) * float(scale)
    f = z.astype(np.float32)
    if dtype == "f32":
        return f.reshape(shape)
    if dtype == "bf16":
        return f32_bits_to_bf16_bits(f).reshape(shape)
    raise ValueError(dtype)


def uniform_f32(shape, seed: int, stream: int, offset: int = 0) -> np.ndarray:
    """U[0,1) float32 with 24 random bits per element."""
    n = int(np.prod(shape))
    w = raw_words(n, offset, seed, stream)
    return ((w >> np.uint64(8)).astype(np.float64) * (2.0 ** -24)).astype(np.float32).reshape(shape)


def _flat_index(full_shape, index):
    """Flat element indices (uint64) of ``full[index]`` and the result's shape.

    ``index`` is a tuple of ints / slices over the leading dims of ``full_shape``.
    """
    sels = tuple(index) + (slice(None),) * (len(full_shape) - len(index))
    strides = [int(np.prod(full_shape[i + 1:])) for i in range(len(full_shape))]
    flat = np.zeros(1, dtype=np.uint64)
    shape = []
    for size, sel, st in zip(full_shape, sels, strides):
        if isinstance(sel, slice):
            g = np.arange(size, dtype=np.uint64)[sel]
            shape.append(len(g))
        else:
            g = np.array([int(sel)], dtype=np.uint64)
        flat = (flat[:, None] + g[None, :] * np.uint64(st)).reshape(-1)
    return flat, tuple(shape)


def normal_slice(full_shape, index, seed: int, stream: int, scale: float = 1.0, dtype: str = "bf16"):
    """``normal(full_shape, ...)[index]`` without drawing the rest of the tensor."""
    flat, shape = _flat_index(full_shape, index)
    f = (normal_f64_at(flat, seed, stream) * float(scale)).astype(np.float32)
    vals = f if dtype == "f32" else f32_bits_to_bf16_bits(f)
    return vals.reshape(shape)


def uniform_slice(full_shape, index, seed: int, stream: int) -> np.ndarray:
    """``uniform_f32(full_shape, ...)[index]`` without drawing the rest of the tensor."""
    flat, shape = _flat_index(full_shape, index)
    own = _words_for(flat, seed, stream)[0]
    return ((own >> np.uint64(8)).astype(np.float64) * (2.0 ** -24)).astype(np.float32).reshape(shape)
