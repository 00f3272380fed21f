"""Byte layout of the residual code stores (group-packed), for tests.

Pure indexing, none of the method's arithmetic. A (layer, sequence, kv head) row of
a code store is T x 16 bytes. Its tokens form groups of 32 (group g: tokens
32 g .. 32 g + 31, the last possibly shorter) and group g owns the bytes
[512 g, 512 g + 16 n_g). Inside a group the tokens' code slots follow one another
in token order; token t's slot is k_t = 8 ceil(min(r_t, 16) / 8) bytes (0, 8 or 16):
its first min(r_t, 16) codes, then zeros. The other bytes of a group are unused
(whatever the writer left there). include/kvshare.h, kvshare_cache.u_k,
states the same layout for users of the library.
"""
import numpy as np

GROUP = 32
RM = 16


def code_lengths(rank_row):
    """Slot bytes per token: 8 ceil(min(r, 16) / 8)."""
    r = np.minimum(np.asarray(rank_row).astype(np.int64), RM)
    return (r + 7) // 8 * 8


def byte_offsets(rank_row):
    """Row byte offset of each token's first code, [T] int64."""
    k = code_lengths(rank_row)
    T = k.shape[0]
    off = np.empty(T, np.int64)
    for g0 in range(0, T, GROUP):
        kk = k[g0:g0 + GROUP]
        off[g0:g0 + GROUP] = g0 * RM + np.cumsum(kk) - kk
    return off


def used_bytes(rank_row):
    """Boolean [T * 16]: the bytes of the row that hold code slots."""
    k = code_lengths(rank_row)
    off = byte_offsets(rank_row)
    used = np.zeros(k.shape[0] * RM, bool)
    for t in np.nonzero(k)[0]:
        used[off[t]:off[t] + k[t]] = True
    return used


def pack_row(dense_row, rank_row):
    """Dense codes [T, 16] (code i of token t at [t, i], zero past its rank) -> the stored
    row [T, 16]; unused bytes 0."""
    dense_row = np.asarray(dense_row, np.int8)
    T = dense_row.shape[0]
    k = code_lengths(rank_row)
    r = np.minimum(np.asarray(rank_row).astype(np.int64), RM)
    off = byte_offsets(rank_row)
    flat = np.zeros(T * RM, np.int8)
    for t in np.nonzero(k)[0]:
        flat[off[t]:off[t] + r[t]] = dense_row[t, :r[t]]
    return flat.reshape(T, RM)


def unpack_row(row, rank_row):
    """The stored row [T, 16] -> dense codes [T, 16], codes past each token's rank 0."""
    row = np.asarray(row, np.int8)
    T = row.shape[0]
    flat = row.reshape(T * RM)
    r = np.minimum(np.asarray(rank_row).astype(np.int64), RM)
    off = byte_offsets(rank_row)
    idx = off[:, None] + np.arange(RM)[None, :]
    keep = np.arange(RM)[None, :] < r[:, None]
    return np.where(keep, flat[np.minimum(idx, T * RM - 1)], 0).astype(np.int8)


def unpack(packed, rank):
    """packed [L][B][Hkv][T][16] as stored, rank [L][B][T] -> dense [L][B][Hkv][T][16]."""
    packed = np.asarray(packed, np.int8)
    out = np.zeros_like(packed)
    L, B, H = packed.shape[:3]
    for l in range(L):
        for b in range(B):
            for h in range(H):
                out[l, b, h] = unpack_row(packed[l, b, h], rank[l, b])
    return out


def pack(dense, rank):
    """dense [L][B][Hkv][T][16] -> stored layout (unused bytes 0)."""
    dense = np.asarray(dense, np.int8)
    out = np.zeros_like(dense)
    L, B, H = dense.shape[:3]
    for l in range(L):
        for b in range(B):
            for h in range(H):
                out[l, b, h] = pack_row(dense[l, b, h], rank[l, b])
    return out
