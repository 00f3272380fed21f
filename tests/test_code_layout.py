"""CPU pins of the group-packed code layout helper the GPU tests read code stores with.

Hand-placed bytes fix the layout (a rank-8 token takes an 8-byte slot right after the
group's earlier slots, a rank-0 token none, a rank-3 token 8 bytes of which the last
5 are zero, the second group starts at byte 512), so
an off-by-one in the offsets or a group of the wrong size fails here before any GPU
test relies on the helper.
"""
import numpy as np

from code_layout import byte_offsets, pack_row, unpack_row, used_bytes


def dense_codes(T, rank, seed):
    rng = np.random.default_rng(seed)
    d = rng.integers(-127, 128, size=(T, 16)).astype(np.int8)
    d[np.arange(16)[None, :] >= np.minimum(rank, 16)[:, None]] = 0
    return d


def test_hand_placed_bytes():
    T = 40
    rank = np.zeros(T, np.uint8)
    rank[[0, 2, 3, 31, 32, 33]] = [8, 16, 8, 16, 8, 16]
    d = dense_codes(T, rank, 1)
    row = pack_row(d, rank).reshape(-1)
    assert np.array_equal(row[0:8], d[0, :8])          # token 0, rank 8
    assert np.array_equal(row[8:24], d[2, :16])        # token 1 has rank 0: token 2 follows
    assert np.array_equal(row[24:32], d[3, :8])
    assert np.array_equal(row[32:48], d[31, :16])      # tokens 4..30 store nothing
    assert np.array_equal(row[512:520], d[32, :8])     # the second group starts at byte 512
    assert np.array_equal(row[520:536], d[33, :16])
    assert not row[48:512].any() and not row[536:].any()
    off = byte_offsets(rank)
    assert off[0] == 0 and off[2] == 8 and off[3] == 24 and off[31] == 32 and off[32] == 512 and off[33] == 520
    assert used_bytes(rank).sum() == 8 + 16 + 8 + 16 + 8 + 16


def test_round_trip_and_group_bound():
    rng = np.random.default_rng(2)
    for T in (1, 17, 32, 33, 64, 100, 300):
        rank = rng.choice(np.array([0, 8, 16], np.uint8), size=T, p=[0.7, 0.2, 0.1])
        d = dense_codes(T, rank, T)
        row = pack_row(d, rank)
        assert np.array_equal(unpack_row(row, rank), d)
        # every group's codes stay inside its 512 bytes
        k = np.minimum(rank.astype(np.int64), 16)
        for g0 in range(0, T, 32):
            assert k[g0:g0 + 32].sum() <= 16 * min(32, T - g0)
        # unused bytes do not reach the dense codes
        junk = row.copy().reshape(-1)
        junk[~used_bytes(rank)] = 99
        assert np.array_equal(unpack_row(junk.reshape(T, 16), rank), d)


def test_rank_above_sixteen_keeps_sixteen_codes_and_odd_ranks_take_whole_slots():
    rank = np.array([20, 3, 8], np.uint8)
    d = dense_codes(3, np.array([16, 3, 8]), 3)
    row = pack_row(d, rank).reshape(-1)
    assert np.array_equal(row[:16], d[0]) and np.array_equal(row[16:19], d[1, :3])
    assert not row[19:24].any()                        # the rest of token 1's 8-byte slot
    assert np.array_equal(row[24:32], d[2, :8])        # token 2's slot starts 8-byte aligned
    assert np.array_equal(byte_offsets(rank), [0, 16, 24])
