"""Pins of the oracle's tensor-core block-scale layout (CPU).

The layout (128-row x 4-column tiles of 512 bytes, the scale of tile row r
and column c at byte (r % 32) * 16 + (r // 32) * 4 + c, zero padding) is
checked on hand-derived positions -- one 16-byte line holds rows r, r + 32,
r + 64 and r + 96 of one tile -- on the order of the tiles, on the padding,
and by the round trip through the inverse map.
"""
import numpy as np
import pytest

from oracle import oracle as O


def test_one_tile_by_hand():
    dense = (np.arange(128 * 4) % 251).astype(np.uint8).reshape(128, 4)
    m = O.mma_scale_layout(dense)
    assert m.size == 512
    # line 0: rows 0, 32, 64, 96, columns 0..3 each
    assert list(m[:16]) == list(dense[0]) + list(dense[32]) + list(dense[64]) + list(dense[96])
    # line 1: rows 1, 33, 65, 97
    assert list(m[16:32]) == list(dense[1]) + list(dense[33]) + list(dense[65]) + list(dense[97])
    # the last byte: row 127 (line 31, group 3), column 3
    assert m[511] == dense[127, 3]
    # row 33, column 2: line 1, group 1 -> byte 16 + 4 + 2
    assert m[22] == dense[33, 2]


def test_tile_order_and_padding():
    M, S = 200, 10                 # two row bands (the second padded), three column tiles (the last padded)
    rng = np.random.default_rng(1)
    dense = rng.integers(1, 256, size=(M, S), dtype=np.uint8)
    m = O.mma_scale_layout(dense)
    assert m.size == 2 * 3 * 512
    # tile (band 0, column tile 1) is the second 512-byte block; its first byte is (0, 4)
    assert m[512] == dense[0, 4]
    # tile (band 1, column tile 0) is the fourth block; its first byte is (128, 0)
    assert m[3 * 512] == dense[128, 0]
    # padding: columns 10, 11 of every row and rows 200..255 are zero bytes
    pad = np.ones(m.size, bool)
    b, r, c = np.meshgrid([0], np.arange(M), np.arange(S), indexing="ij")
    pad[O.mma_scale_offset(M, S, b, r, c)] = False
    assert pad.sum() == m.size - M * S and not m[pad].any()
    # no two scales share a byte
    assert len(set(O.mma_scale_offset(M, S, b, r, c).ravel().tolist())) == M * S


@pytest.mark.parametrize("shape", [(1, 1, 1), (3, 130, 7), (2, 256, 64), (5, 4)], ids=str)
def test_round_trip(shape):
    rng = np.random.default_rng(sum(shape))
    dense = rng.integers(0, 256, size=shape, dtype=np.uint8)
    d3 = dense if dense.ndim == 3 else dense[None]
    m = O.mma_scale_layout(dense)
    assert m.size == O.mma_scale_bytes(*d3.shape)
    assert np.array_equal(O.mma_scale_dense(m, *d3.shape), d3)
    # batches are consecutive slabs
    B, M, S = d3.shape
    slab = m.size // B
    for b in range(B):
        assert np.array_equal(O.mma_scale_layout(d3[b]), m[b * slab:(b + 1) * slab])
