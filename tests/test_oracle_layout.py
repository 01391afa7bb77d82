"""Pins of the oracle's 128 x 4 tiled scale layout (oracle/layout.py).

The pages define no tiled layout; the reading is the block-scaling
convention of tensor-core GEMMs (stated in tests/golden/tiled_scale_offsets.txt
and in include/mxq.h).  Pinned here by hand-worked offsets and by the
structural facts the convention states: every tile is one contiguous
512-byte run holding exactly its 128 x 4 submatrix, every 16-byte line holds
rows r, r + 32, r + 64, r + 96 for the tile's four columns, the map is a
bijection onto the padded matrix, and the padding is zero."""
import numpy as np
import pytest

from conftest import read_golden
from oracle import layout


def test_hand_worked_offsets():
    for cols, r, c, off in (map(int, row) for row in read_golden("tiled_scale_offsets.txt")):
        assert layout.tile_offset(r, c, cols) == off, (cols, r, c)


@pytest.mark.parametrize("rows,cols", [(1, 1), (128, 4), (130, 5), (256, 12), (77, 48), (300, 130)])
def test_bijection_onto_padded_matrix(rows, cols):
    pr, pc = layout.padded_shape(rows, cols)
    assert pr % 128 == 0 and pc % 4 == 0 and pr >= rows and pc >= cols and pr - rows < 128 and pc - cols < 4
    offs = {layout.tile_offset(r, c, cols) for r in range(pr) for c in range(pc)}
    assert offs == set(range(pr * pc))


@pytest.mark.parametrize("rows,cols", [(128, 4), (130, 5), (200, 70), (384, 48)])
def test_tiles_are_contiguous_submatrices_and_padding_is_zero(rows, cols):
    rng = np.random.default_rng(rows * 1000 + cols)
    s = rng.integers(1, 256, size=(rows, cols), dtype=np.uint8)     # no zeros in the data
    t = layout.to_tiled_128x4(s)
    assert t.size == layout.tiled_bytes(rows, cols)
    pr, pc = layout.padded_shape(rows, cols)
    padded = np.zeros((pr, pc), dtype=np.uint8)
    padded[:rows, :cols] = s
    n_ct = pc // 4
    for i in range(pr // 128):
        for j in range(n_ct):
            tile = t[(i * n_ct + j) * 512:(i * n_ct + j + 1) * 512].reshape(32, 4, 4)  # line, slab, col
            sub = padded[i * 128:(i + 1) * 128, j * 4:(j + 1) * 4]
            for line in range(32):
                for slab in range(4):
                    assert np.array_equal(tile[line, slab], sub[slab * 32 + line])
    assert np.count_nonzero(t) == rows * cols          # every padding byte is 0


def test_round_trip_and_vectorised_path():
    rng = np.random.default_rng(7)
    s = rng.integers(0, 256, size=(200, 70), dtype=np.uint8)        # > 4096 entries: numpy path
    t = layout.to_tiled_128x4(s)
    assert np.array_equal(layout.from_tiled_128x4(t, 200, 70), s)
    small = s[:40, :30]                                              # element-by-element path
    assert np.array_equal(layout.from_tiled_128x4(layout.to_tiled_128x4(small), 40, 30), small)
