"""Scale layouts (test infrastructure only).

The oracle quantizers write block scales in the linear checkpoint layout,
row-major [rows, cols / block].  Block-scaled tensor-core GEMMs read scales
in a tiled layout instead; the pages only note that a loader may repack or
interleave quantized weights for its kernel
(josch15366/Qwen3.8-Flash-Next-NVFP4-LocalHessian-Experts, "Verifying the
merge").  The tiled layout is therefore a reading, written out here as the
plain index permutation it is:

* pad the scale matrix with zeros to a multiple of 128 rows and 4 columns;
* cut it into tiles of 128 rows x 4 columns; tile (i, j) (i = row // 128,
  j = col // 4) occupies bytes [512 * (i * n_col_tiles + j), +512);
* inside a tile, the 128 rows are four slabs of 32 rows, and the scale of
  (row r, column c) of the tile sits at byte 16 * (r % 32) + 4 * (r // 32)
  + c: one 16-byte line holds rows r, r + 32, r + 64, r + 96 for the four
  columns.

``tile_offset`` states the permutation for one element;
``to_tiled_128x4`` applies it to a whole matrix (element by element for
small matrices, as numpy index arrays for large ones, the same formula).
"""
import numpy as np

TILE_ROWS = 128
TILE_COLS = 4
TILE_BYTES = TILE_ROWS * TILE_COLS


def padded_shape(rows, cols):
    """(rows, cols) of a scale matrix after padding to whole tiles."""
    return (-(-rows // TILE_ROWS) * TILE_ROWS, -(-cols // TILE_COLS) * TILE_COLS)


def tiled_bytes(rows, cols):
    pr, pc = padded_shape(rows, cols)
    return pr * pc


def tile_offset(r, c, cols):
    """Byte offset of scale (r, c) in the tiled layout of a matrix with
    `cols` scale columns."""
    n_col_tiles = -(-cols // TILE_COLS)
    tile = (r // TILE_ROWS) * n_col_tiles + c // TILE_COLS
    rr, cc = r % TILE_ROWS, c % TILE_COLS
    return tile * TILE_BYTES + 16 * (rr % 32) + 4 * (rr // 32) + cc


def to_tiled_128x4(scales):
    """uint8 [rows, cols] (linear) -> uint8 [tiled_bytes(rows, cols)]."""
    scales = np.asarray(scales, dtype=np.uint8)
    rows, cols = scales.shape
    out = np.zeros(tiled_bytes(rows, cols), dtype=np.uint8)
    if rows * cols <= 4096:
        for r in range(rows):
            for c in range(cols):
                out[tile_offset(r, c, cols)] = scales[r, c]
        return out
    r = np.arange(rows, dtype=np.int64)[:, None]
    c = np.arange(cols, dtype=np.int64)[None, :]
    n_col_tiles = -(-cols // TILE_COLS)
    off = ((r // TILE_ROWS) * n_col_tiles + c // TILE_COLS) * TILE_BYTES \
        + 16 * ((r % TILE_ROWS) % 32) + 4 * ((r % TILE_ROWS) // 32) + c % TILE_COLS
    out[off.reshape(-1)] = scales.reshape(-1)
    return out


def from_tiled_128x4(tiled, rows, cols):
    """Inverse of to_tiled_128x4 (drops the padding)."""
    tiled = np.asarray(tiled, dtype=np.uint8).reshape(-1)
    out = np.empty((rows, cols), dtype=np.uint8)
    for r in range(rows):
        for c in range(cols):
            out[r, c] = tiled[tile_offset(r, c, cols)]
    return out
