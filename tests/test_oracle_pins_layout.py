"""Pins of the oracle's blocked scale layout: it must equal an independent formulation
of the same layout by tensor reshapes (pad to 128 x 4 tiles; tiles in row-tile order;
inside a tile, the 128 rows split as 4 groups of 32 and interleaved so that each 16-byte
line holds rows i, i+32, i+64, i+96), and from_blocked must invert it."""
import numpy as np
import pytest


def _blocked_by_reshape(m: np.ndarray) -> np.ndarray:
    rows, cols = m.shape
    R, C = -(-rows // 128) * 128, -(-cols // 4) * 4
    p = np.zeros((R, C), np.uint8)
    p[:rows, :cols] = m
    tiles = p.reshape(R // 128, 128, C // 4, 4).transpose(0, 2, 1, 3)     # (row tile, col tile, 128, 4)
    inner = tiles.reshape(-1, 4, 32, 4).transpose(0, 2, 1, 3)             # (tile, r % 32, r // 32, c)
    return inner.reshape(-1)


@pytest.mark.parametrize("rows,cols", [(1, 1), (5, 8), (128, 4), (130, 8), (300, 9), (1024, 8)])
def test_blocked_layout_matches_reshape_formulation(orc, rows, cols):
    rng = np.random.default_rng(rows * 100 + cols)
    m = rng.integers(1, 255, (rows, cols), dtype=np.uint8)
    got = orc.scales_to_blocked(m.reshape(-1), rows, cols)
    np.testing.assert_array_equal(got, _blocked_by_reshape(m))
    np.testing.assert_array_equal(orc.scales_from_blocked(got, rows, cols), m.reshape(-1))


def test_blocked_tile_lines_hold_rows_32_apart(orc):
    m = np.arange(128 * 4, dtype=np.uint32).reshape(128, 4) % 251
    b = orc.scales_to_blocked(m.astype(np.uint8).reshape(-1), 128, 4).reshape(32, 16)
    for i in range(32):
        np.testing.assert_array_equal(b[i], np.concatenate([m[i], m[i + 32], m[i + 64], m[i + 96]]).astype(np.uint8))
