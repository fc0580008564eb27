"""The test suite's index maps of the library's data layouts, checked against
the layouts as the public header describes them (CPU only).  The GPU tests
read the library's tiled scales and staged codes back through these maps."""
import numpy as np
import pytest

from _util import canonical_to_staged, staged_to_canonical, staged_unit_index, tiled_index


@pytest.mark.parametrize("rows,cols", [(128, 256), (256, 512), (384, 6144), (2048, 256)])
def test_staged_index_is_a_permutation(rows, cols):
    idx = staged_unit_index(rows, cols).reshape(-1)
    assert np.array_equal(np.sort(idx), np.arange(rows * cols // 16))


def test_staged_layout_matches_the_header():
    """Tile (i, j) = rows [128 i, 128 i + 128) x columns [256 j, 256 j + 256)
    starts at byte (i * cols/256 + j) * 16384; inside it, the 16 bytes of row
    r's columns [256 j + 32 c, 256 j + 32 c + 32) sit at 128 r + 16 (c ^ (r % 8))."""
    rows, cols = 384, 1024
    codes = np.random.default_rng(1).integers(0, 256, (rows, cols // 2), dtype=np.uint8)
    flat = canonical_to_staged(codes, rows, cols).reshape(-1)
    rng = np.random.default_rng(2)
    for _ in range(200):
        r_abs, col = int(rng.integers(rows)), int(rng.integers(cols // 32)) * 32
        i, j = r_abs // 128, col // 256
        r, c = r_abs % 128, (col % 256) // 32
        start = (i * (cols // 256) + j) * 16384 + 128 * r + 16 * (c ^ (r % 8))
        assert np.array_equal(flat[start:start + 16], codes[r_abs, col // 2:col // 2 + 16])
    assert np.array_equal(staged_to_canonical(flat, rows, cols), codes)


def test_tiled_scale_index_matches_the_header():
    """Atom (row tile, block group of 4) is 512 bytes, row-tile major; inside
    it row r, block b sits at (r % 32) * 16 + (r / 32) * 4 + b."""
    rows, cols = 256, 512
    idx = tiled_index(rows, cols)
    nb = cols // 16
    for r in (0, 31, 32, 127, 128, 255):
        for b in (0, 3, 4, nb - 1):
            atom = (r // 128) * (nb // 4) + b // 4
            assert idx[r, b] == atom * 512 + (r % 128 % 32) * 16 + ((r % 128) // 32) * 4 + b % 4
    assert np.array_equal(np.sort(idx.reshape(-1)), np.arange(rows * nb))
