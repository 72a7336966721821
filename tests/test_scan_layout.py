"""Chunk layout of the pipelined kernel against the oracle's direction map (CPU only).

gla_scan_layout runs the kernel's own host/device chunk geometry on the host: for every scan
position it names the token the kernel's tiles place there.  The scan order it must reproduce is
the one of the scan-direction paragraph of the GTR paper's method section, as the oracle states it
(lines in increasing order, the state carried from one line's end to the next line's start).
"""
import pytest

import oracle
from recurrent_vision_backbone_only_b200 import gla

GRIDS = [(8, 8), (40, 40), (80, 80), (24, 37), (37, 24), (16, 20), (42, 50), (5, 7), (128, 128),
         (1, 64), (64, 1), (3, 96)]


@pytest.mark.parametrize("grid", GRIDS)
@pytest.mark.parametrize("chunk", [0, 16, 32, 48])
def test_layout_matches_the_oracle_scan_order(grid, chunk):
    gh, gw = grid
    for d in range(4):
        spatial, rows = gla.scan_layout(gh, gw, d, chunk)
        want = [oracle.spatial_index(d, p, gh, gw) for p in range(gh * gw)]
        assert spatial == want, (grid, chunk, d)
        assert rows in (8, 16, 32, 64)


@pytest.mark.parametrize("grid,chunk,rows", [((40, 40), 0, 8), ((80, 80), 0, 16), ((128, 128), 0, 64),
                                             ((24, 37), 0, 64), ((40, 40), 48, 8), ((80, 80), 48, 16),
                                             ((8, 8), 16, 8)])
def test_box_height(grid, chunk, rows):
    """Packed chunks where the line length has a power-of-two factor >= 8 in common with the
    chunk length; 64-row boxes (line-aligned chunks) otherwise (shown on R->L, which packs
    within lines)."""
    gh, gw = grid
    assert gla.scan_layout(gh, gw, 1, chunk)[1] == rows


@pytest.mark.parametrize("grid,chunk,rows", [((40, 40), 0, 64), ((24, 37), 0, 64), ((7, 5), 32, 32),
                                             ((40, 40), 48, 16)])
def test_forward_row_scans_load_whole_chunks(grid, chunk, rows):
    """L->R visits token rows in memory order: a chunk is consecutive rows across lines, loaded
    in boxes of the largest power of two dividing the chunk length."""
    gh, gw = grid
    assert gla.scan_layout(gh, gw, 0, chunk)[1] == rows


def test_layout_rejects():
    with pytest.raises(RuntimeError):
        gla.scan_layout(8, 8, 0, 0, kernel=gla.KERNEL_TC64)
    with pytest.raises(RuntimeError):
        gla.scan_layout(8, 8, 4, 0)
    with pytest.raises(RuntimeError):
        gla.scan_layout(8, 8, 0, 24)
