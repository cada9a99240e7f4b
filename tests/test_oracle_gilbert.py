"""Pins for the oracle's Gilbert order (Video-BLADE, "Preprocessing: Locality-preserving
token rearrangement").  The pages name the curve without defining it, so the pins are
the properties any generalised Hilbert curve has: a bijection onto the grid whose
consecutive cells are neighbours, identity on a 1-D grid, the textbook Hilbert curve
on 2^m x 2^m frames, and better block locality than raster order."""
import itertools

import numpy as np
import pytest

from oracle.gilbert import gilbert_cells, gilbert_order


def _steps_ok(cells):
    a = np.asarray(cells)
    d = np.abs(np.diff(a, axis=0))
    return bool(np.all(d.max(axis=1) == 1)), int(np.sum(d.sum(axis=1) > 1))


def test_bijection_and_unit_steps_all_small_grids():
    for T, H, W in itertools.product(range(1, 9), repeat=3):
        cells = gilbert_cells(T, H, W)
        assert len(cells) == T * H * W
        assert len(set(cells)) == T * H * W
        assert all(0 <= x < W and 0 <= y < H and 0 <= t < T for x, y, t in cells)
        if len(cells) > 1:
            cheb_ok, diagonal = _steps_ok(cells)
            assert cheb_ok, (T, H, W)
            # the construction never needs a diagonal step
            assert diagonal == 0, (T, H, W)
        perm = gilbert_order(T, H, W)
        assert sorted(perm.tolist()) == list(range(T * H * W))


@pytest.mark.parametrize("shape", [(21, 30, 52), (13, 30, 45), (21, 45, 80), (4, 16, 16)])
def test_workload_grids(shape):
    cells = gilbert_cells(*shape)
    T, H, W = shape
    assert len(set(cells)) == T * H * W
    cheb_ok, diagonal = _steps_ok(cells)
    assert cheb_ok and diagonal == 0
    assert cells[0] == (0, 0, 0)


@pytest.mark.parametrize("n", [1, 2, 3, 7, 52, 80])
def test_one_dimensional_grid_is_identity(n):
    for shape in [(1, 1, n), (1, n, 1), (n, 1, 1)]:
        assert gilbert_order(*shape).tolist() == list(range(n))


def _textbook_hilbert(n):
    """Classic iterative Hilbert index -> (x, y) map on an n x n grid, n = 2^m."""
    pts = []
    for d in range(n * n):
        x = y = 0
        t = d
        s = 1
        while s < n:
            rx = 1 & (t // 2)
            ry = 1 & (t ^ rx)
            if ry == 0:
                if rx == 1:
                    x, y = s - 1 - x, s - 1 - y
                x, y = y, x
            x += s * rx
            y += s * ry
            t //= 4
            s *= 2
        pts.append((x, y))
    return pts


@pytest.mark.parametrize("n", [2, 4, 8, 16, 32, 64])
def test_square_frame_is_hilbert_curve(n):
    ours = [(x, y) for (x, y, t) in gilbert_cells(1, n, n)]
    ref = _textbook_hilbert(n)
    syms = [
        lambda x, y: (x, y), lambda x, y: (y, x),
        lambda x, y: (n - 1 - x, y), lambda x, y: (x, n - 1 - y),
        lambda x, y: (n - 1 - x, n - 1 - y), lambda x, y: (y, n - 1 - x),
        lambda x, y: (n - 1 - y, x), lambda x, y: (n - 1 - y, n - 1 - x),
    ]
    assert any([f(*p) for p in ref] == ours for f in syms)


def _block_stats(cells, b=128):
    a = np.asarray(cells, dtype=np.float64)
    vols, dists = [], []
    for s in range(0, len(a), b):
        blk = a[s:s + b]
        vols.append(np.prod(blk.max(0) - blk.min(0) + 1))
        c = blk - blk.mean(0)
        dists.append(np.sqrt((c ** 2).sum(1)).mean())
    return float(np.mean(vols)), float(np.mean(dists))


@pytest.mark.parametrize("shape", [(21, 30, 52), (13, 30, 45), (21, 45, 80)])
def test_blocks_more_local_than_raster(shape):
    T, H, W = shape
    raster = [(x, y, t) for t in range(T) for y in range(H) for x in range(W)]
    gv, gd = _block_stats(gilbert_cells(*shape))
    rv, rd = _block_stats(raster)
    assert gv < rv and gd < rd
