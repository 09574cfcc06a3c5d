"""Pins for the oracle's window-first permutation and window-neighbour lists.

Each check ties the oracle to something other than itself: a hand-derived
fixture, a brute-force construction by enumeration, or a counting argument.
"""
import itertools
import os

import numpy as np
import pytest

from oracle import hier_local_attn as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def geom(H, W, wh, ww, r=1, lr=(0, 0), heads=1, d=8):
    return O.Geometry(batch=1, grid_h=H, grid_w=W, win_h=wh, win_w=ww, radius=r,
                      lr_h=lr[0], lr_w=lr[1], rho=4.0, heads=heads, head_dim=d,
                      rope_dim_y=d // 2, rope_dim_x=d // 2)


def test_golden_permutation_fixture():
    rows = [l for l in open(os.path.join(GOLDEN, "permute_4x6_win2x2.txt"))
            if l.strip() and not l.startswith("#")]
    H, W, wh, ww = map(int, rows[0].split())
    at_p = np.array(rows[1].split(), dtype=np.int64)
    perm = np.array(rows[2].split(), dtype=np.int64)
    g = geom(H, W, wh, ww)
    np.testing.assert_array_equal(O.window_first_index(g), perm)
    np.testing.assert_array_equal(O.raster_index(g), at_p)
    x = np.arange(H * W).reshape(1, H * W, 1)
    np.testing.assert_array_equal(O.permute_window_first(x, g)[0, :, 0], at_p)


def enumerate_window_first(H, W, wh, ww):
    """Brute force: walk the windows in raster order, and each window's cells
    in raster order, listing the raster token id of every cell met."""
    order = []
    for wy in range(H // wh):
        for wx in range(W // ww):
            for ly in range(wh):
                for lx in range(ww):
                    order.append((wy * wh + ly) * W + (wx * ww + lx))
    return np.array(order)


GRIDS = [(4, 4, 2, 2), (4, 6, 2, 2), (6, 4, 3, 2), (8, 8, 8, 8), (12, 20, 4, 5),
         (16, 16, 1, 1), (9, 15, 3, 5), (32, 32, 8, 8), (48, 36, 12, 12)]


@pytest.mark.parametrize("H,W,wh,ww", GRIDS)
def test_permutation_matches_enumeration(H, W, wh, ww):
    g = geom(H, W, wh, ww)
    np.testing.assert_array_equal(O.raster_index(g), enumerate_window_first(H, W, wh, ww))


@pytest.mark.parametrize("H,W,wh,ww", GRIDS)
def test_permutation_is_bijection_and_inverse(H, W, wh, ww):
    g = geom(H, W, wh, ww)
    perm = O.window_first_index(g)
    assert sorted(perm.tolist()) == list(range(H * W))
    x = np.random.default_rng(0).integers(0, 1 << 16, size=(2, H * W, 3), dtype=np.uint16)
    np.testing.assert_array_equal(O.unpermute(O.permute_window_first(x, g), g), x)
    y = O.permute_window_first(O.unpermute(x, g), g)
    np.testing.assert_array_equal(y, x)


@pytest.mark.parametrize("H,W,wh,ww", GRIDS)
def test_windows_are_contiguous_runs(H, W, wh, ww):
    """Every window occupies [w*T, (w+1)*T) of the window-first sequence."""
    g = geom(H, W, wh, ww)
    inv = O.raster_index(g)
    y, x = np.divmod(inv, W)
    w = (y // wh) * (W // ww) + (x // ww)
    np.testing.assert_array_equal(w, np.arange(H * W) // (wh * ww))


@pytest.mark.parametrize("nwy,nwx", [(1, 1), (1, 5), (2, 2), (3, 4), (4, 4), (8, 8), (16, 16), (5, 9)])
def test_neighbour_counts_closed_form(nwy, nwx):
    """Radius 1, clipped: sum of |N(w)| factorises per axis into
    (3n - 2) (corner/edge windows lose one neighbour row or column), and the
    interior/edge/corner histogram is (n-2)^2 x 9, 2(n-2) x 6 ... per axis."""
    g = geom(nwy * 2, nwx * 2, 2, 2, r=1)
    off, idx = O.window_neighbours(g)
    counts = np.diff(off)
    per_axis = lambda n: 1 if n == 1 else 3 * n - 2
    assert counts.sum() == per_axis(nwy) * per_axis(nwx)
    if nwy >= 2 and nwx >= 2:
        hist = {k: int((counts == k).sum()) for k in set(counts.tolist())}
        assert hist.get(4, 0) == 4
        assert hist.get(6, 0) == 2 * (nwy - 2) + 2 * (nwx - 2)
        assert hist.get(9, 0) == (nwy - 2) * (nwx - 2)


@pytest.mark.parametrize("r", [0, 1, 2, 5])
def test_neighbours_by_brute_force(r):
    """Window v is listed for w exactly when some cell of v lies within r
    window steps of w along both axes (checked on window centres)."""
    g = geom(5 * 4, 7 * 3, 4, 3, r=r)
    off, idx = O.window_neighbours(g)
    nwy, nwx = 5, 7
    for w, (wy, wx) in enumerate(itertools.product(range(nwy), range(nwx))):
        cy, cx = wy * 4 + 1.5, wx * 3 + 1.0
        expect = []
        for v, (vy, vx) in enumerate(itertools.product(range(nwy), range(nwx))):
            dy = abs((vy * 4 + 1.5) - cy) / 4
            dx = abs((vx * 3 + 1.0) - cx) / 3
            if max(dy, dx) <= r + 1e-9:
                expect.append(v)
        assert idx[off[w]:off[w + 1]].tolist() == expect
