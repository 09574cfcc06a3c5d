"""The attention kernels' work lists (host-built, exported by
ug_build_work_lists) against the oracle's visibility mask, on the CPU.

The kernels visit only the 128-key blocks (forward, dQ) or 128-row query
tiles (dK/dV) their lists name, and skip the per-pair test on entries not
flagged.  So the lists must name exactly the blocks (tiles) holding a visible
pair, each once, and an unflagged entry must be fully visible and in range.
"""
import numpy as np
import pytest

from block_sparse_local_raster_b200 import ug, workloads
from oracle import hier_local_attn as O

B = 128
IDX, LOWRES, MASKED = (1 << 29) - 1, 1 << 29, 1 << 30
NAMES = ["tiny"] + list(workloads.TEST_GEOMETRIES)


def setup(name):
    wl = workloads.get(name)
    g = O.Geometry.from_dict(wl.geom_dict())
    vis = O.visibility(g, O.HR_WINDOW_FIRST, np.arange(g.N + g.L))  # [rows, keys], joint
    return g, vis, ug.work_lists(ug.make_geom(**wl.geom_dict()))


def span(lowres, start, count, g):
    """Joint-sequence indices of [start, start+count) in a token set, clipped."""
    n, base = (g.L, g.N) if lowres else (g.N, 0)
    return base + np.arange(start, min(start + count, n))


@pytest.mark.parametrize("name", NAMES)
def test_forward_lists_name_exactly_the_visible_blocks(name):
    g, vis, (qctas, kvlist, _, _) = setup(name)
    covered = np.zeros_like(vis)
    for lowres, q0, off, n in qctas:
        rows = span(lowres, q0, 2 * B, g)
        entries = kvlist[off:off + n]
        got = {(int(e & LOWRES) != 0, int(e & IDX)) for e in entries}
        assert len(got) == len(entries), "duplicate block"
        need = set()
        for lr_keys, nk in ((False, g.N), (True, g.L)):
            for kb in range((nk + B - 1) // B):
                if vis[np.ix_(rows, span(lr_keys, kb * B, B, g))].any():
                    need.add((lr_keys, kb))
        assert got == need
        for e in entries:
            lr_keys, kb = bool(e & LOWRES), int(e & IDX)
            keys = span(lr_keys, kb * B, B, g)
            covered[np.ix_(rows, keys)] = True
            if not e & MASKED:
                assert keys.size == B and vis[np.ix_(rows, keys)].all()
    assert not (vis & ~covered).any()  # every visible pair is visited


@pytest.mark.parametrize("name", NAMES)
def test_backward_lists_name_exactly_the_visible_tiles(name):
    g, vis, (_, _, kctas, qlist) = setup(name)
    covered = np.zeros_like(vis)
    for lowres, k0, off, n in kctas:
        keys = span(lowres, k0, B, g)
        entries = qlist[off:off + n]
        got = {(int(e & LOWRES) != 0, int(e & IDX)) for e in entries}
        assert len(got) == len(entries), "duplicate tile"
        need = set()
        for lr_rows, nq in ((False, g.N), (True, g.L)):
            for qt in range((nq + B - 1) // B):
                if vis[np.ix_(span(lr_rows, qt * B, B, g), keys)].any():
                    need.add((lr_rows, qt))
        assert got == need
        for e in entries:
            rows = span(bool(e & LOWRES), int(e & IDX) * B, B, g)
            covered[np.ix_(rows, keys)] = True
            if not e & MASKED:
                assert vis[np.ix_(rows, keys)].all()
    assert not (vis & ~covered).any()


@pytest.mark.parametrize("name", NAMES)
def test_every_query_and_key_has_exactly_one_cta(name):
    g, _, (qctas, _, kctas, _) = setup(name)
    for lists, width in ((qctas, 2 * B), (kctas, B)):
        seen = np.zeros(g.N + g.L, dtype=int)
        for lowres, start, _, _ in lists:
            seen[span(lowres, start, width, g)] += 1
        assert (seen == 1).all()
