"""Host-side index maps, visible-pair counts and attention work lists against
the oracle on random small geometries (property-based, CPU only).

Every generated geometry is valid for the library: windows tile the grid,
the RoPE split is two multiples of 8 summing to the head dim, and the
low-res grid is either empty or non-empty on both axes.
"""
import numpy as np
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

from block_sparse_local_raster_b200 import ug
from oracle import hier_local_attn as O

B = 128
IDX, LOWRES, MASKED = (1 << 29) - 1, 1 << 29, 1 << 30


@st.composite
def geometries(draw):
    win_h, win_w = draw(st.integers(1, 12)), draw(st.integers(1, 12))
    nwy, nwx = draw(st.integers(1, 6)), draw(st.integers(1, 6))
    d = draw(st.sampled_from([64, 128]))
    ay = 8 * draw(st.integers(0, d // 8))
    lr = draw(st.sampled_from([(0, 0), (1, 1), (3, 2), (5, 7)]))
    return dict(batch=1, grid_h=win_h * nwy, grid_w=win_w * nwx, win_h=win_h, win_w=win_w,
                radius=draw(st.integers(0, 3)), lr_h=lr[0], lr_w=lr[1],
                rho=draw(st.sampled_from([1.0, 2.5, 4.0])), heads=draw(st.integers(1, 3)),
                head_dim=d, rope_dim_y=ay, rope_dim_x=d - ay, rope_theta=10000.0,
                softmax_scale=0.0, text_len=draw(st.integers(0, 40)))


SETTINGS = settings(max_examples=40, deadline=None, suppress_health_check=[HealthCheck.too_slow])


@SETTINGS
@given(geometries())
def test_index_maps_and_pair_counts(gd):
    g = O.Geometry.from_dict(gd)
    cg = ug.make_geom(**gd)
    assert ug.geom_validate(cg) == ug.UG_OK
    perm, off, idx = ug.build_index_maps(cg)
    np.testing.assert_array_equal(perm, O.window_first_index(g))
    o_off, o_idx = O.window_neighbours(g)
    np.testing.assert_array_equal(off, o_off)
    np.testing.assert_array_equal(idx, o_idx)
    c = O.visible_pairs(g)
    assert ug.visible_pairs(cg) == (c["hr_hr"], c["hr_lr"], c["lr_lr"])


def span(lowres, start, count, g):
    n, base = (g.L, g.N) if lowres else (g.N, 0)
    return base + np.arange(start, min(start + count, n))


@SETTINGS
@given(geometries())
def test_work_lists_cover_exactly_the_visible_pairs(gd):
    g = O.Geometry.from_dict(gd)
    vis = O.visibility(g, O.HR_WINDOW_FIRST, np.arange(g.N + g.L))
    qctas, kvlist, kctas, qlist = ug.work_lists(ug.make_geom(**gd))
    # forward: CTAs of 256 rows visit exactly the key blocks with a visible pair
    covered = np.zeros_like(vis)
    for lowres, q0, o, n in qctas:
        rows = span(lowres, q0, 2 * B, g)
        need = {(lk, kb) for lk, nk in ((False, g.N), (True, g.L))
                for kb in range((nk + B - 1) // B)
                if vis[np.ix_(rows, span(lk, kb * B, B, g))].any()}
        entries = kvlist[o:o + n]
        assert {(bool(e & LOWRES), int(e & IDX)) for e in entries} == need
        assert len(entries) == len(need)
        for e in entries:
            keys = span(bool(e & LOWRES), int(e & IDX) * B, B, g)
            covered[np.ix_(rows, keys)] = True
            if not e & MASKED:
                assert keys.size == B and vis[np.ix_(rows, keys)].all()
    assert not (vis & ~covered).any()
    # backward: key blocks visit exactly the query tiles with a visible pair
    covered[:] = False
    for lowres, k0, o, n in kctas:
        keys = span(lowres, k0, B, g)
        need = {(lq, qt) for lq, nq in ((False, g.N), (True, g.L))
                for qt in range((nq + B - 1) // B)
                if vis[np.ix_(span(lq, qt * B, B, g), keys)].any()}
        entries = qlist[o:o + n]
        assert {(bool(e & LOWRES), int(e & IDX)) for e in entries} == need
        assert len(entries) == len(need)
        for e in entries:
            rows = span(bool(e & LOWRES), int(e & IDX) * B, B, g)
            covered[np.ix_(rows, keys)] = True
            if not e & MASKED:
                assert vis[np.ix_(rows, keys)].all()
    assert not (vis & ~covered).any()
