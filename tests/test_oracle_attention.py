"""Pins for the oracle's block-sparse joint attention.

Library routines (torch's fp64 scaled_dot_product_attention and logsumexp),
special geometries that reduce to plain attention, closed forms and
invariants; a mask built by independent enumeration of grid cells.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import hier_local_attn as O


def geom(H, W, wh, ww, r=1, lr=(0, 0), heads=2, d=16, rho=4.0, batch=1):
    return O.Geometry(batch=batch, grid_h=H, grid_w=W, win_h=wh, win_w=ww, radius=r,
                      lr_h=lr[0], lr_w=lr[1], rho=rho, heads=heads, head_dim=d,
                      rope_dim_y=d // 2, rope_dim_x=d // 2)


def inputs(g, seed=0, scale=1.0):
    rng = np.random.default_rng(seed)
    mk = lambda n: O.f64_to_bf16(scale * rng.standard_normal((g.batch, n, g.heads, g.head_dim)))
    return dict(q_hr=mk(g.N), k_hr=mk(g.N), v_hr=mk(g.N), q_lr=mk(g.L), k_lr=mk(g.L), v_lr=mk(g.L))


def run(g, x, order=O.HR_WINDOW_FIRST, rows=None):
    return O.attention(x["q_hr"], x["k_hr"], x["v_hr"], x["q_lr"], x["k_lr"], x["v_lr"],
                       g, order, rows)


def joint(x, name, b, h):
    return torch.from_numpy(np.concatenate([O.bf16_to_f64(x[name + "_hr"][b, :, h]),
                                            O.bf16_to_f64(x[name + "_lr"][b, :, h])]))


def sdpa(q, k, v, mask=None, scale=None):
    return F.scaled_dot_product_attention(q[None], k[None], v[None], attn_mask=None if mask is None
                                          else mask[None], scale=scale)[0].numpy()


def test_one_window_no_lowres_is_full_attention():
    g = geom(8, 12, 8, 12, lr=(0, 0))
    x = inputs(g, 1)
    o, _ = run(g, x)
    for h in range(g.heads):
        want = sdpa(joint(x, "q", 0, h), joint(x, "k", 0, h), joint(x, "v", 0, h), scale=g.scale)
        np.testing.assert_allclose(o[0, :, h], want, rtol=0, atol=1e-12)


def test_large_radius_is_full_attention_plus_lowres():
    g = geom(12, 16, 4, 4, r=4, lr=(3, 4))
    x = inputs(g, 2)
    o, _ = run(g, x)
    N = g.N
    for h in range(g.heads):
        q, k, v = joint(x, "q", 0, h), joint(x, "k", 0, h), joint(x, "v", 0, h)
        np.testing.assert_allclose(o[0, :N, h], sdpa(q[:N], k, v, scale=g.scale), atol=1e-12, rtol=0)
        np.testing.assert_allclose(o[0, N:, h], sdpa(q[N:], k[N:], v[N:], scale=g.scale),
                                   atol=1e-12, rtol=0)


def test_radius_zero_is_independent_windows():
    g = geom(8, 12, 4, 4, r=0, lr=(0, 0))
    x = inputs(g, 3)
    o, _ = run(g, x)
    T = g.T
    for h in range(g.heads):
        q, k, v = joint(x, "q", 0, h), joint(x, "k", 0, h), joint(x, "v", 0, h)
        for w in range(g.N // T):
            s = slice(w * T, (w + 1) * T)
            np.testing.assert_allclose(o[0, s, h], sdpa(q[s], k[s], v[s], scale=g.scale),
                                       atol=1e-12, rtol=0)


def cell_mask(g, order):
    """Visibility by enumerating grid cells: key cell (y', x') is visible to
    query cell (y, x) iff their windows are at most `radius` window steps
    apart along each axis; any low-res key is visible to a high-res query;
    low-res queries see the low-res keys only."""
    N, L = g.N, g.L
    cells = [divmod(r, g.grid_w) for r in range(N)]
    if order == O.HR_WINDOW_FIRST:
        cells = [cells[r] for r in O.raster_index(g)]
    m = np.zeros((N + L, N + L), dtype=bool)
    for i, (y, x) in enumerate(cells):
        for j, (yy, xx) in enumerate(cells):
            m[i, j] = (abs(y // g.win_h - yy // g.win_h) <= g.radius
                       and abs(x // g.win_w - xx // g.win_w) <= g.radius)
    m[:N, N:] = True
    m[N:, N:] = True
    return m


@pytest.mark.parametrize("order", [O.HR_WINDOW_FIRST, O.HR_RASTER])
@pytest.mark.parametrize("shape", [(12, 16, 4, 4, 1, (3, 2)), (16, 8, 4, 2, 2, (2, 5)),
                                   (8, 8, 2, 2, 1, (1, 1))])
def test_general_case_matches_library_with_enumerated_mask(order, shape):
    H, W, wh, ww, r, lr = shape
    g = geom(H, W, wh, ww, r=r, lr=lr)
    x = inputs(g, 4)
    o, lse = run(g, x, order)
    mask = torch.from_numpy(cell_mask(g, order))
    for h in range(g.heads):
        q, k, v = joint(x, "q", 0, h), joint(x, "k", 0, h), joint(x, "v", 0, h)
        np.testing.assert_allclose(o[0, :, h], sdpa(q, k, v, mask, g.scale), atol=1e-12, rtol=0)
        s = (q @ k.T) * g.scale
        s[~mask] = -math.inf
        np.testing.assert_allclose(lse[0, h], torch.logsumexp(s, dim=1).numpy(), atol=1e-12, rtol=0)


def test_probabilities_sum_to_one_and_masked_are_zero():
    """With V = identity (d >= N + L) the output rows are the softmax rows."""
    g = geom(4, 8, 2, 2, r=1, lr=(2, 2), heads=1, d=64)
    assert g.N + g.L <= g.head_dim
    x = inputs(g, 5)
    eye = np.eye(g.N + g.L, g.head_dim)
    x["v_hr"] = O.f64_to_bf16(eye[:g.N].reshape(1, g.N, 1, -1))
    x["v_lr"] = O.f64_to_bf16(eye[g.N:].reshape(1, g.L, 1, -1))
    o, _ = run(g, x)
    P = o[0, :, 0, :g.N + g.L]
    np.testing.assert_allclose(P.sum(axis=1), 1.0, atol=1e-12)
    mask = cell_mask(g, O.HR_WINDOW_FIRST)
    assert np.all(P[~mask] == 0.0)
    assert np.all(P[mask] > 0.0)


def test_constant_values_and_convex_hull():
    g = geom(8, 8, 4, 4, r=1, lr=(2, 2), heads=1, d=16)
    x = inputs(g, 6)
    c = O.f64_to_bf16(np.full((1, g.N, 1, 16), 0.375))
    xc = dict(x, v_hr=c, v_lr=O.f64_to_bf16(np.full((1, g.L, 1, 16), 0.375)))
    o, _ = run(g, xc)
    np.testing.assert_allclose(o, 0.375, atol=1e-15, rtol=0)
    o, _ = run(g, x)
    mask = cell_mask(g, O.HR_WINDOW_FIRST)
    V = joint(x, "v", 0, 0).numpy()
    for i in range(g.N + g.L):
        vis = V[mask[i]]
        assert np.all(o[0, i, 0] <= vis.max(axis=0) + 1e-12)
        assert np.all(o[0, i, 0] >= vis.min(axis=0) - 1e-12)


def test_two_key_closed_form():
    """1x2 grid of 1x1 windows, radius 0, one low-res token.  High-res query
    0 sees its own key and the low-res key; the low-res query sees only the
    low-res key, so its output is that value exactly."""
    g = O.Geometry(batch=1, grid_h=1, grid_w=2, win_h=1, win_w=1, radius=0, lr_h=1, lr_w=1,
                   rho=4.0, heads=1, head_dim=4, rope_dim_y=2, rope_dim_x=2, softmax_scale=0.5)
    f = lambda a: O.f64_to_bf16(np.array(a, dtype=np.float64).reshape(1, -1, 1, 4))
    x = dict(q_hr=f([[1, 0, 0, 0], [0, 2, 0, 0]]), k_hr=f([[2, 0, 0, 0], [0, 0, 1, 0]]),
             v_hr=f([[1, 0, 0, 0], [0, 1, 0, 0]]), q_lr=f([[0, 0, 0, 1]]),
             k_lr=f([[1, 1, 0, 0]]), v_lr=f([[0, 0, 4, 0]]))
    o, lse = run(g, x, O.HR_RASTER)
    # query 0: s = 0.5*<q0,k0> = 1, s_lr = 0.5*<q0,k_lr> = 0.5
    p0 = math.exp(1.0) / (math.exp(1.0) + math.exp(0.5))
    np.testing.assert_allclose(o[0, 0, 0], [p0, 0, 4 * (1 - p0), 0], atol=1e-15)
    np.testing.assert_allclose(lse[0, 0, 0], math.log(math.exp(1.0) + math.exp(0.5)), atol=1e-15)
    # query 1: s = 0.5*<q1,k1> = 0, s_lr = 0.5*<q1,k_lr> = 1
    p1 = 1.0 / (1.0 + math.exp(1.0))
    np.testing.assert_allclose(o[0, 1, 0], [0, p1, 4 * (1 - p1), 0], atol=1e-15)
    np.testing.assert_allclose(o[0, 2, 0], [0, 0, 4, 0], atol=0)
    np.testing.assert_allclose(lse[0, 0, 2], 0.0, atol=0)


def test_equivariant_under_window_first_reordering():
    g = geom(12, 16, 4, 4, r=1, lr=(2, 3), heads=2, d=16, batch=2)
    x = inputs(g, 7)
    xw = {k: (O.permute_window_first(v, g) if k.endswith("_hr") else v) for k, v in x.items()}
    o_r, l_r = run(g, x, O.HR_RASTER)
    o_w, l_w = run(g, xw, O.HR_WINDOW_FIRST)
    N = g.N
    np.testing.assert_allclose(O.permute_window_first(o_r[:, :N], g), o_w[:, :N], atol=1e-13, rtol=0)
    np.testing.assert_allclose(o_r[:, N:], o_w[:, N:], atol=1e-13, rtol=0)
    np.testing.assert_allclose(O.permute_window_first(l_r[:, :, :N].transpose(0, 2, 1), g),
                               l_w[:, :, :N].transpose(0, 2, 1), atol=1e-13, rtol=0)


def test_row_subsets_match_full():
    g = geom(12, 16, 4, 4, r=1, lr=(2, 3))
    x = inputs(g, 8)
    o, lse = run(g, x)
    rows = np.array([0, 5, 17, g.N - 1, g.N, g.N + g.L - 1, 40])
    o2, l2 = run(g, x, rows=rows)
    np.testing.assert_array_equal(o2, o[:, rows])
    np.testing.assert_array_equal(l2, lse[:, :, rows])


@pytest.mark.parametrize("H,W,wh,ww,r,lr", [(32, 32, 8, 8, 1, (8, 8)), (128, 128, 16, 16, 1, (32, 32)),
                                             (24, 40, 8, 8, 2, (3, 5)), (48, 36, 12, 12, 1, (7, 5))])
def test_visible_pair_counts_closed_form(H, W, wh, ww, r, lr):
    """Per head: high-res/high-res pairs = T^2 * sum_w |N(w)|, and the clipped
    neighbour count factorises per axis: sum over n windows of the clipped
    span, n(2r+1) - r(r+1) when n > r."""
    g = geom(H, W, wh, ww, r=r, lr=lr)
    span = lambda n: sum(min(n, w + r + 1) - max(0, w - r) for w in range(n))
    closed = lambda n: n * (2 * r + 1) - r * (r + 1) if n > r else n * n
    ny, nx = H // wh, W // ww
    assert span(ny) == closed(ny) and span(nx) == closed(nx)
    cnt = O.visible_pairs(g)
    assert cnt["hr_hr"] == (wh * ww) ** 2 * closed(ny) * closed(nx)
    assert cnt["hr_lr"] == g.N * g.L
    assert cnt["lr_lr"] == g.L ** 2


def test_layer_is_rope_then_attention():
    """layer_forward on raster inputs equals: rotate (raster positions), move
    to window-first order, attend there, move back."""
    g = geom(16, 16, 8, 8, r=1, lr=(4, 4), heads=2, d=16)
    x = inputs(g, 9)
    o, lse = O.layer_forward(x, g)
    r = {k: O.rope_2d(x[k], g, O.HR_RASTER) for k in ("q_hr", "k_hr")}
    r.update({k: O.rope_2d(x[k], g, O.LOWRES) for k in ("q_lr", "k_lr")})
    wf = {k: O.permute_window_first(v, g) for k, v in r.items() if k.endswith("_hr")}
    o2, l2 = O.attention(wf["q_hr"], wf["k_hr"], O.permute_window_first(x["v_hr"], g),
                         r["q_lr"], r["k_lr"], x["v_lr"], g, O.HR_WINDOW_FIRST)
    N = g.N
    np.testing.assert_allclose(O.unpermute(o2[:, :N], g), o[:, :N], atol=1e-13, rtol=0)
    np.testing.assert_allclose(o2[:, N:], o[:, N:], atol=1e-13, rtol=0)
    rows = np.array([3, 100, N + 2])
    o3, l3 = O.layer_forward(x, g, rows=rows)
    np.testing.assert_allclose(o3, o[:, rows], atol=1e-14, rtol=0)


# Random small geometries (ragged grids, radius 0-3, text tokens, any
# low-res grid): the oracle against torch's fp64 attention with the mask
# enumerated cell by cell.
from hypothesis import HealthCheck, given, settings  # noqa: E402
from hypothesis import strategies as st  # noqa: E402


@st.composite
def small_geometries(draw):
    wh, ww = draw(st.integers(1, 4)), draw(st.integers(1, 4))
    lr = draw(st.sampled_from([(0, 0), (1, 1), (2, 3)]))
    g = O.Geometry(batch=1, grid_h=wh * draw(st.integers(1, 4)), grid_w=ww * draw(st.integers(1, 4)),
                   win_h=wh, win_w=ww, radius=draw(st.integers(0, 3)), lr_h=lr[0], lr_w=lr[1],
                   rho=4.0, heads=1, head_dim=8, rope_dim_y=4, rope_dim_x=4,
                   text_len=draw(st.integers(0, 5)))
    return g, draw(st.sampled_from([O.HR_WINDOW_FIRST, O.HR_RASTER])), draw(st.integers(0, 99))


@settings(max_examples=60, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(small_geometries())
def test_random_geometries_match_library_with_enumerated_mask(case):
    g, order, seed = case
    if g.N + g.L == 0:
        return
    x = inputs(g, seed)
    o, lse = run(g, x, order)
    mask = torch.from_numpy(cell_mask(g, order))
    q, k, v = joint(x, "q", 0, 0), joint(x, "k", 0, 0), joint(x, "v", 0, 0)
    np.testing.assert_allclose(o[0, :, 0], sdpa(q, k, v, mask, g.scale), atol=1e-12, rtol=0)
    s = (q @ k.T) * g.scale
    s[~mask] = -math.inf
    np.testing.assert_allclose(lse[0, 0], torch.logsumexp(s, dim=1).numpy(), atol=1e-12, rtol=0)
