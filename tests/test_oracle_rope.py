"""Pins for the oracle's 2-D axial RoPE with rho-scaled low-res positions."""
import math
import os

import numpy as np
import pytest

from oracle import hier_local_attn as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def geom(H=32, W=32, wh=8, ww=8, lr=(8, 8), rho=4.0, heads=2, d=64, ay=None, theta=10000.0):
    ay = d // 2 if ay is None else ay
    return O.Geometry(batch=1, grid_h=H, grid_w=W, win_h=wh, win_w=ww, radius=1,
                      lr_h=lr[0], lr_w=lr[1], rho=rho, heads=heads, head_dim=d,
                      rope_dim_y=ay, rope_dim_x=d - ay, rope_theta=theta)


def rand_bits(shape, seed=0):
    x = np.random.default_rng(seed).standard_normal(shape).astype(np.float32)
    return O.f64_to_bf16(x.astype(np.float64))


def test_golden_worked_example():
    g = geom(H=4, W=4, wh=2, ww=2, lr=(2, 2), rho=4.0, heads=1, d=8, ay=4)
    cases = {}
    for line in open(os.path.join(GOLDEN, "rope_worked_example.txt")):
        if line.strip() and not line.startswith("#"):
            tag, a, b, *vals = line.split()
            cases[tag] = (int(a), int(b), np.array(vals, dtype=np.float64))
    x = np.array([1, 0, 0, 1, 1, 0, 0, 1], dtype=np.float64).reshape(1, 1, 1, 8)
    y, xx, want = cases["A"]
    got = O.rope_2d_f64(x, g, O.HR_RASTER, tokens=np.array([y * g.grid_w + xx]))
    # The tables hold fp32-rounded cos/sin: agreement to fp32 precision.
    np.testing.assert_allclose(got.ravel(), want, rtol=0, atol=2 ** -24)
    i, j, want = cases["B"]
    got = O.rope_2d_f64(x, g, O.LOWRES, tokens=np.array([i * g.lr_w + j]))
    np.testing.assert_allclose(got.ravel(), want, rtol=0, atol=2 ** -24)


def test_position_zero_is_identity():
    g = geom()
    x = rand_bits((1, 1, 2, 64))
    np.testing.assert_array_equal(O.rope_2d(x, g, O.HR_RASTER, tokens=np.array([0])), x)
    np.testing.assert_array_equal(O.rope_2d(x, g, O.LOWRES, tokens=np.array([0])), x)


def test_pairs_keep_their_norm():
    g = geom()
    x = O.bf16_to_f64(rand_bits((1, g.N, 2, 64), 3))
    y = O.rope_2d_f64(x, g, O.HR_RASTER)
    n0 = x[..., 0::2] ** 2 + x[..., 1::2] ** 2
    n1 = y[..., 0::2] ** 2 + y[..., 1::2] ** 2
    # |c^2 + s^2 - 1| <= ~2^-23 for fp32-rounded cos/sin
    np.testing.assert_allclose(n1, n0, rtol=3e-7, atol=1e-30)


def test_relative_position_property():
    """<R(p)q, R(p')k> depends on p - p' only: shift every position by the
    same offset (along each axis) and the dot products do not move."""
    g = geom(H=64, W=64, lr=(0, 0))
    rng = np.random.default_rng(5)
    q = O.bf16_to_f64(rand_bits((1, 1, 1, 64), 6))
    k = O.bf16_to_f64(rand_bits((1, 1, 1, 64), 7))
    for _ in range(20):
        y0, x0, y1, x1 = rng.integers(0, 32, size=4)
        dy, dx = rng.integers(0, 32, size=2)
        def dot(ya, xa, yb, xb):
            a = O.rope_2d_f64(q, g, O.HR_RASTER, tokens=np.array([ya * 64 + xa]))
            b = O.rope_2d_f64(k, g, O.HR_RASTER, tokens=np.array([yb * 64 + xb]))
            return float((a * b).sum())
        assert abs(dot(y0, x0, y1, x1) - dot(y0 + dy, x0 + dx, y1 + dy, x1 + dx)) < 1e-4


def test_axes_own_their_channels():
    """Moving a token along x leaves channels [0, a_y) untouched; moving it
    along y leaves [a_y, d) untouched (axial split)."""
    g = geom(d=128, ay=48, H=16, W=16, wh=4, ww=4, lr=(0, 0))
    x = rand_bits((1, 1, 1, 128), 9)
    a = O.rope_2d(x, g, O.HR_RASTER, tokens=np.array([3 * 16 + 5]))
    b = O.rope_2d(x, g, O.HR_RASTER, tokens=np.array([3 * 16 + 11]))
    c = O.rope_2d(x, g, O.HR_RASTER, tokens=np.array([9 * 16 + 5]))
    np.testing.assert_array_equal(a[..., :48], b[..., :48])
    assert (a[..., 48:] != b[..., 48:]).any()
    np.testing.assert_array_equal(a[..., 48:], c[..., 48:])
    assert (a[..., :48] != c[..., :48]).any()


def test_rho_scales_lowres_positions():
    """Low-res token (i, j) sits at high-res position (rho*i, rho*j): with an
    integer rho it rotates exactly like the high-res token there."""
    g = geom(H=32, W=32, lr=(8, 8), rho=4.0)
    x = rand_bits((1, 64, 2, 64), 11)
    lr = O.rope_2d(x, g, O.LOWRES)
    i, j = np.divmod(np.arange(64), 8)
    hr = O.rope_2d(x, g, O.HR_RASTER, tokens=(4 * i) * 32 + 4 * j)
    np.testing.assert_array_equal(lr, hr)


def test_rope_commutes_with_permutation():
    g = geom(H=24, W=40, wh=8, ww=8, lr=(0, 0))
    x = rand_bits((2, g.N, 2, 64), 13)
    a = O.rope_2d(O.permute_window_first(x, g), g, O.HR_WINDOW_FIRST)
    b = O.permute_window_first(O.rope_2d(x, g, O.HR_RASTER), g)
    np.testing.assert_array_equal(a, b)


def test_rotation_is_complex_multiplication():
    """Pair (x0, x1) as x0 + i x1, rotated by the unit complex number of the
    table angle: numpy's complex128 product gives the same fp64 values."""
    g = geom(H=8, W=8, wh=4, ww=4, lr=(0, 0), d=16)
    x = O.bf16_to_f64(rand_bits((1, 64, 1, 16), 17))
    y = O.rope_2d_f64(x, g, O.HR_RASTER)
    tab = O.rope_tables(g)
    yy, xx = np.divmod(np.arange(64), 8)
    z = x[0, :, 0, 0::2] + 1j * x[0, :, 0, 1::2]
    ang = np.concatenate([tab["hr_y"][0][yy] + 1j * tab["hr_y"][1][yy],
                          tab["hr_x"][0][xx] + 1j * tab["hr_x"][1][xx]], axis=1)
    w = z * ang.astype(np.complex128)
    np.testing.assert_allclose(y[0, :, 0, 0::2], w.real, rtol=0, atol=1e-15)
    np.testing.assert_allclose(y[0, :, 0, 1::2], w.imag, rtol=0, atol=1e-15)


def test_frequency_ladder():
    """Pair k of an a-channel axis turns by theta^(-2k/a) rad per position
    step: the angle between positions 1 and 0, read back with atan2."""
    g = geom(H=8, W=8, wh=4, ww=4, lr=(0, 0), d=32)
    tab = O.rope_tables(g)
    c, s = tab["hr_y"][0][1].astype(np.float64), tab["hr_y"][1][1].astype(np.float64)
    ang = np.arctan2(s, c)
    want = np.array([10000.0 ** (-k / 8.0) for k in range(8)])  # a = 16 -> 2k/16 = k/8
    np.testing.assert_allclose(ang, want, rtol=1e-6)
    np.testing.assert_array_equal(tab["hr_y"][0][0], np.ones(8, np.float32))


from hypothesis import given, settings  # noqa: E402
from hypothesis import strategies as st  # noqa: E402


@settings(max_examples=40, deadline=None)
@given(st.sampled_from([16, 32, 64]), st.integers(0, 200), st.integers(0, 200),
       st.integers(0, 200), st.integers(0, 999))
def test_random_positions_rotation_properties(a, p1, p2, shift, seed):
    """One axis of a positions p1, p2 (exact fp64 rotation before rounding):
    pair norms are preserved, <R(p1) x, R(p2) y> depends only on p2 - p1
    up to the fp32 rounding of cos and sin, and the transpose is the adjoint."""
    rng = np.random.default_rng(seed)
    f = O.rope_frequencies(a, 10000.0)
    c, s_ = O._cos_sin_table([float(p1), float(p2), float(p1 + shift), float(p2 + shift)], f)
    c, s_ = c.astype(np.float64), s_.astype(np.float64)
    x = rng.standard_normal(a)
    y = rng.standard_normal(a)
    rx = O.rope_rotate_f64(x, c[0], s_[0])
    np.testing.assert_allclose(np.hypot(rx[0::2], rx[1::2]), np.hypot(x[0::2], x[1::2]),
                               rtol=1e-6)
    ry = O.rope_rotate_f64(y, c[1], s_[1])
    rx2 = O.rope_rotate_f64(x, c[2], s_[2])
    ry2 = O.rope_rotate_f64(y, c[3], s_[3])
    np.testing.assert_allclose(rx @ ry, rx2 @ ry2, rtol=0, atol=1e-5 * (1 + abs(rx @ ry)))
    np.testing.assert_allclose(rx @ y, x @ O.rope_rotate_f64(y, c[0], -s_[0]), rtol=0,
                               atol=1e-12)
