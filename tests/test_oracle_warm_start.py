"""Pins for the warm-start oracle: a library routine for the upsampling
(torch's fp64 bilinear interpolation with align_corners=False is the same
half-pixel, edge-clamped sampling), closed forms for constant and linear
images, the t = 0 / t = 1 end points, and a 2x2 example worked by hand."""
import numpy as np
import torch
import torch.nn.functional as F

from oracle import warm_start as W


def test_upsample_is_torch_bilinear_half_pixel():
    rng = np.random.default_rng(0)
    for (h, w, s) in [(5, 7, 4), (3, 3, 2), (1, 4, 3), (6, 2, 8)]:
        x = rng.standard_normal((2, 3, h, w))
        want = F.interpolate(torch.from_numpy(x), scale_factor=s, mode="bilinear",
                             align_corners=False).numpy()
        np.testing.assert_allclose(W.bilinear_upsample(x, s), want, rtol=0, atol=1e-13)


def test_blur_matches_replicate_padded_convolution():
    rng = np.random.default_rng(1)
    u = rng.standard_normal((2, 1, 9, 6))
    k = torch.tensor([0.25, 0.5, 0.25], dtype=torch.float64)
    pad = F.pad(torch.from_numpy(u), (1, 1, 1, 1), mode="replicate")
    want = F.conv2d(pad, torch.outer(k, k)[None, None]).numpy()
    np.testing.assert_allclose(W.binomial_blur(u), want, rtol=0, atol=1e-14)


def test_constant_image_passes_through():
    x = np.full((1, 2, 4, 5), 0.75)
    noise = np.random.default_rng(2).standard_normal((1, 2, 16, 20))
    out = W.warm_start(x, noise, 4, 0.8, 0.3)
    np.testing.assert_allclose(out, 0.7 * 0.75 + 0.3 * noise, rtol=0, atol=1e-15)


def test_linear_ramp_is_unchanged_away_from_the_border():
    """Bilinear interpolation reproduces a linear function, and a symmetric
    blur leaves it unchanged, so the sharpened upsample equals the ramp at
    (y + 0.5)/s - 0.5 wherever no clamp is involved."""
    h, w, s = 6, 8, 4
    i, j = np.meshgrid(np.arange(h), np.arange(w), indexing="ij")
    x = (0.5 * i - 0.25 * j)[None, None].astype(np.float64)
    out = W.warm_start(x, np.zeros((1, 1, h * s, w * s)), s, 1.5, 0.0)[0, 0]
    yy, xx = np.meshgrid((np.arange(h * s) + 0.5) / s - 0.5,
                         (np.arange(w * s) + 0.5) / s - 0.5, indexing="ij")
    ramp = 0.5 * yy - 0.25 * xx
    inner = (slice(s, (h - 1) * s), slice(s, (w - 1) * s))
    np.testing.assert_allclose(out[inner], ramp[inner], rtol=0, atol=1e-14)


def test_end_points_of_t():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((1, 1, 3, 4))
    noise = rng.standard_normal((1, 1, 6, 8))
    np.testing.assert_array_equal(W.warm_start(x, noise, 2, 0.5, 1.0), noise)
    np.testing.assert_allclose(W.warm_start(x, noise, 2, 0.0, 0.0), W.bilinear_upsample(x, 2),
                               rtol=0, atol=0)


def test_two_by_two_worked_by_hand():
    """x = [[0, 1], [2, 3]] = 2i + j, s = 2, amount 1, t = 0.

    Upsampling samples at -0.25, 0.25, 0.75, 1.25, clamped to [0, 1] at the
    ends: the column part j gives [0, .25, .75, 1], the row part 2i gives
    [0, .5, 1.5, 2].  The blur (edges replicated) of [0, .25, .75, 1] is
    [.0625, .3125, .6875, .9375], of [0, .5, 1.5, 2] it is
    [.125, .625, 1.375, 1.875].  With amount 1 each part becomes 2u - blur(u):
    [-.0625, .1875, .8125, 1.0625] and [-.125, .375, 1.625, 2.125]; the image
    is their outer sum (the blur of a sum is the sum of the blurs)."""
    x = np.array([[[[0.0, 1.0], [2.0, 3.0]]]])
    col = np.array([-0.0625, 0.1875, 0.8125, 1.0625])
    row = np.array([-0.125, 0.375, 1.625, 2.125])
    want = row[:, None] + col[None, :]
    out = W.warm_start(x, np.zeros((1, 1, 4, 4)), 2, 1.0, 0.0)[0, 0]
    np.testing.assert_array_equal(out, want)


from hypothesis import given, settings  # noqa: E402
from hypothesis import strategies as st  # noqa: E402


@settings(max_examples=40, deadline=None)
@given(st.integers(1, 9), st.integers(1, 9), st.integers(1, 6), st.integers(0, 999))
def test_random_shapes_reduce_to_torch_bilinear(h, w, s, seed):
    """With no sharpening and t = 0 the state is the bilinear upsample, for
    any size and integer factor; with t = 1 it is the noise."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((1, 2, h, w))
    noise = rng.standard_normal((1, 2, h * s, w * s))
    want = F.interpolate(torch.from_numpy(x), scale_factor=s, mode="bilinear",
                         align_corners=False).numpy()
    np.testing.assert_allclose(W.warm_start(x, noise, s, 0.0, 0.0), want, rtol=0, atol=1e-13)
    np.testing.assert_array_equal(W.warm_start(x, noise, s, 0.7, 1.0), noise)
