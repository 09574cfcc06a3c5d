"""The factor-4 warm start's stencil weights, through the C ABI on the host
(no GPU): ug_warm_start_stencil_weights returns the weights the factor-4
kernel applies, so its arithmetic is checked here against the oracle
(UltraGen-ar §2.د "Warm-Start Initialization"; readings W1-W3) and against
closed forms:
  * applied to random latents (odd sizes, one-pixel planes, a 3 x 70 strip)
    with the clamped 3 x 3 neighbourhood, they reproduce the oracle's
    bilinear upsample + unsharp mask + noise blend within fp32 rounding of
    the weights, borders included;
  * each output's nine weights sum to 1 - t (bilinear weights and blur
    weights each sum to one, so the sharpening adds (1 + a) - a = 1);
  * t = 1 gives all-zero weights (pure noise), sharpen 0 gives the plain
    bilinear weights, which are the outer product of the two axes' weights.
"""
import numpy as np
import pytest

from block_sparse_local_raster_b200 import ug
from oracle import warm_start as W

S = 4


def apply(wt, x, noise, t):
    B, C, h, w = x.shape
    out = np.empty((B, C, S * h, S * w))
    for Y in range(h):
        ys = [max(Y - 1, 0), Y, min(Y + 1, h - 1)]
        for X in range(w):
            xs = [max(X - 1, 0), X, min(X + 1, w - 1)]
            nb = x[:, :, ys][:, :, :, xs]  # [B, C, 3, 3]
            for py in range(S):
                for px in range(S):
                    out[:, :, S * Y + py, S * X + px] = (
                        (nb * wt[py, px]).sum(axis=(-2, -1)) + t * noise[:, :, S * Y + py, S * X + px])
    return out


@pytest.mark.parametrize("h,w,sharpen,t", [(5, 9, 0.8, 0.45), (1, 1, 0.5, 0.6), (3, 70, 0.0, 0.0),
                                           (16, 16, 0.5, 0.6), (2, 3, 1.25, 0.3), (7, 4, 2.0, 0.9)])
def test_weights_reproduce_the_oracle(h, w, sharpen, t):
    rng = np.random.default_rng(h * 100 + w)
    x = rng.standard_normal((2, 3, h, w))
    noise = rng.standard_normal((2, 3, S * h, S * w))
    wt = ug.warm_start_stencil_weights(sharpen, t).astype(np.float64)
    want = W.warm_start(x, noise, S, sharpen, t)
    got = apply(wt, x, noise, t)
    m = max(np.abs(x).max(), np.abs(noise).max())
    # each weight is within 2^-24 relative of its exact value; sum |w| <= (1 - t)(1 + 2 sharpen)
    assert np.abs(got - want).max() <= 2.0 ** -22 * (1 + 2 * sharpen) * m


@pytest.mark.parametrize("sharpen,t", [(0.5, 0.6), (1.25, 0.3), (0.0, 0.0), (3.0, 0.05)])
def test_each_output_weights_sum_to_one_minus_t(sharpen, t):
    wt = ug.warm_start_stencil_weights(sharpen, t).astype(np.float64)
    np.testing.assert_allclose(wt.sum(axis=(-2, -1)), 1.0 - t, rtol=0, atol=2e-6 * (1 + 2 * sharpen))


def test_end_points():
    assert not ug.warm_start_stencil_weights(0.7, 1.0).any()
    wt = ug.warm_start_stencil_weights(0.0, 0.0).astype(np.float64)
    # plain bilinear: phase p samples Y + (p + 0.5)/4 - 0.5 between two source rows
    e = np.zeros((S, 3))
    for p in range(S):
        q = (p + 0.5) / S - 0.5
        fl = int(np.floor(q))
        e[p, fl + 1] += 1 - (q - fl)
        e[p, fl + 2] += q - fl
    np.testing.assert_array_equal(wt, np.einsum("ar,bc->abrc", e, e))


def test_argument_errors():
    import ctypes
    buf = (ctypes.c_float * 144)()
    assert ug.lib().ug_warm_start_stencil_weights(0.5, 1.5, buf) == ug.UG_ERR_INVALID_ARG
    assert ug.lib().ug_warm_start_stencil_weights(float("nan"), 0.5, buf) == ug.UG_ERR_INVALID_ARG
    assert ug.lib().ug_warm_start_stencil_weights(0.5, 0.5, None) == ug.UG_ERR_INVALID_ARG
