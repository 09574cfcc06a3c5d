"""fp64 CPU oracle of UltraGen's warm-start initialisation.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's
CPU-baseline leg may import this module.  It shares nothing with the CUDA
library.

What the pages state (UltraGen-ar §2.د "Warm-Start Initialization"; UltraGen-fr
§2.D "Accélération par Initialisation"; UltraGen-it §2, inference item): the
low-res result is upsampled to the high-res size, sharpened, and combined with
Gaussian noise as the high-res state at an intermediate timestep, so that the
sampler skips the early denoising steps.

Readings where the pages are silent (each is listed in the design notes):
  * the state is a latent image [B, C, H, W]; the high-res size is the
    low-res size times an integer factor s (rho = 4 between the token grids of
    the pages' configs);
  * upsampling is bilinear with half-pixel centres: high-res pixel (y, x)
    samples the low-res image at ((y + 0.5) / s - 0.5, (x + 0.5) / s - 0.5),
    reading indices clamped to the image (edge replicate);
  * sharpening is an unsharp mask: u + lambda * (u - blur(u)), blur the 3x3
    binomial filter (1/4, 1/2, 1/4) in each direction, edges replicated;
  * the combination is the rectified-flow interpolation of FLUX-class
    samplers at timestep t: x_t = (1 - t) * x0 + t * noise, t = 1 is pure
    noise.  The noise is an input (the caller draws it).
"""
from __future__ import annotations

import numpy as np


def bilinear_upsample(x: np.ndarray, s: int) -> np.ndarray:
    """x: [..., h, w] -> [..., h*s, w*s], fp64, half-pixel centres, edge clamp."""
    h, w = x.shape[-2:]

    def taps(n_lo: int):
        dst = np.arange(n_lo * s, dtype=np.float64)
        src = (dst + 0.5) / s - 0.5
        i0 = np.floor(src).astype(np.int64)
        f = src - i0
        return np.clip(i0, 0, n_lo - 1), np.clip(i0 + 1, 0, n_lo - 1), f

    y0, y1, fy = taps(h)
    x0, x1, fx = taps(w)
    x = np.asarray(x, dtype=np.float64)
    rows = x[..., y0, :] * (1.0 - fy)[:, None] + x[..., y1, :] * fy[:, None]
    return rows[..., :, x0] * (1.0 - fx) + rows[..., :, x1] * fx


def binomial_blur(u: np.ndarray) -> np.ndarray:
    """3x3 binomial blur (1/4, 1/2, 1/4) x (1/4, 1/2, 1/4), edges replicated."""
    H, W = u.shape[-2:]
    w = (0.25, 0.5, 0.25)
    out = np.zeros_like(u, dtype=np.float64)
    for dy in (-1, 0, 1):
        ry = np.clip(np.arange(H) + dy, 0, H - 1)
        for dx in (-1, 0, 1):
            rx = np.clip(np.arange(W) + dx, 0, W - 1)
            out += w[dy + 1] * w[dx + 1] * u[..., ry, :][..., :, rx]
    return out


def sharpen(u: np.ndarray, amount: float) -> np.ndarray:
    """Unsharp mask: u + amount * (u - blur(u))."""
    return u + amount * (u - binomial_blur(u))


def warm_start(x_lr: np.ndarray, noise: np.ndarray, scale: int, amount: float,
               t: float) -> np.ndarray:
    """x_lr: [B, C, h, w]; noise: [B, C, h*s, w*s].  Returns the fp64 state
    (1 - t) * sharpen(upsample(x_lr)) + t * noise."""
    x0 = sharpen(bilinear_upsample(x_lr, scale), amount)
    return (1.0 - t) * x0 + t * np.asarray(noise, dtype=np.float64)
