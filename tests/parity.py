"""Shared helpers of the GPU parity tests: inputs, row sampling, error stats."""
import numpy as np
import torch

from block_sparse_local_raster_b200 import ug, workloads
from oracle import hier_local_attn as O

# Tolerance for the attention output on unit-variance inputs, in units of the
# values' scale: max-abs 1e-2 and mean-abs 1e-3.
MAX_ABS = 1e-2
MEAN_ABS = 1e-3
# lse (natural log of the softmax denominator): fp32 accumulation of up to
# ~3e5 bf16-rounded exponentials; its value is O(10); absolute bound.
LSE_ABS = 2e-3


def bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().to(torch.float64).numpy()


def ogeom(wl) -> O.Geometry:
    return O.Geometry.from_dict(wl.geom_dict())


def plan(wl) -> ug.Plan:
    return ug.Plan(**wl.geom_dict())


def sample_hr_tokens(g: O.Geometry, order: str, seed: int, n_interior: int = 4,
                     per_window: int = 6) -> np.ndarray:
    """Stratified high-res rows: the four corner windows, four edge windows,
    random interior windows; in each, its first and last token and random
    others.  Returned as token indices in ``order``."""
    rng = np.random.default_rng(seed)
    ny, nx = g.n_win_y, g.n_win_x
    wins = {(0, 0), (0, nx - 1), (ny - 1, 0), (ny - 1, nx - 1),
            (0, nx // 2), (ny - 1, nx // 2), (ny // 2, 0), (ny // 2, nx - 1)}
    for _ in range(n_interior):
        wins.add((int(rng.integers(0, ny)), int(rng.integers(0, nx))))
    T = g.T
    toks = []
    for wy, wx in sorted(wins):
        w = wy * nx + wx
        local = {0, T - 1} | set(rng.integers(0, T, size=per_window).tolist())
        toks += [w * T + l for l in sorted(local)]
    toks = np.array(sorted(set(toks)), dtype=np.int64)  # window-first indices
    if order == O.HR_RASTER:
        toks = O.raster_index(g)[toks]
    return np.sort(toks)


def sample_lr_tokens(g: O.Geometry, seed: int, n: int = 12) -> np.ndarray:
    if g.L == 0:
        return np.zeros(0, dtype=np.int64)
    rng = np.random.default_rng(seed + 1)
    t = {0, g.L - 1} | set(rng.integers(0, g.L, size=n).tolist())
    if g.text_len:  # both sides of the text / low-res boundary
        t |= {g.text_len - 1, min(g.text_len, g.L - 1)}
    return np.array(sorted(t), dtype=np.int64)


def err_stats(got: np.ndarray, ref: np.ndarray, v_scale=None):
    """(max-abs, mean-abs) of got - ref over [..., h, d] arrays.

    Unit-variance inputs: the plain errors, held to MAX_ABS / MEAN_ABS.
    Inputs with per-head scales (v_scale, shape [h]): the bound is stated for
    unit variance, so each head's error is divided by its value scale; and
    because larger q/k scales sharpen the softmax, outputs reach several
    times the value scale, where the bf16 output format alone rounds by up to
    half an ulp, at most 2^-8 |ref| (unit roundoff of an 8-bit significand).
    That part is subtracted (never below zero)
    before the max bound applies; the mean bound is unchanged.
    """
    d = np.abs(got - ref)
    if v_scale is None:
        return float(d.max()), float(d.mean())
    s = np.asarray(v_scale, dtype=np.float64)[:, None]
    d = d / s
    dmax = np.maximum(d - 2.0 ** -8 * np.abs(ref) / s, 0.0)
    return float(dmax.max()), float(d.mean())
