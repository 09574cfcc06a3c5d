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


def half_ulp_bf16(x: np.ndarray) -> np.ndarray:
    """Half a bf16 ulp of |x|: 2^(e - 8) for 2^e <= |x| < 2^(e+1) (8-bit
    significand), the most that rounding x to bf16 can move it."""
    m, e = np.frexp(np.abs(x))  # |x| = m 2^e, 0.5 <= m < 1
    return np.where(x == 0, 0.0, np.ldexp(1.0, e - 9))


def err_stats(got: np.ndarray, ref: np.ndarray, v_scale=None):
    """(max-abs, mean-abs, raw max-abs, raw bound) of got - ref over
    [..., h, d] arrays.

    Unit-variance inputs: the plain errors, held to MAX_ABS / MEAN_ABS; the
    raw values repeat the max and MAX_ABS.
    Inputs with per-head scales (v_scale, shape [h]; reading R2): the bound
    is stated for unit variance, so each head's error is divided by its value
    scale.  Larger q/k scales sharpen the softmax, so outputs reach several
    times the value scale, where the bf16 output format alone moves a value
    by up to half an ulp of |ref| (at most 2^-8 |ref|).  The first value sets
    that rounding aside element by element (never below zero) before the max
    bound applies; the mean is unchanged.  The raw max keeps it, and its
    bound is MAX_ABS plus the largest half-ulp of |ref| / scale in the head:
    the test asserts raw <= raw bound too, so the allowance is an explicit
    bound, not a silent subtraction.
    """
    d = np.abs(got - ref)
    if v_scale is None:
        return float(d.max()), float(d.mean()), float(d.max()), MAX_ABS
    s = np.asarray(v_scale, dtype=np.float64)[:, None]
    d = d / s
    hu = half_ulp_bf16(ref) / s
    dmax = np.maximum(d - hu, 0.0)
    # per head: raw max against MAX_ABS + that head's largest half-ulp; report
    # the head with the smallest margin
    ax = tuple(i for i in range(d.ndim) if i != d.ndim - 2)
    raw_h = d.max(axis=ax)
    lim_h = MAX_ABS + hu.max(axis=ax)
    k = int(np.argmax(raw_h - lim_h))
    return float(dmax.max()), float(d.mean()), float(raw_h[k]), float(lim_h[k])


# ----------------------------------------------------------------- backward

U = 2.0 ** -8  # unit roundoff of bf16: 8-bit significand, |fl(x) - x| <= 2^-8 |x|


def bwd_error_bounds(g: O.Geometry, hr_order: str, q, k, v, do, rows=None, keys=None,
                     heads=None, chunk_rows: int = 512):
    """Per-element bounds on |GPU - exact| for dQ (rows) and dK, dV (keys).

    q, k, v, do: joint-sequence fp64 arrays [B, n, h, d] (the bf16 inputs
    widened).  The kernels round P and dS to bf16 as tensor-core operands
    (relative U each), compute D = rowsum(dO * O) from the bf16 forward output
    (relative U per product, so |dD| <= 2U sum |dO O| with the fp32 sum), sum
    in fp32 and round every output to bf16 (U |result|).  With these:
      |e dV_j| <= 2U sum_i P_ij |dO_i| + U |dV_j|
      |e dS_ij| <= 2U |dS_ij| + P_ij |dD_i|
      |e dQ_i| <= scale sum_j |e dS_ij| |K_j| + U |dQ_i|, likewise dK with Q.
    These are the first-order terms, with no extra factor: the fp32
    accumulation and the approximate exp2 (relative errors near 2^-22) add
    far less than one rounding to bf16, and each bound is floored at 1e-6.
    The tests report the worst ratio error / bound, i.e. the headroom that is
    actually left.  Returns (bq, bk, bv) shaped like the oracle's
    attention_backward outputs."""
    B, n, H, d = q.shape
    rows = np.arange(n) if rows is None else np.asarray(rows, np.int64)
    keys = np.arange(n) if keys is None else np.asarray(keys, np.int64)
    heads = range(H) if heads is None else heads
    need = np.union1d(rows, O.rows_seeing(g, hr_order, keys)) if keys.size else rows
    pos = {int(r): i for i, r in enumerate(rows)}
    bq = np.zeros((B, rows.size, H, d))
    bk = np.zeros((B, keys.size, H, d))
    bv = np.zeros((B, keys.size, H, d))
    gq = np.zeros_like(bq)
    gk = np.zeros_like(bk)
    gv = np.zeros_like(bv)
    for b in range(B):
        for h in heads:
            Q, K, V, dO = q[b, :, h], k[b, :, h], v[b, :, h], do[b, :, h]
            for i0 in range(0, need.size, chunk_rows):
                r = need[i0:i0 + chunk_rows]
                s = (Q[r] @ K.T) * g.scale
                s[~O.visibility(g, hr_order, r)] = -np.inf
                p = np.exp(s - s.max(axis=1, keepdims=True))
                p /= p.sum(axis=1, keepdims=True)
                o = p @ V
                dP = dO[r] @ V.T
                D = (p * dP).sum(axis=1, keepdims=True)
                dS = p * (dP - D)
                dD = 2 * U * (np.abs(dO[r]) * np.abs(o)).sum(axis=1, keepdims=True)
                eS = 2 * U * np.abs(dS) + p * dD
                eq = g.scale * (eS @ np.abs(K))
                gq_c = g.scale * (dS @ K)
                for j, ri in enumerate(r):
                    t = pos.get(int(ri))
                    if t is not None:
                        bq[b, t, h] = eq[j]
                        gq[b, t, h] = gq_c[j]
                bk[b, :, h] += g.scale * (eS.T @ np.abs(Q[r]))[keys]
                gk[b, :, h] += g.scale * (dS.T @ Q[r])[keys]
                bv[b, :, h] += 2 * U * (p.T @ np.abs(dO[r]))[keys]
                gv[b, :, h] += (p.T @ dO[r])[keys]
    fin = lambda e, gg: e + U * np.abs(gg) + 1e-6
    return fin(bq, gq), fin(bk, gk), fin(bv, gv)


def joint_f64(x: dict, name: str, heads=None) -> np.ndarray:
    """[B, N + L, h, d] fp64 from the bf16 tensors name_hr, name_lr (only the
    listed heads, in that order, if given)."""
    sel = (lambda t: t) if heads is None else (lambda t: t[:, :, list(heads)])
    hr = f64(sel(x[name + "_hr"]))
    lr = f64(sel(x[name + "_lr"])) if x.get(name + "_lr") is not None else hr[:, :0]
    return np.concatenate([hr, lr], axis=1)


def rotated_bound(b: np.ndarray, ref: np.ndarray) -> np.ndarray:
    """Bound after the transposed RoPE and its bf16 rounding: a rotation moves
    an error pair (e0, e1) to components of size at most |(e0, e1)| <=
    sqrt(2) max(b0, b1); the rounding adds U |ref|."""
    m = np.maximum(b[..., 0::2], b[..., 1::2])
    out = np.repeat(m, 2, axis=-1) * np.sqrt(2.0)
    return out + U * np.abs(ref)
