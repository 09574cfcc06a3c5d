"""fp64 CPU oracle of one hierarchical-local-attention layer (UltraGen).

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's
CPU-baseline leg may import this module.  It shares no code with the CUDA
library (no kernels, headers, tables or helpers): it rebuilds every index map
and table itself, from the definitions below, and it imports nothing from the
package.  It is deliberately slow and plain: numpy in float64, explicit index
arithmetic, dense attention over the whole joint sequence with an explicit
-inf mask, and a library matmul as the only composite step.

Sources.  "UltraGen-xx" is the gist.science summary of arXiv 2510.16325
("UltraGen: Efficient Ultra-High-Resolution Image Generation with Hierarchical
Local Attention") in language xx; the section follows.

  * Fixed non-overlapping windows, window-first token order
    (UltraGen-it §2 "Attenzione Gerarchica Locale con Permutazione Window-First";
    UltraGen-fr §2.A "Découpage en fenêtres", "Ordre Window-First";
    UltraGen-ar §2.أ).
  * Low-res guidance tokens with RoPE positions multiplied by rho (= 4 on the
    pages) (UltraGen-ar §2.ب "Scaled Positional Embeddings";
    UltraGen-fr §2.B; UltraGen-es §2 "Guía Global de Baja Resolución").
  * The joint MMDiT sequence concatenates text, high-res and low-res tokens
    (UltraGen-it §2, LoRA item; UltraGen-fr §2.C).
  * The attention mask: a high-res window sees itself, its adjacent windows and
    every low-res token; low-res tokens see each other
    (UltraGen-ar §2.ب "Attention Masking"; UltraGen-es §2, last bullet of the
    guidance item).  One joint softmax over local and low-res keys
    (UltraGen-it §2: a window "looks at" both its own tokens and the guidance).

Readings where the pages are silent (each is listed in the design notes):
  * window-first order = windows in raster order, tokens in raster order inside
    each window; "adjacent" = Chebyshev distance <= radius (3x3 for radius 1),
    clipped at the border, no wrap;
  * high-res RoPE positions are the token's global (y, x); low-res token (i, j)
    sits at (rho*i, rho*j) (multiply only);
  * axial RoPE: channels [0, a_y) rotate with y, [a_y, d) with x; pairs are
    adjacent channels (2k, 2k+1) of a segment; frequency f_k = theta^(-2k/a);
    cos/sin evaluated in fp64 by the C library and rounded to fp32; each output
    is x0*c - x1*s (or x0*s + x1*c) from exact fp64 products with one fp64
    rounding, then rounded to nearest-even bf16;
  * low-res queries do not see high-res keys; softmax scale 1/sqrt(d);
  * text tokens (the pages give no mask for them) join the low-res tokens in
    one global set, placed first: every query sees them, they see the global
    set only, and having no grid position they are not rotated.

bf16 values travel as their uint16 bit patterns (numpy has no bf16 type).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Iterable, Optional, Sequence, Tuple

import numpy as np

HR_RASTER = "raster"
HR_WINDOW_FIRST = "window_first"
LOWRES = "lowres"


@dataclasses.dataclass(frozen=True)
class Geometry:
    batch: int
    grid_h: int
    grid_w: int
    win_h: int
    win_w: int
    radius: int
    lr_h: int
    lr_w: int
    rho: float
    heads: int
    head_dim: int
    rope_dim_y: int
    rope_dim_x: int
    rope_theta: float = 10000.0
    softmax_scale: float = 0.0
    text_len: int = 0

    @staticmethod
    def from_dict(d: dict) -> "Geometry":
        names = {f.name for f in dataclasses.fields(Geometry)}
        return Geometry(**{k: v for k, v in d.items() if k in names})

    def __post_init__(self):
        if self.grid_h % self.win_h or self.grid_w % self.win_w:
            raise ValueError("windows must tile the grid exactly (no padding)")
        if self.rope_dim_y + self.rope_dim_x != self.head_dim:
            raise ValueError("axial RoPE split must sum to head_dim")
        if self.rope_dim_y % 2 or self.rope_dim_x % 2:
            raise ValueError("RoPE segments must hold whole pairs")
        if self.text_len < 0:
            raise ValueError("text_len must be >= 0")

    @property
    def N(self) -> int:
        return self.grid_h * self.grid_w

    @property
    def L(self) -> int:
        """Global tokens: ``text_len`` text tokens, then the low-res grid."""
        return self.text_len + self.lr_h * self.lr_w

    @property
    def T(self) -> int:
        return self.win_h * self.win_w

    @property
    def n_win_y(self) -> int:
        return self.grid_h // self.win_h

    @property
    def n_win_x(self) -> int:
        return self.grid_w // self.win_w

    @property
    def scale(self) -> float:
        return self.softmax_scale if self.softmax_scale else 1.0 / math.sqrt(self.head_dim)


# --------------------------------------------------------------------------
# Window-first permutation (UltraGen-fr §2.A "Ordre Window-First")
# --------------------------------------------------------------------------

def window_first_index(g: Geometry) -> np.ndarray:
    """perm[r] = p: the window-first position of the raster token r.

    Raster token r sits at (y, x) = (r // W, r % W), inside window
    (wy, wx) = (y // wh, x // ww) at local offset (ly, lx) = (y % wh, x % ww).
    Windows are numbered in raster order, w = wy * nWx + wx, and occupy the
    contiguous range [w*T, (w+1)*T); inside, tokens keep raster order.
    """
    r = np.arange(g.N, dtype=np.int64)
    y, x = np.divmod(r, g.grid_w)
    wy, ly = np.divmod(y, g.win_h)
    wx, lx = np.divmod(x, g.win_w)
    return (wy * g.n_win_x + wx) * g.T + ly * g.win_w + lx


def raster_index(g: Geometry) -> np.ndarray:
    """inv[p] = r, the inverse of ``window_first_index``."""
    perm = window_first_index(g)
    inv = np.empty_like(perm)
    inv[perm] = np.arange(g.N, dtype=np.int64)
    return inv


def permute_window_first(x: np.ndarray, g: Geometry) -> np.ndarray:
    """x: [B, N, ...] in raster order -> [B, N, ...] window-first (bit copy)."""
    out = np.empty_like(x)
    out[:, window_first_index(g)] = x
    return out


def unpermute(x_wf: np.ndarray, g: Geometry) -> np.ndarray:
    """x_wf: [B, N, ...] window-first -> raster order (bit copy)."""
    return x_wf[:, window_first_index(g)]


def window_neighbours(g: Geometry) -> Tuple[np.ndarray, np.ndarray]:
    """CSR lists of visible windows: (off[nWin+1], idx[...]).

    Window w = (wy, wx) lists every window (vy, vx) of the grid with
    |vy - wy| <= radius and |vx - wx| <= radius (itself included), in
    ascending raster window id.  UltraGen-ar §2.ب: local windows attend to
    themselves and to the neighbouring windows.
    """
    off = [0]
    idx = []
    for wy in range(g.n_win_y):
        for wx in range(g.n_win_x):
            for vy in range(max(0, wy - g.radius), min(g.n_win_y, wy + g.radius + 1)):
                for vx in range(max(0, wx - g.radius), min(g.n_win_x, wx + g.radius + 1)):
                    idx.append(vy * g.n_win_x + vx)
            off.append(len(idx))
    return np.asarray(off, dtype=np.int64), np.asarray(idx, dtype=np.int64)


# --------------------------------------------------------------------------
# bf16 <-> fp64
# --------------------------------------------------------------------------

def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening: a bf16 pattern is the top half of an fp32 pattern."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    with np.errstate(invalid="ignore"):
        return b.view(np.float32).astype(np.float64)


def f64_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round fp64 to the nearest bf16 (ties to even), per IEEE 754.

    bf16 has 8 significant bits and fp32's exponent range: for |x| with
    binade exponent e (2^e <= |x| < 2^(e+1)), the spacing of bf16 values is
    2^(max(e, -126) - 7) (-126 is the lowest normal binade; below it the
    spacing stays 2^-133).  Dividing by a power of two is exact, so
    rint(|x| / q) * q is the correctly rounded magnitude; it is then exactly an
    fp32 value whose upper 16 bits are the bf16 pattern.
    """
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    _, ex = np.frexp(a)  # a = m * 2**ex with m in [0.5, 1)
    e = np.maximum(ex.astype(np.int64) - 1, -126)
    q = np.ldexp(1.0, (e - 7).astype(np.int32))
    with np.errstate(over="ignore", invalid="ignore"):
        r = np.rint(a / q) * q
        r32 = r.astype(np.float32)  # exact for finite r < 2**128; inf beyond
    bits = (r32.view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    bits = np.where(np.signbit(x), bits | np.uint16(0x8000), bits)
    bits = np.where(np.isnan(x), np.uint16(0x7FC0), bits)
    return bits.astype(np.uint16)


# --------------------------------------------------------------------------
# 2-D axial RoPE with rho-scaled low-res positions (UltraGen-ar §2.ب)
# --------------------------------------------------------------------------

def rope_frequencies(a: int, theta: float) -> list:
    """f_k = theta^(-2k/a), k = 0 .. a/2-1, each one C-library pow in fp64."""
    return [theta ** (-2.0 * k / a) for k in range(a // 2)]


def _cos_sin_table(positions: Sequence[float], freqs: Sequence[float]):
    """fp32(cos(pos*f)), fp32(sin(pos*f)); angle = one fp64 product."""
    shape = (len(positions), len(freqs))
    c = np.array([[math.cos(p * f) for f in freqs] for p in positions], dtype=np.float64)
    s = np.array([[math.sin(p * f) for f in freqs] for p in positions], dtype=np.float64)
    return c.reshape(shape).astype(np.float32), s.reshape(shape).astype(np.float32)


def rope_tables(g: Geometry) -> Dict[str, Tuple[np.ndarray, np.ndarray]]:
    """Per-axis cos/sin tables (fp32), indexed [grid coordinate][pair k].

    High-res coordinate y (or x) sits at position y; low-res coordinate i sits
    at position rho * i (one fp64 product).
    """
    fy = rope_frequencies(g.rope_dim_y, g.rope_theta)
    fx = rope_frequencies(g.rope_dim_x, g.rope_theta)
    return {
        "hr_y": _cos_sin_table([float(y) for y in range(g.grid_h)], fy),
        "hr_x": _cos_sin_table([float(x) for x in range(g.grid_w)], fx),
        "lr_y": _cos_sin_table([g.rho * float(i) for i in range(g.lr_h)], fy),
        "lr_x": _cos_sin_table([g.rho * float(j) for j in range(g.lr_w)], fx),
    }


def token_coords(g: Geometry, token_set: str, tokens: Optional[np.ndarray] = None):
    """(row, col) grid coordinates of each token of a token set.

    For the global set (LOWRES) the index counts the text tokens first; a text
    token has no grid position and gets (-1, -1).
    """
    if token_set == LOWRES:
        t = np.arange(g.L, dtype=np.int64) if tokens is None else np.asarray(tokens, np.int64)
        lr = t - g.text_len
        row, col = np.divmod(np.maximum(lr, 0), max(g.lr_w, 1))
        return np.where(lr < 0, -1, row), np.where(lr < 0, -1, col)
    t = np.arange(g.N, dtype=np.int64) if tokens is None else np.asarray(tokens, np.int64)
    if token_set == HR_WINDOW_FIRST:
        t = raster_index(g)[t]
    elif token_set != HR_RASTER:
        raise ValueError(token_set)
    return np.divmod(t, g.grid_w)


def rope_rotate_f64(x: np.ndarray, c: np.ndarray, s: np.ndarray) -> np.ndarray:
    """Rotate adjacent channel pairs: (x0, x1) -> (x0 c - x1 s, x0 s + x1 c).

    x: [..., 2m] float64; c, s broadcastable to [..., m].  With bf16 x and
    fp32 c, s every product is exact in fp64; the sum is one fp64 rounding.
    """
    x0 = x[..., 0::2]
    x1 = x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = x0 * c - x1 * s
    out[..., 1::2] = x0 * s + x1 * c
    return out


def rope_2d_f64(x64: np.ndarray, g: Geometry, token_set: str,
                tokens: Optional[np.ndarray] = None, tables=None) -> np.ndarray:
    """RoPE in fp64 before the final rounding.  x64: [B, T, h, d]."""
    tab = rope_tables(g) if tables is None else tables
    row, col = token_coords(g, token_set, tokens)
    text = row < 0  # text tokens: no position, left as they are
    out = x64.copy()
    if text.all():
        return out
    row, col, keep = row[~text], col[~text], np.nonzero(~text)[0]
    ky, kx = ("lr_y", "lr_x") if token_set == LOWRES else ("hr_y", "hr_x")
    cy, sy = tab[ky][0][row], tab[ky][1][row]  # [T, a_y/2]
    cx, sx = tab[kx][0][col], tab[kx][1][col]
    ay = g.rope_dim_y
    c64 = lambda v: v.astype(np.float64)[None, :, None, :]
    x = x64[:, keep]
    out[:, keep, :, :ay] = rope_rotate_f64(x[..., :ay], c64(cy), c64(sy))
    out[:, keep, :, ay:] = rope_rotate_f64(x[..., ay:], c64(cx), c64(sx))
    return out


def rope_2d(x_bits: np.ndarray, g: Geometry, token_set: str,
            tokens: Optional[np.ndarray] = None, tables=None) -> np.ndarray:
    """bf16 in, bf16 out (uint16 patterns).  x_bits: [B, T, h, d]; ``tokens``
    names the token index of each of the T rows (default 0..T-1)."""
    return f64_to_bf16(rope_2d_f64(bf16_to_f64(x_bits), g, token_set, tokens, tables))


# --------------------------------------------------------------------------
# Block-sparse joint attention, written as its definition: dense scores over
# the joint sequence [high-res (N); low-res (L)], -inf where not visible.
# --------------------------------------------------------------------------

def window_coords_of_tokens(g: Geometry, hr_order: str) -> Tuple[np.ndarray, np.ndarray]:
    """(window row, window col) of each high-res token in the given order."""
    y, x = token_coords(g, hr_order)
    return y // g.win_h, x // g.win_w


def visibility(g: Geometry, hr_order: str, rows: np.ndarray) -> np.ndarray:
    """Boolean [len(rows), N+L]: may query ``rows[i]`` see key j?

    Rows and keys index the joint sequence (high-res first, in ``hr_order``).
    High-res query: high-res key in a window at Chebyshev distance <= radius,
    or any global (text or low-res) key.  Global query: global keys only.
    """
    N, L = g.N, g.L
    wy, wx = window_coords_of_tokens(g, hr_order)
    rows = np.asarray(rows, dtype=np.int64)
    q_hr = rows < N
    vis = np.zeros((rows.size, N + L), dtype=bool)
    if q_hr.any():
        qi = rows[q_hr]
        near = ((np.abs(wy[qi][:, None] - wy[None, :]) <= g.radius)
                & (np.abs(wx[qi][:, None] - wx[None, :]) <= g.radius))
        vis[np.ix_(np.nonzero(q_hr)[0], np.arange(N))] = near
        vis[np.nonzero(q_hr)[0], N:] = True
    vis[np.nonzero(~q_hr)[0], N:] = True
    return vis


def attend_rows(Q: np.ndarray, K: np.ndarray, V: np.ndarray, vis: np.ndarray,
                scale: float) -> Tuple[np.ndarray, np.ndarray]:
    """Masked softmax attention for the given query rows, fp64.

    Q: [r, d]; K, V: [N+L, d]; vis: [r, N+L].  Returns (O [r, d], lse [r]) with
    s = scale * Q K^T, s = -inf where not visible, p = exp(s - max) / sum,
    O = p V, lse = log sum exp(s).
    """
    s = (Q @ K.T) * scale
    s[~vis] = -np.inf
    m = s.max(axis=1, keepdims=True)
    p = np.exp(s - m)
    l = p.sum(axis=1, keepdims=True)
    o = (p @ V) / l
    return o, (m + np.log(l))[:, 0]


def attention(q_hr, k_hr, v_hr, q_lr, k_lr, v_lr, g: Geometry, hr_order: str,
              rows: Optional[np.ndarray] = None, heads: Optional[Iterable[int]] = None,
              chunk_elems: int = 1 << 25):
    """Joint attention for every (batch, head) on bf16 inputs (uint16 patterns).

    q_hr..v_hr: [B, N, h, d] in ``hr_order``; q_lr..v_lr: [B, L, h, d].
    rows: joint-sequence query indices (default: all N+L).
    Returns O [B, len(rows), h, d] and lse [B, h, len(rows)], float64.
    """
    N, L = g.N, g.L
    rows = np.arange(N + L, dtype=np.int64) if rows is None else np.asarray(rows, np.int64)
    heads = list(range(g.heads)) if heads is None else list(heads)
    B = q_hr.shape[0]
    O = np.zeros((B, rows.size, g.heads, g.head_dim))
    LSE = np.zeros((B, g.heads, rows.size))
    step = max(1, chunk_elems // max(1, N + L))
    for b in range(B):
        for h in heads:
            Q = np.concatenate([bf16_to_f64(q_hr[b, :, h]), bf16_to_f64(q_lr[b, :, h])])
            K = np.concatenate([bf16_to_f64(k_hr[b, :, h]), bf16_to_f64(k_lr[b, :, h])])
            V = np.concatenate([bf16_to_f64(v_hr[b, :, h]), bf16_to_f64(v_lr[b, :, h])])
            for i0 in range(0, rows.size, step):
                r = rows[i0:i0 + step]
                o, lse = attend_rows(Q[r], K, V, visibility(g, hr_order, r), g.scale)
                O[b, i0:i0 + step, h] = o
                LSE[b, h, i0:i0 + step] = lse
    return O, LSE


# --------------------------------------------------------------------------
# The whole layer on raster-order inputs.  Attention is equivariant under a
# reordering of the high-res tokens (positions and windows follow each
# token), so the plain statement needs no permutation at all: rotate every
# token at its own position, attend with the geometric mask, done.
# --------------------------------------------------------------------------

def layer_forward(inp: Dict[str, np.ndarray], g: Geometry,
                  rows: Optional[np.ndarray] = None,
                  heads: Optional[Iterable[int]] = None):
    """inp: uint16 q_hr/k_hr/v_hr [B, N, h, d] (raster) and q_lr/k_lr/v_lr.

    Returns (O, lse) as ``attention`` with hr_order = raster: rows index the
    joint sequence [raster high-res; low-res].
    """
    tab = rope_tables(g)
    N, L = g.N, g.L
    rows = np.arange(N + L, dtype=np.int64) if rows is None else np.asarray(rows, np.int64)
    heads = list(range(g.heads)) if heads is None else list(heads)
    B = inp["q_hr"].shape[0]
    O = np.zeros((B, rows.size, g.heads, g.head_dim))
    LSE = np.zeros((B, g.heads, rows.size))
    for h in heads:
        sl = slice(h, h + 1)
        # Keys and values: every token; queries: only the requested rows.
        k_hr = rope_2d(inp["k_hr"][:, :, sl], g, HR_RASTER, tables=tab)
        k_lr = rope_2d(inp["k_lr"][:, :, sl], g, LOWRES, tables=tab)
        qr_hr = rows[rows < N]
        qr_lr = rows[rows >= N] - N
        q_hr = np.zeros_like(inp["q_hr"][:, :, sl])
        q_lr = np.zeros_like(inp["q_lr"][:, :, sl])
        if qr_hr.size:
            q_hr[:, qr_hr] = rope_2d(inp["q_hr"][:, qr_hr][:, :, sl], g, HR_RASTER, qr_hr, tab)
        if qr_lr.size:
            q_lr[:, qr_lr] = rope_2d(inp["q_lr"][:, qr_lr][:, :, sl], g, LOWRES, qr_lr, tab)
        g1 = dataclasses.replace(g, heads=1)
        o, lse = attention(q_hr, k_hr, inp["v_hr"][:, :, sl], q_lr, k_lr,
                           inp["v_lr"][:, :, sl], g1, HR_RASTER, rows)
        O[:, :, h] = o[:, :, 0]
        LSE[:, h] = lse[:, 0]
    return O, LSE


def visible_pairs(g: Geometry, block_rows: int = 512) -> Dict[str, int]:
    """Visible (query, key) pairs per (batch, head), counted from the mask."""
    N, L = g.N, g.L
    cnt = {"hr_hr": 0, "hr_lr": 0, "lr_lr": 0}
    for i0 in range(0, N + L, block_rows):
        r = np.arange(i0, min(N + L, i0 + block_rows))
        v = visibility(g, HR_RASTER, r)
        hr = r < N
        cnt["hr_hr"] += int(v[hr][:, :N].sum())
        cnt["hr_lr"] += int(v[hr][:, N:].sum())
        cnt["lr_lr"] += int(v[~hr][:, N:].sum())
        assert not v[~hr][:, :N].any()
    return cnt


# --------------------------------------------------------------------------
# Backward pass.  The gradients of the layer's loss with respect to q, k, v,
# given dO, the gradient with respect to its output.  The pages train LoRA
# adapters on the q/k/v projections of the low-res guidance
# (UltraGen-ar §2.ج, UltraGen-fr §2.C), which needs these gradients through
# the attention and the RoPE.  Written from the derivative of
# O = softmax(scale * Q K^T, masked) V, row by row:
#   dV = P^T dO;  dP = dO V^T;  dS = P * (dP - rowsum(P * dP));
#   dQ = scale * dS K;  dK = scale * dS^T Q.
# RoPE is a rotation per channel pair, so its backward is the transposed
# rotation: (g0, g1) -> (g0 c + g1 s, -g0 s + g1 c), with the same fp32 c, s.
# --------------------------------------------------------------------------

def _as_f64(a: np.ndarray) -> np.ndarray:
    """uint16 arrays hold bf16 patterns; float64 arrays are taken as they are."""
    return a if a.dtype == np.float64 else bf16_to_f64(a)


def attention_backward_rows(Q, K, V, dO, vis, scale):
    """One chunk of query rows, fp64.  Q, dO: [r, d]; K, V: [n, d];
    vis: [r, n].  Returns (dQ [r, d], dK part [n, d], dV part [n, d]): the
    rows' own dQ and their contributions to every key's dK and dV."""
    s = (Q @ K.T) * scale
    s[~vis] = -np.inf
    m = s.max(axis=1, keepdims=True)
    p = np.exp(s - m)
    p /= p.sum(axis=1, keepdims=True)
    dP = dO @ V.T
    D = (p * dP).sum(axis=1, keepdims=True)
    dS = p * (dP - D)
    return scale * (dS @ K), scale * (dS.T @ Q), p.T @ dO


def rows_seeing(g: Geometry, hr_order: str, keys: np.ndarray, block_rows: int = 1024):
    """Every query row (joint sequence) that sees at least one of ``keys``."""
    keys = np.asarray(keys, dtype=np.int64)
    if (keys >= g.N).any():
        return np.arange(g.N + g.L, dtype=np.int64)  # every query sees a global key
    out = []
    for i0 in range(0, g.N + g.L, block_rows):
        r = np.arange(i0, min(g.N + g.L, i0 + block_rows))
        out.append(r[visibility(g, hr_order, r)[:, keys].any(axis=1)])
    return np.concatenate(out) if out else np.zeros(0, dtype=np.int64)


def attention_backward(q_hr, k_hr, v_hr, q_lr, k_lr, v_lr, do_hr, do_lr, g: Geometry,
                       hr_order: str, rows: Optional[np.ndarray] = None,
                       keys: Optional[np.ndarray] = None,
                       heads: Optional[Iterable[int]] = None, chunk_elems: int = 1 << 24):
    """Gradients of the joint attention on bf16 inputs (uint16 patterns; fp64
    arrays are also accepted and used as they are).

    q..v and do: as ``attention`` ([B, N, h, d] high-res in ``hr_order``,
    [B, L, h, d] global).  rows: query rows whose dQ is wanted; keys: key
    rows whose dK, dV are wanted (joint-sequence indices; default all).
    Returns dQ [B, len(rows), h, d], dK and dV [B, len(keys), h, d], fp64.
    """
    N, L = g.N, g.L
    n = N + L
    rows = np.arange(n, dtype=np.int64) if rows is None else np.asarray(rows, np.int64)
    keys = np.arange(n, dtype=np.int64) if keys is None else np.asarray(keys, np.int64)
    heads = list(range(g.heads)) if heads is None else list(heads)
    need = np.union1d(rows, rows_seeing(g, hr_order, keys)) if keys.size else rows
    where_row = {int(r): i for i, r in enumerate(rows)}
    B = q_hr.shape[0]
    dQ = np.zeros((B, rows.size, g.heads, g.head_dim))
    dK = np.zeros((B, keys.size, g.heads, g.head_dim))
    dV = np.zeros((B, keys.size, g.heads, g.head_dim))
    step = max(1, chunk_elems // max(1, n))
    for b in range(B):
        for h in heads:
            joint = lambda a, c: np.concatenate([_as_f64(a[b, :, h]), _as_f64(c[b, :, h])])
            Q, K, V, dO = joint(q_hr, q_lr), joint(k_hr, k_lr), joint(v_hr, v_lr), joint(do_hr, do_lr)
            for i0 in range(0, need.size, step):
                r = need[i0:i0 + step]
                dq, dk, dv = attention_backward_rows(Q[r], K, V, dO[r],
                                                     visibility(g, hr_order, r), g.scale)
                dK[b, :, h] += dk[keys]
                dV[b, :, h] += dv[keys]
                for j, ri in enumerate(r):
                    i = where_row.get(int(ri))
                    if i is not None:
                        dQ[b, i, h] = dq[j]
    return dQ, dK, dV


def rope_2d_backward_f64(g64: np.ndarray, g: Geometry, token_set: str,
                         tokens: Optional[np.ndarray] = None, tables=None) -> np.ndarray:
    """Gradient through RoPE: each channel pair's rotation transposed, i.e.
    (g0, g1) -> (g0 c + g1 s, -g0 s + g1 c) with the forward's fp32 c, s
    (products exact in fp64, one fp64 rounding each).  Text rows pass."""
    tab = rope_tables(g) if tables is None else tables
    neg = {k: (c, -s) for k, (c, s) in tab.items()}  # R(-a) = R(a)^T: c kept, s negated
    return rope_2d_f64(g64, g, token_set, tokens, neg)


def rope_2d_backward(g_bits: np.ndarray, g: Geometry, token_set: str,
                     tokens: Optional[np.ndarray] = None, tables=None) -> np.ndarray:
    """bf16 in, bf16 out (round to nearest even), as ``rope_2d``."""
    return f64_to_bf16(rope_2d_backward_f64(bf16_to_f64(g_bits), g, token_set, tokens, tables))


def layer_backward(inp: Dict[str, np.ndarray], dout: Dict[str, np.ndarray], g: Geometry,
                   rows: Optional[np.ndarray] = None, keys: Optional[np.ndarray] = None,
                   heads: Optional[Iterable[int]] = None, exact_rope: bool = False):
    """Gradients of the whole layer on raster-order inputs.

    inp: uint16 q/k/v as ``layer_forward``; dout: uint16 do_hr [B, N, h, d]
    (raster) and do_lr [B, L, h, d].  The forward's bf16 rounding of the
    rotated q and k passes gradients unchanged.  rows: joint rows (raster
    high-res first) whose dq is wanted; keys: joint rows whose dk, dv are
    wanted.  Returns fp64 (dq, dk, dv), gradients w.r.t. the unrotated inputs.
    exact_rope: keep the rotated q and k in fp64 (no bf16 rounding), the
    layer in exact arithmetic.
    """
    tab = rope_tables(g)
    N, L = g.N, g.L
    rows = np.arange(N + L, dtype=np.int64) if rows is None else np.asarray(rows, np.int64)
    keys = np.arange(N + L, dtype=np.int64) if keys is None else np.asarray(keys, np.int64)
    heads = list(range(g.heads)) if heads is None else list(heads)
    B = inp["q_hr"].shape[0]
    dq = np.zeros((B, rows.size, g.heads, g.head_dim))
    dk = np.zeros((B, keys.size, g.heads, g.head_dim))
    dv = np.zeros((B, keys.size, g.heads, g.head_dim))
    g1 = dataclasses.replace(g, heads=1)
    for h in heads:
        sl = slice(h, h + 1)
        rot = ((lambda a, s: rope_2d_f64(bf16_to_f64(a), g, s, tables=tab)) if exact_rope
               else (lambda a, s: rope_2d(a, g, s, tables=tab)))
        q = (rot(inp["q_hr"][:, :, sl], HR_RASTER), rot(inp["q_lr"][:, :, sl], LOWRES))
        k = (rot(inp["k_hr"][:, :, sl], HR_RASTER), rot(inp["k_lr"][:, :, sl], LOWRES))
        a, kk, vv = attention_backward(q[0], k[0], inp["v_hr"][:, :, sl], q[1], k[1],
                                       inp["v_lr"][:, :, sl], dout["do_hr"][:, :, sl],
                                       dout["do_lr"][:, :, sl], g1, HR_RASTER, rows, keys)
        for src, idx, dst in ((a, rows, dq), (kk, keys, dk)):
            hr, lr = idx < N, idx >= N
            if hr.any():
                dst[:, hr, h] = rope_2d_backward_f64(src[:, hr], g, HR_RASTER, idx[hr], tab)[:, :, 0]
            if lr.any():
                dst[:, lr, h] = rope_2d_backward_f64(src[:, lr], g, LOWRES, idx[lr] - N, tab)[:, :, 0]
        dv[:, :, h] = vv[:, :, 0]
    return dq, dk, dv
