"""Workload geometries and seeded synthetic inputs.

This module is the one piece shared by the CUDA path, the fp64 oracle and the
benchmark.  It describes shapes and draws random numbers; it holds none of the
layer's arithmetic (no permutation, rotation, masking or softmax).

The geometries stand in for the pages' FLUX workloads (UltraGen, "Il Problema"
and "Risultati": 2K/4K/8K generations, 16 px per latent token, fixed
non-overlapping windows, a low-res guidance latent whose RoPE positions are
scaled by rho = 4).  No dataset or trained weight is involved: Q, K and V are
i.i.d. normal draws, rounded once to bf16.

Draw recipe (every config): ``torch.Generator('cpu').manual_seed(seed)``, then
``randn`` in the order q_hr, k_hr, v_hr, q_lr, k_lr, v_lr, each shaped
``[batch, tokens, heads, head_dim]`` in raster token order, fp32.  The ``_lr``
tensors hold the global tokens: ``text_len`` text tokens first (drawn like the
rest; no text encoder is involved), then the low-res grid.  Configs with
``head_scale`` then draw one U[0.5, 2] factor per (tensor in q, k, v; head),
shared by the high-res and low-res parts and by every batch element, and
multiply it in fp32.  Finally every tensor is rounded to bf16 (round to nearest
even, torch's conversion).
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
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
    softmax_scale: float = 0.0  # 0 -> 1/sqrt(head_dim)
    head_scale: bool = False  # per-(tensor, head) U[0.5, 2] factor
    text_len: int = 0  # text tokens at the head of the global tensors

    @property
    def n_hr(self) -> int:
        return self.grid_h * self.grid_w

    @property
    def n_lr(self) -> int:
        """Rows of the global (``_lr``) tensors: text tokens, then low-res."""
        return self.text_len + self.lr_h * self.lr_w

    @property
    def window_tokens(self) -> int:
        return self.win_h * self.win_w

    def geom_dict(self) -> dict:
        """Plain-number geometry, the fields of the C ABI's ``ug_geom``."""
        return dict(batch=self.batch, grid_h=self.grid_h, grid_w=self.grid_w,
                    win_h=self.win_h, win_w=self.win_w, radius=self.radius,
                    lr_h=self.lr_h, lr_w=self.lr_w, rho=self.rho, heads=self.heads,
                    head_dim=self.head_dim, rope_dim_y=self.rope_dim_y,
                    rope_dim_x=self.rope_dim_x, rope_theta=self.rope_theta,
                    softmax_scale=self.softmax_scale, text_len=self.text_len)


def _wl(name, batch, grid, win, lr, heads, d, split, radius=1, rho=4.0, **kw) -> Workload:
    return Workload(name=name, batch=batch, grid_h=grid[0], grid_w=grid[1],
                    win_h=win[0], win_w=win[1], radius=radius, lr_h=lr[0], lr_w=lr[1],
                    rho=rho, heads=heads, head_dim=d, rope_dim_y=split[0],
                    rope_dim_x=split[1], **kw)


# The five benchmark geometries.
CONFIGS: Dict[str, Workload] = {
    "tiny": _wl("tiny", 1, (32, 32), (8, 8), (8, 8), 2, 64, (32, 32)),
    "2K": _wl("2K", 1, (128, 128), (16, 16), (32, 32), 24, 128, (64, 64)),
    "4K": _wl("4K", 1, (256, 256), (16, 16), (64, 64), 24, 128, (64, 64)),
    "8K": _wl("8K", 1, (512, 512), (16, 16), (128, 128), 24, 128, (64, 64)),
    "4K-CFG": _wl("4K-CFG", 2, (256, 256), (32, 32), (64, 64), 24, 128, (64, 64),
                  head_scale=True),
}

# The 4K layer with the text tokens of the joint MMDiT sequence added to the
# global set (512: the T5 prompt length of FLUX-class models).
EXTRA_CONFIGS: Dict[str, Workload] = {
    "4K-text": _wl("4K-text", 1, (256, 256), (16, 16), (64, 64), 24, 128, (64, 64),
                   text_len=512),
}

# Small geometries for element-by-element parity: several tiles, ragged tails,
# non-square grids, windows that do not divide the 128-token tile, radius 0/2,
# no low-res set, one window covering the whole grid, 1024-token windows.
TEST_GEOMETRIES: Dict[str, Workload] = {
    "multi_tile": _wl("multi_tile", 2, (64, 48), (16, 16), (12, 10), 3, 128, (64, 64)),
    "win12_d64": _wl("win12_d64", 1, (48, 36), (12, 12), (7, 5), 2, 64, (32, 32)),
    "win8_ragged": _wl("win8_ragged", 1, (40, 24), (8, 8), (5, 3), 2, 64, (32, 32)),
    "radius2": _wl("radius2", 1, (80, 64), (16, 16), (8, 8), 2, 128, (64, 64), radius=2),
    "radius0_nolr": _wl("radius0_nolr", 1, (48, 32), (16, 16), (0, 0), 2, 128, (64, 64),
                        radius=0),
    "one_window": _wl("one_window", 1, (16, 24), (16, 24), (0, 0), 2, 128, (64, 64)),
    "asym_split": _wl("asym_split", 1, (32, 64), (16, 16), (4, 8), 2, 128, (32, 96),
                      rho=8.0),
    "rho_frac": _wl("rho_frac", 1, (32, 32), (8, 8), (6, 6), 1, 64, (32, 32), rho=2.5),
    "text77": _wl("text77", 1, (48, 32), (16, 16), (6, 4), 2, 128, (64, 64), text_len=77),
    "text_only": _wl("text_only", 1, (32, 24), (8, 8), (0, 0), 2, 64, (32, 32),
                     text_len=130),
    # the 1024-token windows of 4K-CFG (8 key blocks per window, raster v/o
    # eligible) on a 3 x 2 window grid, where corner windows do not see the far row
    "win32": _wl("win32", 1, (96, 64), (32, 32), (24, 16), 2, 128, (64, 64)),
}


def get(name: str) -> Workload:
    if name in CONFIGS:
        return CONFIGS[name]
    if name in EXTRA_CONFIGS:
        return EXTRA_CONFIGS[name]
    return TEST_GEOMETRIES[name]


def make_inputs(wl: Workload, seed: int = 0,
                device: Optional[str] = None) -> Dict[str, torch.Tensor]:
    """Seeded bf16 q/k/v for the high-res grid (raster order) and low-res grid.

    Returns a dict with keys q_hr, k_hr, v_hr ([B, N, h, d]) and q_lr, k_lr,
    v_lr ([B, L, h, d]); all bf16, contiguous, on the CPU unless ``device``.
    Configs with ``head_scale`` add "head_scale", the fp32 [3, heads] factors.
    """
    g = torch.Generator(device="cpu").manual_seed(seed)
    shp_hr = (wl.batch, wl.n_hr, wl.heads, wl.head_dim)
    shp_lr = (wl.batch, wl.n_lr, wl.heads, wl.head_dim)
    names = (("q_hr", shp_hr), ("k_hr", shp_hr), ("v_hr", shp_hr),
             ("q_lr", shp_lr), ("k_lr", shp_lr), ("v_lr", shp_lr))
    out: Dict[str, torch.Tensor] = {}
    raw = {}
    for name, shp in names:
        t = torch.randn(shp, generator=g, dtype=torch.float32)
        if wl.head_scale:
            raw[name] = t  # the factors are drawn after every normal
        else:
            out[name] = t.to(torch.bfloat16).contiguous()
            del t
    if wl.head_scale:
        s = torch.empty((3, wl.heads), dtype=torch.float32).uniform_(0.5, 2.0, generator=g)
        for name, _ in names:
            row = "qkv".index(name[0])
            t = raw.pop(name)
            t.mul_(s[row].view(1, 1, wl.heads, 1))
            out[name] = t.to(torch.bfloat16).contiguous()
            del t
        out["head_scale"] = s
    if device is not None:
        for name in list(out):
            out[name] = out[name].to(device)
    return out


def make_inputs_on_device(wl: Workload, seed: int, device) -> Dict[str, torch.Tensor]:
    """The same distributions as make_inputs, drawn on the device by a seeded
    CUDA generator (a different random stream, so different values): for
    timing runs at sizes where the CPU draw takes minutes (8K: 805 M normals
    per tensor).  Parity tests use make_inputs."""
    g = torch.Generator(device=device).manual_seed(seed)
    shp_hr = (wl.batch, wl.n_hr, wl.heads, wl.head_dim)
    shp_lr = (wl.batch, wl.n_lr, wl.heads, wl.head_dim)
    out: Dict[str, torch.Tensor] = {}
    s = None
    if wl.head_scale:
        s = torch.empty((3, wl.heads), dtype=torch.float32, device=device).uniform_(
            0.5, 2.0, generator=g)
    for name, shp in (("q_hr", shp_hr), ("k_hr", shp_hr), ("v_hr", shp_hr),
                      ("q_lr", shp_lr), ("k_lr", shp_lr), ("v_lr", shp_lr)):
        t = torch.randn(shp, generator=g, dtype=torch.float32, device=device)
        if s is not None:
            t.mul_(s["qkv".index(name[0])].view(1, 1, wl.heads, 1))
        out[name] = t.to(torch.bfloat16).contiguous()
        del t
    if s is not None:
        out["head_scale"] = s
    return out


def make_grad_outputs(wl: Workload, seed: int = 1,
                      device: Optional[str] = None) -> Dict[str, torch.Tensor]:
    """Seeded output gradients for the backward pass: do_hr [B, N, h, d] and
    do_lr [B, L, h, d], i.i.d. N(0, 1) drawn in that order, rounded to bf16."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    out = {}
    for name, n in (("do_hr", wl.n_hr), ("do_lr", wl.n_lr)):
        t = torch.randn((wl.batch, n, wl.heads, wl.head_dim), generator=g, dtype=torch.float32)
        out[name] = t.to(torch.bfloat16).contiguous()
    if device is not None:
        out = {k: v.to(device) for k, v in out.items()}
    return out


def make_tensor(shape, seed: int, scale: float = 1.0) -> torch.Tensor:
    """One seeded N(0, scale^2) bf16 tensor (CPU), for single-kernel tests."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    t = torch.randn(tuple(shape), generator=g, dtype=torch.float32)
    if scale != 1.0:
        t.mul_(scale)
    return t.to(torch.bfloat16).contiguous()


# Warm-start initialisation: FLUX-class latents have 16 channels at 1/8 of
# the image size (two latent pixels per token side), so the 4K image is a
# 16 x 512 x 512 latent and its low-res guidance (the 64 x 64 token grid) a
# 16 x 128 x 128 one: factor 4 = rho.  The sharpening amount and the timestep
# are not given on the pages; 0.5 and 0.6 stand in.
@dataclasses.dataclass(frozen=True)
class WarmStart:
    name: str
    batch: int
    channels: int
    lr_h: int
    lr_w: int
    scale: int
    sharpen: float = 0.5
    t: float = 0.6

    @property
    def hr_shape(self):
        return (self.batch, self.channels, self.lr_h * self.scale, self.lr_w * self.scale)

    @property
    def lr_shape(self):
        return (self.batch, self.channels, self.lr_h, self.lr_w)


WARM_START: Dict[str, WarmStart] = {
    "4K": WarmStart("4K", 1, 16, 128, 128, 4),
    "8K": WarmStart("8K", 1, 16, 256, 256, 4),
    "odd": WarmStart("odd", 2, 3, 13, 7, 3, sharpen=1.25, t=0.3),
    "s1": WarmStart("s1", 1, 2, 9, 20, 1),
    "wide": WarmStart("wide", 1, 1, 3, 70, 4, sharpen=0.0, t=0.0),
    # factor 4 with every border case: odd sizes, a one-pixel-wide plane
    "s4_edges": WarmStart("s4_edges", 2, 3, 5, 9, 4, sharpen=0.8, t=0.45),
    "s4_thin": WarmStart("s4_thin", 1, 2, 1, 1, 4, sharpen=0.5, t=0.6),
}


def make_warm_start_inputs(ws: WarmStart, seed: int = 0) -> Dict[str, torch.Tensor]:
    """x_lr then noise, i.i.d. N(0, 1) fp32 from one seeded CPU generator."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    x_lr = torch.randn(ws.lr_shape, generator=g, dtype=torch.float32)
    noise = torch.randn(ws.hr_shape, generator=g, dtype=torch.float32)
    return {"x_lr": x_lr, "noise": noise}
