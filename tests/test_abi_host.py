"""Host-side checks of the C-ABI library (no GPU needed)."""
import os
import re

import numpy as np
import pytest

from block_sparse_local_raster_b200 import ug, workloads
from oracle import hier_local_attn as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    names = set()
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            src = open(os.path.join(ROOT, "include", f)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(ug_[a-z0-9_]+)\s*\(", src))
    return names


def test_library_exports_every_declared_symbol():
    L = ug.lib()
    decl = declared_symbols()
    assert decl, "no declarations found"
    assert decl == set(ug.EXPORTS)
    for name in decl:
        assert hasattr(L, name), name


def g_of(wl, **over):
    d = wl.geom_dict()
    d.update(over)
    return ug.make_geom(**d)


ALL = (list(workloads.CONFIGS.values()) + list(workloads.EXTRA_CONFIGS.values())
       + list(workloads.TEST_GEOMETRIES.values()))


@pytest.mark.parametrize("wl", ALL, ids=lambda w: w.name)
def test_index_maps_match_oracle(wl):
    perm, off, idx = ug.build_index_maps(g_of(wl))
    og = O.Geometry.from_dict(wl.geom_dict())
    np.testing.assert_array_equal(perm, O.window_first_index(og))
    ooff, oidx = O.window_neighbours(og)
    np.testing.assert_array_equal(off, ooff)
    np.testing.assert_array_equal(idx, oidx)


@pytest.mark.parametrize("wl", ALL, ids=lambda w: w.name)
def test_visible_pairs_match_oracle_count(wl):
    got = ug.visible_pairs(g_of(wl))
    og = O.Geometry.from_dict(wl.geom_dict())
    if og.N + og.L <= 20000:
        c = O.visible_pairs(og)
        assert got == (c["hr_hr"], c["hr_lr"], c["lr_lr"])
    # closed form for radius-1 windows clipped at the border
    span = lambda n, r: sum(min(n, w + r + 1) - max(0, w - r) for w in range(n))
    T = wl.win_h * wl.win_w
    assert got[0] == T * T * span(wl.grid_h // wl.win_h, wl.radius) * span(wl.grid_w // wl.win_w, wl.radius)
    assert got[1] == wl.n_hr * wl.n_lr and got[2] == wl.n_lr ** 2


def test_useful_flops_of_the_benchmark_configs():
    """4 * d * visible pairs * heads * batch for the five configs, from the
    closed form T^2 (3n - 2)^2 + N L + L^2 pairs per head (n windows a side)."""
    want = {"tiny": 245_366_784, "2K": 608_811_614_208, "4K": 5_208_721_588_224,
            "8K": 63_190_780_084_224, "4K-CFG": 19_481_971_654_656}
    for name, wl in workloads.CONFIGS.items():
        pairs = sum(ug.visible_pairs(g_of(wl)))
        assert 4 * wl.head_dim * pairs * wl.heads * wl.batch == want[name], name


def test_useful_flops_with_text_tokens():
    """4K with 512 text tokens: G = 512 + 64^2 = 4608 global tokens, so
    256^2 * 14^2 ... = 138,674,176 + 65,536 * 4608 + 4608^2 pairs per head."""
    wl = workloads.EXTRA_CONFIGS["4K-text"]
    assert ug.visible_pairs(g_of(wl)) == (138_674_176, 301_989_888, 21_233_664)


@pytest.mark.parametrize("over,status", [
    (dict(win_h=7), ug.UG_ERR_INVALID_ARG),            # windows must tile the grid
    (dict(grid_w=0), ug.UG_ERR_INVALID_ARG),
    (dict(batch=0), ug.UG_ERR_INVALID_ARG),
    (dict(radius=-1), ug.UG_ERR_INVALID_ARG),
    (dict(lr_h=0), ug.UG_ERR_INVALID_ARG),              # 0 x 8 low-res grid
    (dict(rho=0.0), ug.UG_ERR_INVALID_ARG),
    (dict(rope_theta=1.0), ug.UG_ERR_INVALID_ARG),
    (dict(rope_dim_y=20, rope_dim_x=44), ug.UG_ERR_INVALID_ARG),  # segment not a multiple of 8
    (dict(rope_dim_y=32, rope_dim_x=64), ug.UG_ERR_INVALID_ARG),  # split != head_dim
    (dict(heads=1 << 20), ug.UG_ERR_INVALID_ARG),       # element count past 2^31
    (dict(), ug.UG_OK),
    (dict(lr_h=0, lr_w=0), ug.UG_OK),
    (dict(text_len=-1), ug.UG_ERR_INVALID_ARG),
    (dict(text_len=77), ug.UG_OK),
    (dict(lr_h=0, lr_w=0, text_len=5), ug.UG_OK),      # text as the only global tokens
])
def test_geometry_validation(over, status):
    assert ug.geom_validate(g_of(workloads.CONFIGS["tiny"], **over)) == status


def test_status_strings():
    for s in range(8):
        assert ug.status_string(s)
    assert ug.status_string(ug.UG_ERR_TIMEOUT) == "device-side wait timed out"
