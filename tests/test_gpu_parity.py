"""GPU parity: the CUDA library, called through its C ABI, against the oracle.

Index and data-movement work (permute, unpermute, RoPE) must match bit for
bit; attention within max-abs 1e-2 and mean-abs 1e-3 of the fp64 oracle on
unit-variance inputs (per-head value scale divided out for the scaled CFG
config).  Small geometries compare every row; the benchmark geometries
compare stratified row samples (corner, edge and interior windows, low-res
rows) for every head.
"""
import numpy as np
import pytest
import torch

from block_sparse_local_raster_b200 import ug, workloads
from oracle import hier_local_attn as O

from parity import (LSE_ABS, MAX_ABS, MEAN_ABS, bits, err_stats, f64, ogeom, plan,
                    sample_hr_tokens, sample_lr_tokens)

pytestmark = pytest.mark.gpu

DEV = "cuda"
SMALL = list(workloads.TEST_GEOMETRIES) + ["tiny"]
BIG = ["2K", "4K", "8K", "4K-CFG", "4K-text"]


def rand(shape, seed):
    return workloads.make_tensor(shape, seed)


# ----------------------------------------------------------------- permutation

@pytest.mark.parametrize("name", SMALL + BIG)
def test_permute_and_unpermute_bit_exact(name):
    wl = workloads.get(name)
    g = ogeom(wl)
    p = plan(wl)
    x = rand((wl.batch, wl.n_hr, wl.heads, wl.head_dim), 100)
    xd = x.to(DEV)
    y = ug.permute_window_first(p, xd)
    z = ug.unpermute(p, y)
    torch.cuda.synchronize()
    assert p.check_error() == ug.UG_OK
    xb = bits(x)
    np.testing.assert_array_equal(bits(y), O.permute_window_first(xb, g))
    np.testing.assert_array_equal(bits(z), xb)
    np.testing.assert_array_equal(bits(ug.unpermute(p, xd)), O.unpermute(xb, g))


def test_index_maps_of_plan_match_oracle():
    for name in SMALL + ["2K"]:
        wl = workloads.get(name)
        perm, off, idx = plan(wl).index_maps()
        g = ogeom(wl)
        np.testing.assert_array_equal(perm, O.window_first_index(g))
        o_off, o_idx = O.window_neighbours(g)
        np.testing.assert_array_equal(off, o_off)
        np.testing.assert_array_equal(idx, o_idx)


# ----------------------------------------------------------------- RoPE

SETS = [(ug.UG_HR_WINDOW_FIRST, O.HR_WINDOW_FIRST), (ug.UG_HR_RASTER, O.HR_RASTER),
        (ug.UG_LR, O.LOWRES)]


@pytest.mark.parametrize("name", SMALL + BIG)
def test_rope_bit_exact(name):
    wl = workloads.get(name)
    g = ogeom(wl)
    p = plan(wl)
    tab = O.rope_tables(g)
    heads = list(range(wl.heads)) if name != "8K" else [0, 11, 23]
    for k, (uset, oset) in enumerate(SETS):
        n = wl.n_lr if uset == ug.UG_LR else wl.n_hr
        if n == 0:
            continue
        x = rand((wl.batch, n, wl.heads, wl.head_dim), 200 + k)
        xd = x.to(DEV)
        y = ug.rope_2d(p, xd, uset)
        yb = bits(y)
        xb = bits(x)
        for h in heads:
            want = O.rope_2d(xb[:, :, h:h + 1], g, oset, tables=tab)
            np.testing.assert_array_equal(yb[:, :, h:h + 1], want, err_msg=f"{name} set {oset} head {h}")
        if name in SMALL:  # in place gives the same bits
            ug.rope_2d(p, xd, uset, inplace=True)
            np.testing.assert_array_equal(bits(xd), yb)
    assert p.check_error() == ug.UG_OK


@pytest.mark.parametrize("name", SMALL + BIG)
def test_permute_rope_fused_bit_exact(name):
    """Window-first permute with RoPE in the same pass equals the oracle's
    rotation at window-first positions of the permuted tensor."""
    wl = workloads.get(name)
    g = ogeom(wl)
    p = plan(wl)
    tab = O.rope_tables(g)
    x = rand((wl.batch, wl.n_hr, wl.heads, wl.head_dim), 250)
    y = ug.permute_rope_window_first(p, x.to(DEV))
    torch.cuda.synchronize()
    assert p.check_error() == ug.UG_OK
    yb, xb = bits(y), bits(x)
    heads = list(range(wl.heads)) if name != "8K" else [0, 11, 23]
    for h in heads:
        want = O.rope_2d(O.permute_window_first(xb[:, :, h:h + 1], g), g, O.HR_WINDOW_FIRST,
                         tables=tab)
        np.testing.assert_array_equal(yb[:, :, h:h + 1], want, err_msg=f"{name} head {h}")


# ----------------------------------------------------------------- attention alone

def attn_inputs(wl, seed):
    """Random window-first high-res and low-res q/k/v (no RoPE needed)."""
    x = workloads.make_inputs(wl, seed=seed)
    return x


def run_attn(p, x):
    d = {k: v.to(DEV) for k, v in x.items() if k != "head_scale"}
    has_lr = d["q_lr"].shape[1] > 0
    o_hr, o_lr, lse = ug.hier_local_attn_fwd(
        p, d["q_hr"], d["k_hr"], d["v_hr"], d["q_lr"] if has_lr else None,
        d["k_lr"] if has_lr else None, d["v_lr"] if has_lr else None)
    torch.cuda.synchronize()
    assert p.check_error() == ug.UG_OK
    return o_hr, o_lr, lse


def check_rows(wl, g, o_hr, o_lr, lse, ref_o, ref_lse, rows, vscale=None):
    N = g.N
    hr = rows[rows < N]
    lr = rows[rows >= N] - N
    got = np.concatenate([f64(o_hr[:, torch.from_numpy(hr)]),
                          f64(o_lr[:, torch.from_numpy(lr)]) if lr.size else
                          np.zeros((wl.batch, 0, wl.heads, wl.head_dim))], axis=1)
    mx, mean, raw, raw_lim = err_stats(got, ref_o, vscale)
    print(f"max-abs {mx:.3g} (raw {raw:.3g}, raw bound {raw_lim:.3g}), mean-abs {mean:.3g}")
    assert mx <= MAX_ABS and mean <= MEAN_ABS, (mx, mean)
    assert raw <= raw_lim, (raw, raw_lim)
    lse_got = lse.cpu().numpy()[:, :, np.concatenate([hr, N + lr])]
    assert np.abs(lse_got - ref_lse).max() <= LSE_ABS, np.abs(lse_got - ref_lse).max()
    return mx, mean


@pytest.mark.parametrize("name", SMALL)
def test_attention_every_row_small(name):
    wl = workloads.get(name)
    g = ogeom(wl)
    p = plan(wl)
    x = attn_inputs(wl, 300)
    o_hr, o_lr, lse = run_attn(p, x)
    xb = {k: bits(v) for k, v in x.items() if k != "head_scale"}
    ref_o, ref_lse = O.attention(xb["q_hr"], xb["k_hr"], xb["v_hr"], xb["q_lr"], xb["k_lr"],
                                 xb["v_lr"], g, O.HR_WINDOW_FIRST)
    rows = np.arange(g.N + g.L)
    check_rows(wl, g, o_hr, o_lr, lse, ref_o, ref_lse, rows)


@pytest.mark.parametrize("name", BIG)
def test_attention_sampled_rows(name):
    wl = workloads.get(name)
    g = ogeom(wl)
    p = plan(wl)
    x = attn_inputs(wl, 400)
    o_hr, o_lr, lse = run_attn(p, x)
    rows = np.concatenate([sample_hr_tokens(g, O.HR_WINDOW_FIRST, 1),
                           g.N + sample_lr_tokens(g, 1)])
    xb = {k: bits(v) for k, v in x.items() if k != "head_scale"}
    ref_o, ref_lse = O.attention(xb["q_hr"], xb["k_hr"], xb["v_hr"], xb["q_lr"], xb["k_lr"],
                                 xb["v_lr"], g, O.HR_WINDOW_FIRST, rows)
    vs = x["head_scale"][2].numpy() if "head_scale" in x else None
    check_rows(wl, g, o_hr, o_lr, lse, ref_o, ref_lse, rows, vs)


@pytest.mark.parametrize("name", SMALL + BIG)
def test_attention_raster_v_and_o_equal_the_permuted_path(name):
    """ug_hier_local_attn_fwd_vo_raster (v read, o written in raster order)
    gives bit for bit the window-first attention's output, unpermuted, and
    the same lse; geometries whose 128-key tiles are not whole window rows
    are refused."""
    wl = workloads.get(name)
    p = plan(wl)
    x = attn_inputs(wl, 320)
    d = {k: v.to(DEV) for k, v in x.items() if k != "head_scale"}
    has_lr = wl.n_lr > 0
    lr = lambda n: d[n] if has_lr else None
    T = wl.win_h * wl.win_w
    supported = 128 % wl.win_w == 0 and T % 128 == 0
    o_r = torch.empty_like(d["q_hr"])
    o_lr = torch.empty_like(d["q_lr"]) if has_lr else None
    lse = torch.empty((wl.batch, wl.heads, wl.n_hr + wl.n_lr), dtype=torch.float32, device=DEV)
    v_raster = ug.unpermute(p, d["v_hr"])  # the same values in raster order
    st = p.hier_local_attn_fwd_vo_raster(d["q_hr"], d["k_hr"], v_raster, lr("q_lr"), lr("k_lr"),
                                         lr("v_lr"), o_r, o_lr, lse)
    if not supported:
        assert st == ug.UG_ERR_UNSUPPORTED
        return
    assert st == ug.UG_OK
    o_hr, o_lr2, lse2 = run_attn(p, x)
    torch.cuda.synchronize()
    assert p.check_error() == ug.UG_OK
    assert torch.equal(o_r, ug.unpermute(p, o_hr))
    assert torch.equal(lse, lse2)
    if has_lr:
        assert torch.equal(o_lr, o_lr2)


# ----------------------------------------------------------------- whole layer

@pytest.mark.parametrize("name", SMALL + BIG)
def test_layer_end_to_end(name):
    wl = workloads.get(name)
    g = ogeom(wl)
    p = plan(wl)
    x = workloads.make_inputs(wl, seed=0)
    d = {k: v.to(DEV) for k, v in x.items() if k != "head_scale"}
    has_lr = wl.n_lr > 0
    lr = (d["q_lr"], d["k_lr"], d["v_lr"]) if has_lr else (None, None, None)
    o_hr, o_lr, lse = ug.layer_forward(p, d["q_hr"], d["k_hr"], d["v_hr"], *lr)
    torch.cuda.synchronize()
    assert p.check_error() == ug.UG_OK
    # inputs untouched
    for k in d:
        assert torch.equal(d[k].cpu(), x[k]), k
    if name in SMALL:
        rows = np.arange(g.N + g.L)
    else:
        rows = np.concatenate([sample_hr_tokens(g, O.HR_RASTER, 2), g.N + sample_lr_tokens(g, 2)])
    xb = {k: bits(v) for k, v in x.items() if k != "head_scale"}
    ref_o, ref_lse = O.layer_forward(xb, g, rows)
    # the layer's lse keeps high-res rows in window-first order
    perm = O.window_first_index(g)
    lse_rows = np.where(rows < g.N, perm[np.minimum(rows, g.N - 1)], rows)
    N = g.N
    hr = rows[rows < N]
    lrr = rows[rows >= N] - N
    got = np.concatenate([f64(o_hr[:, torch.from_numpy(hr)]),
                          f64(o_lr[:, torch.from_numpy(lrr)]) if lrr.size else
                          np.zeros((wl.batch, 0, wl.heads, wl.head_dim))], axis=1)
    vs = x["head_scale"][2].numpy() if "head_scale" in x else None
    mx, mean, raw, raw_lim = err_stats(got, ref_o, vs)
    print(f"max-abs {mx:.3g} (raw {raw:.3g}, raw bound {raw_lim:.3g}), mean-abs {mean:.3g}")
    assert mx <= MAX_ABS and mean <= MEAN_ABS, (mx, mean)
    assert raw <= raw_lim, (raw, raw_lim)
    lse_got = lse.cpu().numpy()[:, :, lse_rows]
    assert np.abs(lse_got - ref_lse).max() <= LSE_ABS


# ----------------------------------------------------------------- invariants

def test_window_output_ignores_keys_outside_its_neighbourhood():
    """Changing high-res K/V outside N(w) leaves window w's output
    bit-identical; changing any high-res input leaves low-res outputs
    bit-identical."""
    wl = workloads.get("2K")
    g = ogeom(wl)
    p = plan(wl)
    x = attn_inputs(wl, 500)
    o_hr, o_lr, _ = run_attn(p, x)
    off, idx = O.window_neighbours(g)
    w = 9  # interior window (1, 1) of the 8 x 8 window grid
    near = set(idx[off[w]:off[w + 1]].tolist())
    far = [v for v in range(g.n_win_y * g.n_win_x) if v not in near]
    y = dict(x)
    for k in ("k_hr", "v_hr", "q_hr"):
        t = y[k].clone()
        for v in far:
            t[:, v * g.T:(v + 1) * g.T] = -t[:, v * g.T:(v + 1) * g.T]
        y[k] = t
    o2_hr, o2_lr, _ = run_attn(p, y)
    s = slice(w * g.T, (w + 1) * g.T)
    assert torch.equal(o_hr[:, s], o2_hr[:, s])
    assert torch.equal(o_lr, o2_lr)


def test_global_rows_ignore_high_res_inputs():
    """Text and low-res queries see only the global set: replacing every
    high-res q/k/v leaves their outputs bit-identical, and changing the text
    keys changes the high-res outputs (every query sees the text tokens)."""
    wl = workloads.get("text77")
    p = plan(wl)
    x = attn_inputs(wl, 510)
    o_hr, o_lr, _ = run_attn(p, x)
    y = dict(x)
    for k in ("q_hr", "k_hr", "v_hr"):
        y[k] = -x[k]
    _, o2_lr, _ = run_attn(p, y)
    assert torch.equal(o_lr, o2_lr)
    z = dict(x)
    z["v_lr"] = x["v_lr"].clone()
    z["v_lr"][:, :wl.text_len] = 4.0
    o3_hr, _, _ = run_attn(p, z)
    assert ((o3_hr.float() - o_hr.float()).abs() > 0).float().mean() > 0.99


def test_constant_values_give_constant_output():
    wl = workloads.get("multi_tile")
    p = plan(wl)
    x = attn_inputs(wl, 600)
    x["v_hr"] = torch.full_like(x["v_hr"], 0.375)
    x["v_lr"] = torch.full_like(x["v_lr"], 0.375)
    o_hr, o_lr, _ = run_attn(p, x)
    assert torch.all(o_hr.float() == 0.375) and torch.all(o_lr.float() == 0.375)


# ----------------------------------------------------------------- error paths

def test_error_statuses_on_device_pointers():
    wl = workloads.get("tiny")
    p = plan(wl)
    x = rand((1, wl.n_hr, wl.heads, wl.head_dim), 700).to(DEV)
    out = torch.empty_like(x)
    flat = torch.empty(x.numel() + 8, dtype=torch.bfloat16, device=DEV)
    mis = flat[1:1 + x.numel()].view_as(x)  # 2-byte offset
    assert p.permute_window_first(mis, out) == ug.UG_ERR_ALIGNMENT
    assert p.permute_window_first(x, x) == ug.UG_ERR_ALIAS
    assert p.permute_rope_window_first(x, x) == ug.UG_ERR_ALIAS
    assert p.permute_rope_window_first(mis, out) == ug.UG_ERR_ALIGNMENT
    assert p.unpermute(x, x) == ug.UG_ERR_ALIAS
    assert p.rope_2d(x, x, 7) == ug.UG_ERR_INVALID_ARG
    assert p.rope_2d(x, x, ug.UG_HR_RASTER) == ug.UG_OK  # exact in place is allowed
    lr = rand((1, wl.n_lr, wl.heads, wl.head_dim), 701).to(DEV)
    o_lr = torch.empty_like(lr)
    assert p.hier_local_attn_fwd(x, x, x, lr, lr, lr, x, o_lr) == ug.UG_ERR_ALIAS
    assert p.hier_local_attn_fwd(x, x, x, lr, lr, lr, out, None) == ug.UG_ERR_INVALID_ARG
    d96 = ug.Plan(**dict(wl.geom_dict(), head_dim=96, rope_dim_y=48, rope_dim_x=48))
    x96 = torch.zeros((1, wl.n_hr, wl.heads, 96), dtype=torch.bfloat16, device=DEV)
    l96 = torch.zeros((1, wl.n_lr, wl.heads, 96), dtype=torch.bfloat16, device=DEV)
    assert d96.hier_local_attn_fwd(x96, x96, x96, l96, l96, l96, torch.empty_like(x96),
                                   torch.empty_like(l96)) == ug.UG_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert p.check_error() == ug.UG_OK
