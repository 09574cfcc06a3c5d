"""GPU parity of the backward pass (attention, RoPE, whole layer) against the
fp64 oracle, called through the C ABI.

RoPE's transposed rotation and the inverse permutation are bit-exact.  The
attention gradients are held to per-element bounds derived from the kernels'
arithmetic (bf16 rounding of P and dS as tensor-core operands, of the forward
output used for D, and of every output; fp32 sums): see
``parity.bwd_error_bounds``.  Small geometries check every element; the 4K
layer checks sampled query rows and high-res keys for two heads, and for all
heads the identities sum_j dV_j = sum_i dO_i and sum_j dK_j = 0.
"""
import numpy as np
import pytest
import torch

from block_sparse_local_raster_b200 import ug, workloads
from oracle import hier_local_attn as O

from parity import (U, bits, bwd_error_bounds, f64, joint_f64, ogeom, plan, rotated_bound,
                    sample_hr_tokens, sample_lr_tokens)

pytestmark = pytest.mark.gpu
DEV = "cuda"
SMALL = list(workloads.TEST_GEOMETRIES) + ["tiny"]


def inputs(wl, seed):
    x = workloads.make_inputs(wl, seed=seed)
    x.pop("head_scale", None)
    x.update(workloads.make_grad_outputs(wl, seed=seed + 1))
    return x


def forward_backward(p, wl, d):
    has_lr = wl.n_lr > 0
    g = lambda n: d[n] if has_lr else None
    o_hr, o_lr, lse = ug.hier_local_attn_fwd(p, d["q_hr"], d["k_hr"], d["v_hr"], g("q_lr"),
                                             g("k_lr"), g("v_lr"))
    grads = ug.hier_local_attn_bwd(p, d["q_hr"], d["k_hr"], d["v_hr"], g("q_lr"), g("k_lr"),
                                   g("v_lr"), o_hr, o_lr, d["do_hr"], g("do_lr"), lse)
    torch.cuda.synchronize()
    assert p.check_error() == ug.UG_OK
    return grads


def joint_grads(grads, wl, heads=None):
    sel = (lambda t: t) if heads is None else (lambda t: t[:, :, list(heads)])
    out = []
    for i in range(3):
        hr = f64(sel(grads[i]))
        lr = f64(sel(grads[3 + i])) if grads[3 + i] is not None else hr[:, :0]
        out.append(np.concatenate([hr, lr], axis=1))
    return out


def check(got, ref, bound, what):
    """Every element within its derived bound; prints the worst ratio
    |error| / bound (the headroom actually left)."""
    err = np.abs(got - ref)
    excess = err - bound
    worst = np.unravel_index(np.argmax(excess), excess.shape)
    print(f"{what}: max |err| {err.max():.3g}, worst |err| / bound {(err / bound).max():.3f}")
    assert excess.max() <= 0, (what, float(excess.max()), float(err[worst]),
                               float(bound[worst]), worst)
    return float(err.max())


@pytest.mark.parametrize("name", SMALL)
def test_attention_backward_every_element(name):
    wl = workloads.get(name)
    g = ogeom(wl)
    p = plan(wl)
    x = inputs(wl, 800)
    grads = forward_backward(p, wl, {k: v.to(DEV) for k, v in x.items()})
    xb = {k: bits(v) for k, v in x.items()}
    ref = O.attention_backward(xb["q_hr"], xb["k_hr"], xb["v_hr"], xb["q_lr"], xb["k_lr"],
                               xb["v_lr"], xb["do_hr"], xb["do_lr"], g, O.HR_WINDOW_FIRST)
    bnd = bwd_error_bounds(g, O.HR_WINDOW_FIRST, *(joint_f64(x, n) for n in ("q", "k", "v", "do")))
    for what, got, r, b in zip(("dq", "dk", "dv"), joint_grads(grads, wl), ref, bnd):
        check(got, r, b, f"{name} {what}")


@pytest.mark.parametrize("name", ["4K", "4K-CFG", "4K-text"])
def test_attention_backward_sampled_full_size(name):
    """Full-size layers: sampled query rows (dQ) and high-res keys (dK, dV)
    of two heads against the oracle under the derived bounds, plus the
    gradient-sum identities for every head and key.  4K-CFG adds batch 2
    and per-head scales of q, k, v; 4K-text adds 512 text tokens."""
    wl = workloads.get(name)
    g = ogeom(wl)
    p = plan(wl)
    x = inputs(wl, 810)
    grads = forward_backward(p, wl, {k: v.to(DEV) for k, v in x.items()})
    heads = [0, 23]
    rows = np.concatenate([sample_hr_tokens(g, O.HR_WINDOW_FIRST, 5, n_interior=2, per_window=2),
                           g.N + sample_lr_tokens(g, 5, n=4)])
    T, nx = g.T, g.n_win_x
    mid = (g.n_win_y // 2) * nx + nx // 2
    # corner, interior and last window at 4K, the corner key with text
    # tokens; a key's dK, dV need the full rows of every query that sees it,
    # so the 1024-token windows of 4K-CFG (17k such rows) check dQ rows and
    # the identities only
    keys = (np.array([0, mid * T + min(100, T - 1), g.N - 1]) if name == "4K"
            else np.array([0]) if T <= 256 else np.zeros(0, dtype=np.int64))
    xb = {k: bits(v[:, :, heads]) for k, v in x.items()}
    g1 = O.Geometry.from_dict(dict(wl.geom_dict(), heads=len(heads)))
    ref = O.attention_backward(xb["q_hr"], xb["k_hr"], xb["v_hr"], xb["q_lr"], xb["k_lr"],
                               xb["v_lr"], xb["do_hr"], xb["do_lr"], g1, O.HR_WINDOW_FIRST,
                               rows=rows, keys=keys)
    bnd = bwd_error_bounds(g1, O.HR_WINDOW_FIRST,
                           *(joint_f64(x, n, heads) for n in ("q", "k", "v", "do")),
                           rows=rows, keys=keys)
    gq, gk, gv = joint_grads(grads, wl, heads)
    check(gq[:, rows], ref[0], bnd[0], f"{name} dq")
    if keys.size:
        check(gk[:, keys], ref[1], bnd[1], f"{name} dk")
        check(gv[:, keys], ref[2], bnd[2], f"{name} dv")
    # identities of any softmax attention, all heads, every key (sums in fp64
    # on the device)
    tot = lambda a, b_: a.double().sum(1) + b_.double().sum(1)
    mag = lambda a, b_: a.double().abs().sum(1) + b_.double().abs().sum(1)
    dk_hr, dv_hr, dk_lr, dv_lr = grads[1], grads[2], grads[4], grads[5]
    do_sum = tot(x["do_hr"].to(DEV), x["do_lr"].to(DEV))
    assert bool(((tot(dv_hr, dv_lr) - do_sum).abs() <= U * mag(dv_hr, dv_lr) + 1e-3).all())
    assert bool((tot(dk_hr, dk_lr).abs() <= 2 * U * mag(dk_hr, dk_lr) + 1e-3).all())


def test_attention_backward_8K_sampled_rows():
    """The 8K layer (262144 high-res tokens, 16384 global ones): dQ of
    sampled query rows for two heads against the oracle under the derived
    bounds, and the gradient-sum identities for every head and key.  Inputs
    are drawn on the device with the same distributions (the CPU draw of 8K
    takes minutes); the oracle reads the two heads back."""
    wl = workloads.get("8K")
    g = ogeom(wl)
    p = plan(wl)
    d = workloads.make_inputs_on_device(wl, 840, DEV)
    gen = torch.Generator(device=DEV).manual_seed(841)
    for name, n in (("do_hr", wl.n_hr), ("do_lr", wl.n_lr)):
        d[name] = torch.randn((wl.batch, n, wl.heads, wl.head_dim), generator=gen,
                              device=DEV).to(torch.bfloat16)
    grads = forward_backward(p, wl, d)
    heads = [0, 23]
    rows = np.concatenate([sample_hr_tokens(g, O.HR_WINDOW_FIRST, 9, n_interior=2, per_window=2),
                           g.N + sample_lr_tokens(g, 9, n=4)])
    none = np.zeros(0, dtype=np.int64)
    xb = {k: bits(v[:, :, heads]) for k, v in d.items()}
    g1 = O.Geometry.from_dict(dict(wl.geom_dict(), heads=len(heads)))
    ref = O.attention_backward(xb["q_hr"], xb["k_hr"], xb["v_hr"], xb["q_lr"], xb["k_lr"],
                               xb["v_lr"], xb["do_hr"], xb["do_lr"], g1, O.HR_WINDOW_FIRST,
                               rows=rows, keys=none)
    bnd = bwd_error_bounds(g1, O.HR_WINDOW_FIRST,
                           *(joint_f64(d, n, heads) for n in ("q", "k", "v", "do")),
                           rows=rows, keys=none)
    gq, _, _ = joint_grads(grads, wl, heads)
    check(gq[:, rows], ref[0], bnd[0], "8K dq")
    tot = lambda a, b_: a.double().sum(1) + b_.double().sum(1)
    mag = lambda a, b_: a.double().abs().sum(1) + b_.double().abs().sum(1)
    dk_hr, dv_hr, dk_lr, dv_lr = grads[1], grads[2], grads[4], grads[5]
    do_sum = tot(d["do_hr"], d["do_lr"])
    assert bool(((tot(dv_hr, dv_lr) - do_sum).abs() <= U * mag(dv_hr, dv_lr) + 1e-3).all())
    assert bool((tot(dk_hr, dk_lr).abs() <= 2 * U * mag(dk_hr, dk_lr) + 1e-3).all())


SETS = [(ug.UG_HR_WINDOW_FIRST, O.HR_WINDOW_FIRST), (ug.UG_HR_RASTER, O.HR_RASTER),
        (ug.UG_LR, O.LOWRES)]


@pytest.mark.parametrize("name", SMALL + ["4K"])
def test_rope_backward_bit_exact(name):
    wl = workloads.get(name)
    g = ogeom(wl)
    p = plan(wl)
    tab = O.rope_tables(g)
    for k, (uset, oset) in enumerate(SETS):
        n = wl.n_lr if uset == ug.UG_LR else wl.n_hr
        if n == 0:
            continue
        x = workloads.make_tensor((wl.batch, n, wl.heads, wl.head_dim), 900 + k)
        y = ug.rope_2d_bwd(p, x.to(DEV), uset)
        heads = range(wl.heads) if name != "4K" else [0, 13]
        xb, yb = bits(x), bits(y)
        for h in heads:
            want = O.rope_2d_backward(xb[:, :, h:h + 1], g, oset, tables=tab)
            np.testing.assert_array_equal(yb[:, :, h:h + 1], want, err_msg=f"{name} {oset} {h}")
    assert p.check_error() == ug.UG_OK


@pytest.mark.parametrize("name", SMALL + ["4K"])
def test_unpermute_rope_backward_bit_exact(name):
    wl = workloads.get(name)
    g = ogeom(wl)
    p = plan(wl)
    x = workloads.make_tensor((wl.batch, wl.n_hr, wl.heads, wl.head_dim), 950)
    y = ug.unpermute_rope_bwd(p, x.to(DEV))
    xb, yb = bits(x), bits(y)
    heads = range(wl.heads) if name != "4K" else [0, 13]
    for h in heads:
        want = O.unpermute(O.rope_2d_backward(xb[:, :, h:h + 1], g, O.HR_WINDOW_FIRST), g)
        np.testing.assert_array_equal(yb[:, :, h:h + 1], want, err_msg=f"{name} {h}")


@pytest.mark.parametrize("name", SMALL)
def test_layer_backward_every_element(name):
    """ug_layer_bwd on raster inputs against the oracle's layer gradients."""
    wl = workloads.get(name)
    g = ogeom(wl)
    p = plan(wl)
    x = inputs(wl, 820)
    d = {k: v.to(DEV) for k, v in x.items()}
    has_lr = wl.n_lr > 0
    lr = lambda n: d[n] if has_lr else None
    o_hr, o_lr, lse = ug.layer_forward(p, d["q_hr"], d["k_hr"], d["v_hr"], lr("q_lr"),
                                       lr("k_lr"), lr("v_lr"))
    grads = ug.layer_backward(p, d["q_hr"], d["k_hr"], d["v_hr"], lr("q_lr"), lr("k_lr"),
                              lr("v_lr"), o_hr, o_lr, lse, d["do_hr"], lr("do_lr"))
    torch.cuda.synchronize()
    assert p.check_error() == ug.UG_OK
    for k in d:  # inputs untouched
        assert torch.equal(d[k].cpu(), x[k]), k
    xb = {k: bits(v) for k, v in x.items()}
    ref = O.layer_backward(xb, xb, g)
    # bounds in the rotated frame (raster order), then through R^T for dq, dk
    rot = {"q": np.concatenate([O.bf16_to_f64(O.rope_2d(xb["q_hr"], g, O.HR_RASTER)),
                                O.bf16_to_f64(O.rope_2d(xb["q_lr"], g, O.LOWRES))], axis=1),
           "k": np.concatenate([O.bf16_to_f64(O.rope_2d(xb["k_hr"], g, O.HR_RASTER)),
                                O.bf16_to_f64(O.rope_2d(xb["k_lr"], g, O.LOWRES))], axis=1)}
    bq, bk, bv = bwd_error_bounds(g, O.HR_RASTER, rot["q"], rot["k"], joint_f64(x, "v"),
                                  joint_f64(x, "do"))
    got = joint_grads(grads, wl)
    check(got[0], ref[0], rotated_bound(bq, ref[0]), f"{name} layer dq")
    check(got[1], ref[1], rotated_bound(bk, ref[1]), f"{name} layer dk")
    check(got[2], ref[2], bv, f"{name} layer dv")


@pytest.mark.parametrize("name", SMALL + ["2K", "4K-CFG"])
def test_attention_backward_raster_equals_permuted_path(name):
    """ug_hier_local_attn_bwd_vo_raster (v, o, dO read and dv written in
    raster order) gives bit for bit the window-first backward's gradients,
    with dv unpermuted; geometries whose 128-row tiles are not whole window
    rows are refused."""
    wl = workloads.get(name)
    p = plan(wl)
    x = inputs(wl, 830)
    d = {k: v.to(DEV) for k, v in x.items()}
    has_lr = wl.n_lr > 0
    g = lambda n: d[n] if has_lr else None
    T = wl.win_h * wl.win_w
    supported = 128 % wl.win_w == 0 and T % 128 == 0
    o_hr, o_lr, lse = ug.hier_local_attn_fwd(p, d["q_hr"], d["k_hr"], d["v_hr"], g("q_lr"),
                                             g("k_lr"), g("v_lr"))
    ref = ug.hier_local_attn_bwd(p, d["q_hr"], d["k_hr"], d["v_hr"], g("q_lr"), g("k_lr"),
                                 g("v_lr"), o_hr, o_lr, d["do_hr"], g("do_lr"), lse)
    v_r, o_r, do_r = (ug.unpermute(p, t) for t in (d["v_hr"], o_hr, d["do_hr"]))
    like = lambda t: torch.empty_like(t) if t is not None else None
    outs = [like(t) for t in (d["q_hr"], d["k_hr"], d["v_hr"], g("q_lr"), g("k_lr"), g("v_lr"))]
    ws = torch.empty(p.attn_bwd_workspace_bytes(), dtype=torch.uint8, device=DEV)
    st = p.hier_local_attn_bwd_vo_raster(d["q_hr"], d["k_hr"], v_r, g("q_lr"), g("k_lr"),
                                         g("v_lr"), o_r, o_lr, do_r, g("do_lr"), lse, *outs, ws)
    if not supported:
        assert st == ug.UG_ERR_UNSUPPORTED
        return
    assert st == ug.UG_OK, ug.status_string(st)
    torch.cuda.synchronize()
    assert p.check_error() == ug.UG_OK
    assert torch.equal(outs[0], ref[0]) and torch.equal(outs[1], ref[1])
    assert torch.equal(outs[2], ug.unpermute(p, ref[2]))
    for a, b in zip(outs[3:], ref[3:]):
        assert (a is None and b is None) or torch.equal(a, b)


def test_backward_error_statuses():
    wl = workloads.get("tiny")
    p = plan(wl)
    x = {k: v.to(DEV) for k, v in inputs(wl, 830).items()}
    o_hr, o_lr, lse = ug.hier_local_attn_fwd(p, x["q_hr"], x["k_hr"], x["v_hr"], x["q_lr"],
                                             x["k_lr"], x["v_lr"])
    outs = [torch.empty_like(x[n]) for n in ("q_hr", "k_hr", "v_hr", "q_lr", "k_lr", "v_lr")]
    ws = torch.empty(p.attn_bwd_workspace_bytes(), dtype=torch.uint8, device=DEV)
    args = lambda **kw: [kw.get(n, v) for n, v in (
        ("q_hr", x["q_hr"]), ("k_hr", x["k_hr"]), ("v_hr", x["v_hr"]), ("q_lr", x["q_lr"]),
        ("k_lr", x["k_lr"]), ("v_lr", x["v_lr"]), ("o_hr", o_hr), ("o_lr", o_lr),
        ("do_hr", x["do_hr"]), ("do_lr", x["do_lr"]), ("lse", lse), ("dq_hr", outs[0]),
        ("dk_hr", outs[1]), ("dv_hr", outs[2]), ("dq_lr", outs[3]), ("dk_lr", outs[4]),
        ("dv_lr", outs[5]), ("ws", ws))]
    assert p.hier_local_attn_bwd(*args()) == ug.UG_OK
    assert p.hier_local_attn_bwd(*args(lse=None)) == ug.UG_ERR_INVALID_ARG
    assert p.hier_local_attn_bwd(*args(dq_hr=x["q_hr"])) == ug.UG_ERR_ALIAS
    assert p.hier_local_attn_bwd(*args(dk_hr=outs[0])) == ug.UG_ERR_ALIAS
    assert p.hier_local_attn_bwd(*args(ws=ws[:16])) == ug.UG_ERR_INVALID_ARG
    flat = torch.empty(outs[0].numel() + 8, dtype=torch.bfloat16, device=DEV)
    assert p.hier_local_attn_bwd(*args(dq_hr=flat[1:1 + outs[0].numel()].view_as(outs[0]))) \
        == ug.UG_ERR_ALIGNMENT
    assert p.rope_2d_bwd(x["q_hr"], x["q_hr"], 9) == ug.UG_ERR_INVALID_ARG
    assert p.unpermute_rope_bwd(x["q_hr"], x["q_hr"]) == ug.UG_ERR_ALIAS
    torch.cuda.synchronize()
    assert p.check_error() == ug.UG_OK
