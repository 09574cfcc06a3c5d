"""Pins for the oracle's backward pass (attention, RoPE, whole layer).

Central finite differences of the oracle's own forward (pinned elsewhere) in
fp64, torch's fp64 autograd through its scaled_dot_product_attention with an
enumerated mask, the adjoint identity of the rotation, and invariants that
hold for any softmax attention: the dK rows sum to zero and the dV rows sum
to the dO rows.
"""
import dataclasses

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import hier_local_attn as O


def geom(H=8, W=8, wh=4, ww=4, r=0, lr=(2, 2), text=1, heads=1, d=8, rho=4.0):
    return O.Geometry(batch=1, grid_h=H, grid_w=W, win_h=wh, win_w=ww, radius=r,
                      lr_h=lr[0], lr_w=lr[1], rho=rho, heads=heads, head_dim=d,
                      rope_dim_y=d // 2, rope_dim_x=d // 2, text_len=text)


def bf(rng, shape, scale=1.0):
    return O.f64_to_bf16(scale * rng.standard_normal(shape))


def inputs(g, seed):
    rng = np.random.default_rng(seed)
    s = lambda n: (1, n, g.heads, g.head_dim)
    x = {k: bf(rng, s(g.N)) for k in ("q_hr", "k_hr", "v_hr", "do_hr")}
    x.update({k: bf(rng, s(g.L)) for k in ("q_lr", "k_lr", "v_lr", "do_lr")})
    return x


def joint64(x, name):
    return np.concatenate([O.bf16_to_f64(x[name + "_hr"][0, :, 0]),
                           O.bf16_to_f64(x[name + "_lr"][0, :, 0])])


def loss_f64(g, Q, K, V, W, order):
    vis = O.visibility(g, order, np.arange(g.N + g.L))
    o, _ = O.attend_rows(Q, K, V, vis, g.scale)
    return float((o * W).sum())


@pytest.mark.parametrize("order", [O.HR_WINDOW_FIRST, O.HR_RASTER])
def test_attention_gradients_match_central_differences(order):
    g = geom(r=0, text=1)
    x = inputs(g, 1)
    dQ, dK, dV = O.attention_backward(x["q_hr"], x["k_hr"], x["v_hr"], x["q_lr"], x["k_lr"],
                                      x["v_lr"], x["do_hr"], x["do_lr"], g, order)
    Q, K, V, W = (joint64(x, n) for n in ("q", "k", "v", "do"))
    h = 1e-6
    rng = np.random.default_rng(2)
    for name, grad in (("Q", dQ), ("K", dK), ("V", dV)):
        for _ in range(25):
            i, c = rng.integers(0, g.N + g.L), rng.integers(0, g.head_dim)
            args = {"Q": Q.copy(), "K": K.copy(), "V": V.copy()}
            args[name][i, c] += h
            up = loss_f64(g, args["Q"], args["K"], args["V"], W, order)
            args[name][i, c] -= 2 * h
            dn = loss_f64(g, args["Q"], args["K"], args["V"], W, order)
            assert abs((up - dn) / (2 * h) - grad[0, i, 0, c]) < 1e-7, (name, i, c)


def test_attention_gradients_match_torch_autograd():
    """A larger case (several windows, radius 1, text and low-res tokens)
    against autograd through torch's attention with the oracle's mask
    rebuilt by enumerating grid cells."""
    g = geom(H=16, W=12, wh=4, ww=4, r=1, lr=(3, 2), text=3, heads=2, d=16)
    x = inputs(g, 3)
    dQ, dK, dV = O.attention_backward(x["q_hr"], x["k_hr"], x["v_hr"], x["q_lr"], x["k_lr"],
                                      x["v_lr"], x["do_hr"], x["do_lr"], g, O.HR_RASTER)
    n = g.N + g.L
    mask = torch.zeros((n, n), dtype=torch.bool)
    for i in range(n):
        for j in range(n):
            if i >= g.N:
                mask[i, j] = j >= g.N
            elif j >= g.N:
                mask[i, j] = True
            else:
                (yi, xi), (yj, xj) = divmod(i, g.grid_w), divmod(j, g.grid_w)
                mask[i, j] = (abs(yi // g.win_h - yj // g.win_h) <= g.radius
                              and abs(xi // g.win_w - xj // g.win_w) <= g.radius)
    for h in range(g.heads):
        t = lambda nm: torch.from_numpy(np.concatenate(
            [O.bf16_to_f64(x[nm + "_hr"][0, :, h]), O.bf16_to_f64(x[nm + "_lr"][0, :, h])]))
        q, k, v = (t(nm).requires_grad_() for nm in ("q", "k", "v"))
        o = F.scaled_dot_product_attention(q[None], k[None], v[None], attn_mask=mask[None],
                                           scale=g.scale)[0]
        o.backward(t("do"))
        for mine, ref in ((dQ, q.grad), (dK, k.grad), (dV, v.grad)):
            np.testing.assert_allclose(mine[0, :, h], ref.numpy(), rtol=0, atol=1e-12)


def test_gradient_sums():
    """Every softmax row sums to one and its dS row to zero, so summed over
    keys dV equals dO summed over queries and dK sums to zero."""
    g = geom(H=12, W=8, wh=4, ww=4, r=1, lr=(2, 3), text=2, heads=2, d=16)
    x = inputs(g, 4)
    _, dK, dV = O.attention_backward(x["q_hr"], x["k_hr"], x["v_hr"], x["q_lr"], x["k_lr"],
                                     x["v_lr"], x["do_hr"], x["do_lr"], g, O.HR_WINDOW_FIRST)
    do = np.concatenate([O.bf16_to_f64(x["do_hr"]), O.bf16_to_f64(x["do_lr"])], axis=1)
    np.testing.assert_allclose(dV.sum(axis=1), do.sum(axis=1), rtol=0, atol=1e-11)
    np.testing.assert_allclose(dK.sum(axis=1), 0.0, rtol=0, atol=1e-11)


def test_row_and_key_subsets_match_the_full_backward():
    g = geom(H=16, W=16, wh=4, ww=4, r=1, lr=(2, 2), text=1, heads=1, d=8)
    x = inputs(g, 5)
    args = (x["q_hr"], x["k_hr"], x["v_hr"], x["q_lr"], x["k_lr"], x["v_lr"], x["do_hr"],
            x["do_lr"], g, O.HR_WINDOW_FIRST)
    dQ, dK, dV = O.attention_backward(*args)
    rows = np.array([0, 17, 100, g.N, g.N + g.L - 1])
    keys = np.array([3, 60, 255, g.N + 1])
    sQ, sK, sV = O.attention_backward(*args, rows=rows, keys=keys)
    np.testing.assert_allclose(sQ, dQ[:, rows], rtol=0, atol=1e-13)
    np.testing.assert_allclose(sK, dK[:, keys], rtol=0, atol=1e-13)
    np.testing.assert_allclose(sV, dV[:, keys], rtol=0, atol=1e-13)


@pytest.mark.parametrize("token_set", [O.HR_RASTER, O.HR_WINDOW_FIRST, O.LOWRES])
def test_rope_backward_is_the_adjoint_of_rope(token_set):
    """<R x, y> = <x, R^T y> for every token (fp64, before rounding)."""
    g = geom(H=8, W=12, wh=4, ww=4, lr=(3, 2), text=2, heads=2, d=16, rho=2.5)
    n = g.L if token_set == O.LOWRES else g.N
    rng = np.random.default_rng(6)
    x = O.bf16_to_f64(bf(rng, (1, n, 2, 16)))
    y = O.bf16_to_f64(bf(rng, (1, n, 2, 16)))
    rx = O.rope_2d_f64(x, g, token_set)
    rty = O.rope_2d_backward_f64(y, g, token_set)
    np.testing.assert_allclose((rx * y).sum(axis=-1), (x * rty).sum(axis=-1), rtol=0, atol=1e-12)
    # and R^T undoes R up to the fp32 rounding of cos and sin
    np.testing.assert_allclose(O.rope_2d_backward_f64(rx, g, token_set), x, rtol=0, atol=1e-6)


def test_layer_gradients_match_central_differences_of_an_fp64_layer():
    """The layer in exact arithmetic (RoPE without the bf16 rounding, then
    attention) differenced numerically with respect to its raster inputs."""
    g = geom(H=8, W=8, wh=4, ww=4, r=1, lr=(2, 2), text=1, heads=1, d=8, rho=4.0)
    x = inputs(g, 7)
    dq, dk, dv = O.layer_backward(x, {"do_hr": x["do_hr"], "do_lr": x["do_lr"]}, g,
                                  exact_rope=True)
    raw = {n: [O.bf16_to_f64(x[n + "_hr"]), O.bf16_to_f64(x[n + "_lr"])] for n in "qkv"}
    W = joint64(x, "do")

    def loss(r):
        q = np.concatenate([O.rope_2d_f64(r["q"][0], g, O.HR_RASTER),
                            O.rope_2d_f64(r["q"][1], g, O.LOWRES)], axis=1)[0, :, 0]
        k = np.concatenate([O.rope_2d_f64(r["k"][0], g, O.HR_RASTER),
                            O.rope_2d_f64(r["k"][1], g, O.LOWRES)], axis=1)[0, :, 0]
        v = np.concatenate(r["v"], axis=1)[0, :, 0]
        return loss_f64(g, q, k, v, W, O.HR_RASTER)

    rng = np.random.default_rng(8)
    h = 1e-6
    for name, grad in (("q", dq), ("k", dk), ("v", dv)):
        for _ in range(20):
            i, c = int(rng.integers(0, g.N + g.L)), int(rng.integers(0, g.head_dim))
            part, j = (0, i) if i < g.N else (1, i - g.N)
            r = {n: [a.copy() for a in raw[n]] for n in raw}
            r[name][part][0, j, 0, c] += h
            up = loss(r)
            r[name][part][0, j, 0, c] -= 2 * h
            dn = loss(r)
            assert abs((up - dn) / (2 * h) - grad[0, i, 0, c]) < 1e-7, (name, i, c)
