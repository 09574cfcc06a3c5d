"""Pins for the oracle's text tokens in the global set.

The joint MMDiT sequence concatenates text, high-res and low-res tokens
(UltraGen-it §2, LoRA item; UltraGen-fr §2.C); the pages give no mask for the
text tokens.  The oracle's reading: they lead the global set, every query sees
them, they see the global set only, and they are not rotated.  These checks
fix that reading from outside the oracle's own arithmetic: bit identity of
unrotated rows, a closed form for uniform scores, set (permutation)
invariance, independence from high-res keys, and a reduction to torch's
fp64 attention when text is the whole global set.
"""
import numpy as np
import torch
import torch.nn.functional as F

from oracle import hier_local_attn as O


def geom(H, W, wh, ww, r=1, lr=(0, 0), text=0, heads=2, d=16, rho=4.0):
    return O.Geometry(batch=1, grid_h=H, grid_w=W, win_h=wh, win_w=ww, radius=r,
                      lr_h=lr[0], lr_w=lr[1], rho=rho, heads=heads, head_dim=d,
                      rope_dim_y=d // 2, rope_dim_x=d // 2, text_len=text)


def inputs(g, seed=0):
    rng = np.random.default_rng(seed)
    mk = lambda n: O.f64_to_bf16(rng.standard_normal((g.batch, n, g.heads, g.head_dim)))
    return dict(q_hr=mk(g.N), k_hr=mk(g.N), v_hr=mk(g.N), q_lr=mk(g.L), k_lr=mk(g.L), v_lr=mk(g.L))


def run(g, x):
    return O.attention(x["q_hr"], x["k_hr"], x["v_hr"], x["q_lr"], x["k_lr"], x["v_lr"],
                       g, O.HR_WINDOW_FIRST)


def test_text_rows_are_not_rotated_and_low_res_rows_keep_their_positions():
    g = geom(16, 16, 8, 8, lr=(3, 5), text=7)
    g0 = geom(16, 16, 8, 8, lr=(3, 5), text=0)
    x = inputs(g, 1)["k_lr"]
    y = O.rope_2d(x, g, O.LOWRES)
    np.testing.assert_array_equal(y[:, :7], x[:, :7])
    # the low-res grid after the text rows rotates exactly as without text
    np.testing.assert_array_equal(y[:, 7:], O.rope_2d(x[:, 7:], g0, O.LOWRES))
    assert not np.array_equal(y[:, 8:], x[:, 8:])  # (0, 0) is the identity; the rest is not


def test_uniform_scores_weigh_every_visible_key_equally():
    """k = 0 makes every visible score 0: each query averages the values of
    the keys it sees.  One-hot values tag text / low-res / high-res keys, so
    the output is (text, low-res, high-res) counts over the visible total,
    with the neighbour count of each window enumerated here by hand."""
    H, W, wh, ww, r, lr, text = 24, 16, 8, 8, 1, (2, 3), 5
    g = geom(H, W, wh, ww, r=r, lr=lr, text=text, heads=1, d=16)
    x = inputs(g, 2)
    for name in ("k_hr", "k_lr"):
        x[name] = np.zeros_like(x[name])
    onehot = lambda n, c: O.f64_to_bf16(np.eye(16)[c][None, None, None, :].repeat(n, 1))
    x["v_lr"] = np.concatenate([onehot(text, 0), onehot(g.L - text, 1)], axis=1)
    x["v_hr"] = onehot(g.N, 2)
    o, _ = run(g, x)
    T, L, nlr = wh * ww, g.L, lr[0] * lr[1]
    nwy, nwx = H // wh, W // ww
    for p in range(g.N):  # window-first order: window p // T
        wy, wx = divmod(p // T, nwx)
        nbr = sum(1 for vy in range(nwy) for vx in range(nwx)
                  if abs(vy - wy) <= r and abs(vx - wx) <= r)
        tot = nbr * T + L
        np.testing.assert_allclose(o[0, p, 0, :3], [text / tot, nlr / tot, nbr * T / tot],
                                   rtol=0, atol=1e-15)
    for q in range(g.N, g.N + L):  # text and low-res queries: global keys only
        np.testing.assert_allclose(o[0, q, 0, :3], [text / L, nlr / L, 0.0], rtol=0, atol=1e-15)


def test_text_tokens_form_a_set():
    """Reordering the text tokens reorders the text outputs and leaves every
    other output unchanged (no position is attached to text)."""
    g = geom(16, 24, 8, 8, lr=(2, 2), text=9)
    x = inputs(g, 3)
    o, lse = run(g, x)
    perm = np.random.default_rng(4).permutation(9)
    y = dict(x)
    for name in ("q_lr", "k_lr", "v_lr"):
        y[name] = np.concatenate([x[name][:, perm], x[name][:, 9:]], axis=1)
    o2, lse2 = run(g, y)
    N = g.N
    np.testing.assert_allclose(o2[:, :N], o[:, :N], rtol=0, atol=1e-12)
    np.testing.assert_allclose(o2[:, N + 9:], o[:, N + 9:], rtol=0, atol=1e-12)
    np.testing.assert_allclose(o2[:, N:N + 9], o[:, N + perm], rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse2[:, :, N:N + 9], lse[:, :, N + perm], rtol=0, atol=1e-12)


def test_text_queries_do_not_see_high_res_keys():
    g = geom(16, 16, 8, 8, lr=(2, 2), text=6)
    x = inputs(g, 5)
    o, _ = run(g, x)
    y = dict(x, k_hr=inputs(g, 6)["k_hr"], v_hr=inputs(g, 7)["v_hr"])
    o2, _ = run(g, y)
    np.testing.assert_array_equal(o2[:, g.N:], o[:, g.N:])
    assert np.abs(o2[:, :g.N] - o[:, :g.N]).max() > 0.1


def test_text_as_the_whole_global_set_is_plain_attention_for_text_queries():
    """No low-res grid: text queries attend over the text keys alone, which
    torch's fp64 scaled_dot_product_attention computes independently."""
    g = geom(16, 16, 8, 8, lr=(0, 0), text=11)
    x = inputs(g, 8)
    o, _ = run(g, x)
    for h in range(g.heads):
        t = lambda n: torch.from_numpy(O.bf16_to_f64(x[n][0, :, h]))[None]
        want = F.scaled_dot_product_attention(t("q_lr"), t("k_lr"), t("v_lr"), scale=g.scale)[0]
        np.testing.assert_allclose(o[0, g.N:, h], want.numpy(), rtol=0, atol=1e-12)
