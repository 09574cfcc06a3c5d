"""Online-softmax rescaling under large score jumps, against the oracle.

Random unit-variance inputs keep every row's scores within a few log2 units
of each other, so after the first key block the kernel's running reference
max rarely moves and O is rarely rescaled.  This test builds inputs whose
scores climb in large, known steps from one 128-key block of the global set
to the next, and within a block from its first 64 keys to its last 64, so
that every rescaling case runs:
  * a block whose first half already exceeds the reference by 2^40 (O and l
    rescaled before any of the block is used);
  * a block whose first half stays within 2^31 of the reference but whose
    second half exceeds it by 2^33.5 or more (the first half's probabilities,
    taken at the old reference, meet the rescaled O);
  * a final ragged block whose valid keys sit just above the last step.
The top keys of the last steps are 0.3 to 4 log2 units apart, so the output
of every row mixes five value rows with weights between 1 and 1/11: a
probability taken at a wrong reference, or an O or l rescaled by a wrong
factor, moves every row far outside the bounds.

How: the first half of q's channels is exactly 1 and the second half small
noise; a key's first-half channels sum to a chosen value t (bf16 values, the
last channel carrying the remainder), so its score is t * scale plus noise of
about 0.1 log2 units.  High-res keys and the unboosted global keys score ~0.
"""
import math

import numpy as np
import pytest
import torch

from block_sparse_local_raster_b200 import ug, workloads
from oracle import hier_local_attn as O

from parity import LSE_ABS, MEAN_ABS, bits, f64, half_ulp_bf16, ogeom, plan

DEV = "cuda"
LOG2E = 1.0 / math.log(2.0)

# 4 windows of 256 tokens (8 key blocks, each query CTA sees all of them),
# 576 global tokens: 4 full key blocks and a ragged fifth holding 64 keys.
WL = workloads._wl("rescale", 1, (32, 32), (16, 16), (24, 24), 2, 128, (64, 64))

# (global key index, score in log2 units above the previous step's top), by
# block; a block's top key sets the next step's reference.
STEPS = [
    # block 0: its first half is 40 above anything before it
    [(10, 40.0), (20, 39.5), (70, 39.0)],
    # block 1: first half within 2^31 of the reference, second half 33.5 above
    [(128 + 5, 30.5), (128 + 33, 29.0), (128 + 100, 33.5), (128 + 64, 33.0)],
    # block 2: first half 40 above
    [(256 + 50, 40.0), (256 + 0, 39.6), (256 + 127, 40.3)],
    # block 3: first half 31 above, second half 34 above
    [(384 + 63, 31.0), (384 + 64, 34.0), (384 + 90, 33.2)],
    # block 4 (ragged: keys 512..575): just above the last step
    [(512 + 1, 0.5), (512 + 2, -0.5)],
]


def boosted_scores():
    """Global key index -> target score (log2 units)."""
    out, level = {}, 0.0
    for block in STEPS:
        top = max(u for _, u in block)
        for k, u in block:
            out[k] = level + u
        level += top
    return out


def make_inputs(seed):
    wl = WL
    B, N, L, H, D = wl.batch, wl.n_hr, wl.n_lr, wl.heads, wl.head_dim
    scale = 1.0 / math.sqrt(D)
    half = D // 2
    g = torch.Generator().manual_seed(seed)
    bf = torch.bfloat16

    def noise(n, std):
        return (torch.randn((B, n, H, D), generator=g) * std)

    def q_of(n):
        q = noise(n, 0.1)
        q[..., :half] = 1.0
        return q.to(bf)

    def k_plain(n):
        return noise(n, 0.1).to(bf)

    k_lr = noise(L, 0.1)
    for key, u in boosted_scores().items():
        t = u / (scale * LOG2E)  # first-half channel sum giving u log2 units
        c = torch.tensor(t / half, dtype=torch.float32).to(bf).float()
        k_lr[:, key, :, :half - 1] = c
        k_lr[:, key, :, half - 1] = t - float(c) * (half - 1)
    x = {
        "q_hr": q_of(N), "k_hr": k_plain(N), "v_hr": torch.randn((B, N, H, D), generator=g).to(bf),
        "q_lr": q_of(L), "k_lr": k_lr.to(bf), "v_lr": torch.randn((B, L, H, D), generator=g).to(bf),
    }
    return x


def test_construction_hits_every_rescaling_case():
    """The actual bf16 scores keep the margins the cases need, and the output
    mixes five value rows (host only; exact fp64 scores of one query row)."""
    x = make_inputs(5)
    scale = 1.0 / math.sqrt(WL.head_dim)
    q = x["q_lr"][0, 0, 0].double()
    k = x["k_lr"][0, :, 0].double()
    s = (k @ q).numpy() * scale * LOG2E
    want = boosted_scores()
    for key, u in want.items():
        assert abs(s[key] - u) < 0.2, (key, s[key], u)
    others = np.setdiff1d(np.arange(len(s)), list(want))
    assert np.abs(s[others]).max() < 1.0
    top = sorted(want.values(), reverse=True)[:5]
    w = np.array([2.0 ** (u - top[0]) for u in top])
    assert w[-1] > 1.0 / 12 and w[0] / w.sum() < 0.5


@pytest.mark.gpu
def test_rescaling_every_row_against_oracle():
    """Every row and head against the oracle, under an elementwise bound
    derived from the arithmetic: the bf16 probabilities (relative error
    <= 2^-9 each, so <= 2^-9 sum_i w_i |v_i| on a row, where w are the exact
    softmax weights; the oracle gives that sum as the attention output of
    |v|), plus the rounding of the output to bf16 (half an ulp), with a 2x
    margin on both; lse within LSE_ABS."""
    wl = WL
    g = ogeom(wl)
    p = plan(wl)
    x = make_inputs(5)
    d = {k: v.to(DEV) for k, v in x.items()}
    o_hr, o_lr, lse = ug.hier_local_attn_fwd(p, d["q_hr"], d["k_hr"], d["v_hr"], d["q_lr"],
                                             d["k_lr"], d["v_lr"])
    torch.cuda.synchronize()
    assert p.check_error() == ug.UG_OK
    xb = {k: bits(v) for k, v in x.items()}
    ref_o, ref_lse = O.attention(xb["q_hr"], xb["k_hr"], xb["v_hr"], xb["q_lr"], xb["k_lr"],
                                 xb["v_lr"], g, O.HR_WINDOW_FIRST)
    abs_o, _ = O.attention(xb["q_hr"], xb["k_hr"], xb["v_hr"] & 0x7FFF, xb["q_lr"], xb["k_lr"],
                           xb["v_lr"] & 0x7FFF, g, O.HR_WINDOW_FIRST)
    got = np.concatenate([f64(o_hr), f64(o_lr)], axis=1)
    err = np.abs(got - ref_o)
    bound = 2.0 ** -8 * abs_o + 2.0 * half_ulp_bf16(ref_o) + 1e-4
    worst = float((err / bound).max())
    print(f"max-abs {err.max():.3g}, mean-abs {err.mean():.3g}, worst error / bound {worst:.3f}")
    assert worst <= 1.0
    assert err.mean() <= MEAN_ABS
    assert np.abs(lse.cpu().numpy() - ref_lse).max() <= LSE_ABS
