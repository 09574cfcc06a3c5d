"""GPU parity of ug_warm_start against the fp64 oracle.

Tolerance, from the arithmetic: the kernel evaluates each output with about
fifteen fp32 operations on values of magnitude at most
M = (1 + 2|amount|) * max(|x_lr|, |noise|), each rounding by at most 2^-24
relative, so |error| <= 16 * 2^-24 * M < 1e-6 * M; the test allows 4e-6 * M.
The factor-4 kernel instead sums nine weight x sample products (weights
rounded once from fp64; their absolute values sum to at most
(1 - t)(1 + 2|amount|)) and the noise term: ten fused operations, within the
same bound.
"""
import numpy as np
import pytest
import torch

from block_sparse_local_raster_b200 import ug, workloads
from oracle import warm_start as W

pytestmark = pytest.mark.gpu
DEV = "cuda"


def bound(ws, x):
    m = max(float(x["x_lr"].abs().max()), float(x["noise"].abs().max()))
    return 4e-6 * (1 + 2 * abs(ws.sharpen)) * m


@pytest.mark.parametrize("name", list(workloads.WARM_START))
def test_warm_start_matches_oracle(name):
    ws = workloads.WARM_START[name]
    x = workloads.make_warm_start_inputs(ws, seed=11)
    out = ug.warm_start(x["x_lr"].to(DEV), x["noise"].to(DEV), ws.scale, ws.sharpen, ws.t)
    torch.cuda.synchronize()
    want = W.warm_start(x["x_lr"].double().numpy(), x["noise"].double().numpy(), ws.scale,
                        ws.sharpen, ws.t)
    err = np.abs(out.cpu().double().numpy() - want).max()
    assert err <= bound(ws, x), err


@pytest.mark.parametrize("name", ["odd", "s4_edges"])
def test_in_place_over_the_noise_gives_the_same_result(name):
    ws = workloads.WARM_START[name]
    x = workloads.make_warm_start_inputs(ws, seed=12)
    lr, noise = x["x_lr"].to(DEV), x["noise"].to(DEV)
    ref = ug.warm_start(lr, noise, ws.scale, ws.sharpen, ws.t)
    ug.warm_start(lr, noise, ws.scale, ws.sharpen, ws.t, out=noise)
    torch.cuda.synchronize()
    assert torch.equal(ref, noise)


def test_pure_noise_and_no_noise_end_points():
    ws = workloads.WARM_START["wide"]
    x = workloads.make_warm_start_inputs(ws, seed=13)
    lr, noise = x["x_lr"].to(DEV), x["noise"].to(DEV)
    assert torch.equal(ug.warm_start(lr, noise, ws.scale, 0.7, 1.0), noise)
    up = ug.warm_start(lr, noise, ws.scale, 0.0, 0.0).cpu().double().numpy()
    np.testing.assert_allclose(up, W.bilinear_upsample(x["x_lr"].double().numpy(), ws.scale),
                               rtol=0, atol=4e-6 * float(x["x_lr"].abs().max()))


def test_warm_start_argument_errors():
    lr = torch.zeros((1, 2, 4, 4), device=DEV)
    noise = torch.zeros((1, 2, 16, 16), device=DEV)
    out = torch.empty_like(noise)
    assert ug.warm_start_raw(lr, noise, out, 4, 0.5, 1.5) == ug.UG_ERR_INVALID_ARG
    assert ug.warm_start_raw(lr, noise, out, 0, 0.5, 0.5) == ug.UG_ERR_INVALID_ARG
    flat = torch.zeros(noise.numel() + 4, device=DEV)
    assert ug.warm_start_raw(lr, noise, flat[1:1 + noise.numel()].view_as(noise), 4, 0.5,
                             0.5) == ug.UG_ERR_ALIGNMENT
    big = torch.zeros(noise.numel() + 64, device=DEV)
    shifted = big[32:32 + noise.numel()].view_as(noise)
    big_noise = big[:noise.numel()].view_as(noise)
    assert ug.warm_start_raw(lr, big_noise, shifted, 4, 0.5, 0.5) == ug.UG_ERR_ALIAS
    both = torch.zeros(noise.numel() + lr.numel(), device=DEV)
    assert ug.warm_start_raw(both[:lr.numel()].view_as(lr), noise,
                             both[:noise.numel()].view_as(noise), 4, 0.5, 0.5) == ug.UG_ERR_ALIAS
    torch.cuda.synchronize()
