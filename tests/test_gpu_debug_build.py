"""The range-checked debug build, with canaries around every output.

compute-sanitizer is not available on the GPU pool, so memory safety is
checked two other ways on every small geometry (several tiles, ragged tails,
straddling windows, text tokens, no low-res set):
  * libug_debug.so (built with -DUG_DEBUG=1) checks, inside the kernels, every
    global index they compute before the access -- block-list entries, token
    runs of the permutations, rows of the raster scatter, RoPE table rows --
    and records a failure in the plan's error word;
  * every output and workspace buffer sits between two 256-byte canary
    regions, which must be intact after each call.
Every entry point of the layer runs through the debug build; its status and
error word must be clean, the canaries intact, and its outputs equal to the
release build's bit for bit (the checks change no arithmetic).
"""
import math

import pytest
import torch

from block_sparse_local_raster_b200 import build as ugbuild
from block_sparse_local_raster_b200 import ug, workloads

pytestmark = pytest.mark.gpu

SMALL = list(workloads.TEST_GEOMETRIES) + ["tiny"]
PAD = 256
FILL = 0xA5


class Guarded:
    """A tensor between two 256-byte canary regions of one allocation."""

    def __init__(self, shape, dtype):
        self.n = math.prod(shape) * torch.tensor([], dtype=dtype).element_size()
        self.buf = torch.full((self.n + 2 * PAD,), FILL, dtype=torch.uint8, device="cuda")
        self.t = self.buf[PAD:PAD + self.n].view(dtype).view(shape)

    def intact(self) -> bool:
        return bool((self.buf[:PAD] == FILL).all()) and bool((self.buf[PAD + self.n:] == FILL).all())


@pytest.fixture(scope="module")
def debug_lib():
    ugbuild.build(debug=True)  # no-op when up to date
    yield ug.LIB_DEBUG_PATH


def run_all(wl, lib_path, d, g):
    """Every entry point of the layer on one geometry through the library at
    lib_path; returns (outputs, guards)."""
    prev = ug.use_library(lib_path)
    try:
        plan = ug.Plan(**wl.geom_dict())
        B, N, H, D = d["q_hr"].shape
        L = wl.n_lr
        hr, lr = (B, N, H, D), (B, L, H, D)
        bf = torch.bfloat16
        out, guards = {}, []

        def G(name, shape, dtype=bf):
            x = Guarded(shape, dtype)
            guards.append((name, x))
            out[name] = x.t
            return x.t

        lrin = lambda n: d[n] if L else None

        def ok(st, what):
            assert st == ug.UG_OK, (what, ug.status_string(st))

        # permutations and RoPE
        ok(plan.permute_window_first(d["q_hr"], G("perm_q", hr)), "permute")
        ok(plan.unpermute(out["perm_q"], G("unperm_q", hr)), "unpermute")
        ok(plan.permute_rope_window_first(d["q_hr"], G("prope_q", hr)), "permute+rope")
        ok(plan.unpermute_rope_bwd(out["prope_q"], G("unprope_q", hr)), "unpermute+rope bwd")
        for ts in (ug.UG_HR_WINDOW_FIRST, ug.UG_HR_RASTER):
            ok(plan.rope_2d(d["k_hr"], G(f"rope_{ts}", hr), ts), "rope")
            ok(plan.rope_2d_bwd(d["k_hr"], G(f"ropeb_{ts}", hr), ts), "rope bwd")
        if L:
            ok(plan.rope_2d(d["k_lr"], G("rope_lr", lr), ug.UG_LR), "rope lr")
        # attention on window-first operands
        ok(plan.hier_local_attn_fwd(out["perm_q"], d["k_hr"], d["v_hr"], lrin("q_lr"),
                                    lrin("k_lr"), lrin("v_lr"), G("o_wf", hr),
                                    G("o_lr", lr) if L else None,
                                    G("lse", (B, H, N + L), torch.float32)), "attention")
        if ug_vo_raster(wl):
            ok(plan.hier_local_attn_fwd_vo_raster(out["perm_q"], d["k_hr"], d["v_hr"],
                                                  lrin("q_lr"), lrin("k_lr"), lrin("v_lr"),
                                                  G("o_vo", hr), G("o_lr_vo", lr) if L else None,
                                                  G("lse_vo", (B, H, N + L), torch.float32)),
               "attention, raster v/o")
        # the whole layer, forward and backward
        ws = G("ws", (plan.workspace_bytes(),), torch.uint8)
        ok(plan.layer_fwd(d["q_hr"], d["k_hr"], d["v_hr"], lrin("q_lr"), lrin("k_lr"),
                          lrin("v_lr"), G("lo_hr", hr), G("lo_lr", lr) if L else None,
                          G("llse", (B, H, N + L), torch.float32), ws), "layer")
        bws = G("bws", (plan.layer_bwd_workspace_bytes(),), torch.uint8)
        ok(plan.layer_bwd(d["q_hr"], d["k_hr"], d["v_hr"], lrin("q_lr"), lrin("k_lr"),
                          lrin("v_lr"), out["lo_hr"], out.get("lo_lr"), out["llse"], g["do_hr"],
                          g["do_lr"] if L else None, G("dq", hr), G("dk", hr), G("dv", hr),
                          G("dq_lr", lr) if L else None, G("dk_lr", lr) if L else None,
                          G("dv_lr", lr) if L else None, bws), "layer backward")
        torch.cuda.synchronize()
        assert plan.check_error() == ug.UG_OK, ug.status_string(plan.check_error())
        plan.close()
        return out, guards
    finally:
        ug._set_library(prev)


def ug_vo_raster(wl):
    T = wl.win_h * wl.win_w
    return wl.win_w <= 128 and 128 % wl.win_w == 0 and T % 128 == 0


@pytest.mark.parametrize("name", SMALL)
def test_debug_build_checks_and_canaries(name, debug_lib):
    wl = workloads.get(name)
    x = workloads.make_inputs(wl, seed=21)
    x.pop("head_scale", None)
    d = {k: v.to("cuda") for k, v in x.items()}
    g = {k: v.to("cuda") for k, v in workloads.make_grad_outputs(wl, seed=22).items()}
    dbg, guards = run_all(wl, debug_lib, d, g)
    for what, gd in guards:
        assert gd.intact(), f"{name}: canary overwritten around {what}"
    rel, _ = run_all(wl, ug.LIB_PATH, d, g)
    for k, v in rel.items():
        if k in ("ws", "bws"):
            continue  # scratch
        assert torch.equal(dbg[k], v), f"{name}: debug and release builds differ in {k}"
