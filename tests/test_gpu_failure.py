"""Failure detection on the GPU without a fault: every device-side wait of the
attention kernels (forward and backward) is bounded.  With a bound far below ordinary wait times the
waits expire, the kernel records UG_ERR_TIMEOUT, drains its in-flight work,
frees its tensor memory and exits; the host reads the status and the CUDA
context stays usable."""
import numpy as np
import pytest
import torch

from block_sparse_local_raster_b200 import ug, workloads

pytestmark = pytest.mark.gpu


def _run(p, d):
    return ug.hier_local_attn_fwd(p, d["q_hr"], d["k_hr"], d["v_hr"], d["q_lr"], d["k_lr"],
                                  d["v_lr"])


def test_expired_waits_report_timeout_and_context_survives():
    wl = workloads.get("2K")
    x = workloads.make_inputs(wl, seed=900)
    d = {k: v.to("cuda") for k, v in x.items()}
    ref = ug.Plan(**wl.geom_dict())
    want_hr, want_lr, _ = _run(ref, d)
    torch.cuda.synchronize()
    assert ref.check_error() == ug.UG_OK

    p = ug.Plan(**wl.geom_dict())
    assert p.set_wait_timeout(200) == ug.UG_OK      # 200 ns: ordinary waits expire
    _run(p, d)                                      # launch itself succeeds
    assert p.check_error() == ug.UG_ERR_TIMEOUT     # recorded on the device
    assert p.check_error() == ug.UG_OK              # and cleared by the read

    assert p.set_wait_timeout(2_000_000_000) == ug.UG_OK
    got_hr, got_lr, _ = _run(p, d)
    torch.cuda.synchronize()
    assert p.check_error() == ug.UG_OK
    assert torch.equal(got_hr, want_hr) and torch.equal(got_lr, want_lr)


def test_backward_expired_waits_report_timeout_and_context_survives():
    """The dQ and dK/dV kernels give up the same way: their producers drain
    the loads in flight, the polling MMA thread its products, the softmax
    warps leave their (bounded) barriers; a rerun with the normal bound is
    bit-identical to a fresh plan's."""
    wl = workloads.get("2K")
    x = workloads.make_inputs(wl, seed=910)
    x.update(workloads.make_grad_outputs(wl, seed=911))
    d = {k: v.to("cuda") for k, v in x.items()}

    def bwd(p):
        o_hr, o_lr, lse = _run(p, d)
        return ug.hier_local_attn_bwd(p, d["q_hr"], d["k_hr"], d["v_hr"], d["q_lr"], d["k_lr"],
                                      d["v_lr"], o_hr, o_lr, d["do_hr"], d["do_lr"], lse)

    ref = ug.Plan(**wl.geom_dict())
    want = bwd(ref)
    torch.cuda.synchronize()
    assert ref.check_error() == ug.UG_OK

    p = ug.Plan(**wl.geom_dict())
    o_hr, o_lr, lse = _run(p, d)                    # forward with the normal bound
    torch.cuda.synchronize()
    assert p.check_error() == ug.UG_OK
    assert p.set_wait_timeout(200) == ug.UG_OK
    ug.hier_local_attn_bwd(p, d["q_hr"], d["k_hr"], d["v_hr"], d["q_lr"], d["k_lr"], d["v_lr"],
                           o_hr, o_lr, d["do_hr"], d["do_lr"], lse)
    assert p.check_error() == ug.UG_ERR_TIMEOUT
    assert p.check_error() == ug.UG_OK

    assert p.set_wait_timeout(2_000_000_000) == ug.UG_OK
    got = bwd(p)
    torch.cuda.synchronize()
    assert p.check_error() == ug.UG_OK
    assert all(torch.equal(a, b) for a, b in zip(got, want))


def test_wait_timeout_argument_checks():
    p = ug.Plan(**workloads.get("tiny").geom_dict())
    assert p.set_wait_timeout(0) == ug.UG_ERR_INVALID_ARG
    assert p.set_wait_timeout(-5) == ug.UG_ERR_INVALID_ARG
