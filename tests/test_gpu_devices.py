"""Plans and devices: a plan belongs to the device current at its creation.

* Two plans of different geometries on one device, created and run from two
  host threads at once (ctypes releases the GIL during the calls), give the
  same bits as the same calls made one after the other.
* A call made with another device current is refused before any work is
  queued (needs two GPUs; skipped otherwise).
"""
import threading

import pytest
import torch

from block_sparse_local_raster_b200 import ug, workloads

pytestmark = pytest.mark.gpu


def _run(name, seed, out, errors):
    try:
        wl = workloads.get(name)
        plan = ug.Plan(**wl.geom_dict())
        x = workloads.make_inputs(wl, seed=seed)
        x.pop("head_scale", None)
        d = {k: v.to("cuda") for k, v in x.items()}
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            res = ug.layer_forward(plan, d["q_hr"], d["k_hr"], d["v_hr"], d["q_lr"], d["k_lr"],
                                   d["v_lr"])
        s.synchronize()
        assert plan.check_error(s) == ug.UG_OK
        out[name] = [t.clone() for t in res]
        plan.close()
    except Exception as e:  # reported by the main thread
        errors.append(e)


def test_two_plans_two_threads_one_device():
    names = ("tiny", "multi_tile")
    seq, errors = {}, []
    for n in names:
        _run(n, 5, seq, errors)
    assert not errors, errors
    par = {}
    th = [threading.Thread(target=_run, args=(n, 5, par, errors)) for n in names]
    for t in th:
        t.start()
    for t in th:
        t.join()
    assert not errors, errors
    for n in names:
        for a, b in zip(seq[n], par[n]):
            assert torch.equal(a, b), n


@pytest.mark.skipif(torch.cuda.device_count() < 2, reason="needs two GPUs")
def test_call_on_another_device_is_refused():
    wl = workloads.get("tiny")
    with torch.cuda.device(0):
        plan = ug.Plan(**wl.geom_dict())
    with torch.cuda.device(1):
        x = torch.zeros(wl.batch, wl.n_hr, wl.heads, wl.head_dim, dtype=torch.bfloat16,
                        device="cuda:1")
        y = torch.empty_like(x)
        assert plan.permute_window_first(x, y) == ug.UG_ERR_INVALID_ARG
        assert plan.check_error() == ug.UG_ERR_INVALID_ARG
    with torch.cuda.device(0):
        assert plan.check_error() == ug.UG_OK
    plan.close()
