#!/usr/bin/env python
"""Benchmark of one hierarchical-local-attention layer on B200.

A step is one pass of the whole layer over one batch of synthetic raster-order
inputs already resident in HBM: window-first permute of q and k with their RoPE
applied in the same pass (2 launches), RoPE of the global q and k (2), the
block-sparse attention (1).  Where 128-key tiles are whole window rows (2K, 4K,
8K, 4K-CFG) the attention reads v and writes o in raster order itself;
elsewhere v is permuted first and o unpermuted after (2 more launches).  The
metric is useful attention TFLOP/s
(4 * head_dim FLOPs per visible query-key pair per head) over the step, with
ms per layer; the attention kernel alone is also timed and set against the
measured bf16 tensor peak.

The default run times the 4K layer (the JSON line's value), then in the same
process the 2K, 8K and 4K-CFG layers (``per_config``) and the 4K layer's
backward pass (``backward``), each with its own clock record and roofline.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config 4K] [--impl ug|reference]
  python bench.py --op warm_start [--config 4K|8K]   (the warm-start kernel alone)
  python bench.py --op backward [--config 4K]        (the layer's backward pass alone)

N > 1 runs under torchrun, one rank per GPU; every rank runs its own layer on
its own inputs (independent problems, weak scaling, no data-path collective);
the time is the max over ranks.  ``--impl reference`` times the fp64 CPU
oracle on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from block_sparse_local_raster_b200 import workloads  # noqa: E402

METRIC = "useful attn TFLOP/s & ms/layer at 4K/8K token grids; % of B200 bf16 tensor peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 * 1024 * 1024


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)  # --op warm_start: use ~20000 (14 us each)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="4K", choices=list(workloads.CONFIGS) + list(workloads.EXTRA_CONFIGS))
    ap.add_argument("--impl", default="ug", choices=["ug", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=12)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--op", default="layer", choices=["layer", "warm_start", "backward"])
    ap.add_argument("--per-config", default="2K,8K,4K-CFG",
                    help="configs timed after the main one in the same run ('' = none)")
    ap.add_argument("--no-backward", action="store_true",
                    help="skip the backward pass timed after the main layer")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def useful_flops(wl) -> int:
    from block_sparse_local_raster_b200 import ug
    pairs = sum(ug.visible_pairs(ug.make_geom(**wl.geom_dict())))
    return 4 * wl.head_dim * pairs * wl.heads * wl.batch


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(backend: str, world: int):
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))


def reduce_max(x: float, device) -> float:
    """Max over ranks (identity for a single process)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def aggregate(units_per_rank: float, world: int, max_seconds: float) -> float:
    """Whole-job throughput: the units all ranks processed / the slowest rank."""
    return units_per_rank * world / max_seconds


def _nvml_handle(device_index: int):
    """NVML handle of the CUDA device (by UUID, else PCI bus id)."""
    import pynvml
    pynvml.nvmlInit()
    props = torch.cuda.get_device_properties(device_index)
    tries = []
    u = str(getattr(props, "uuid", ""))
    if u:
        tries += [lambda: pynvml.nvmlDeviceGetHandleByUUID(u if u.startswith("GPU-") else "GPU-" + u)]
    if hasattr(props, "pci_bus_id"):
        bus = "%08X:%02X:%02X.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
        tries += [lambda: pynvml.nvmlDeviceGetHandleByPciBusId(bus)]
    for t in tries:
        try:
            return t()
        except Exception:
            continue
    raise RuntimeError("no NVML handle for this device")


class ClockSampler:
    """SM clock, power and clock-event reasons sampled during the timed
    region, read-only: NVML every 10 ms from a thread (nvidia-smi at 20 ms if
    NVML is unavailable).  Each sample carries its host time; stop(t0, t1)
    summarises the samples taken between t0 and t1 (the timed region), or,
    when that window holds fewer than 3 (a region of a few tens of ms, or a
    slow NVML), those of the region and the warm-up just before it, and says
    which."""

    SMI = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
           "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
           "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40),
               ("sw_thermal_slowdown", 0x20), ("sw_power_cap", 0x4))

    def __init__(self, device_index: int, period_s: float = 0.01):
        self.dev = device_index
        self.period = period_s
        self.rows = []  # (sm_mhz, sm_max_mhz, power_w, reason bits, host time)
        self.thread = None
        self.proc = None
        self.stop_flag = False
        self.source = None

    def _nvml_loop(self, h):
        import pynvml
        smax = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        while not self.stop_flag:
            try:
                sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                pw = pynvml.nvmlDeviceGetPowerUsage(h) / 1000.0
                rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.rows.append((float(sm), float(smax), pw, int(rs), time.perf_counter()))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        try:
            import threading
            h = _nvml_handle(self.dev)
            self.thread = threading.Thread(target=self._nvml_loop, args=(h,), daemon=True)
            self.thread.start()
            self.source = "nvml, 10 ms"
            return
        except Exception:
            self.thread = None
        try:
            self.out = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.dev}", f"--query-gpu={self.SMI}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=self.out, stderr=subprocess.DEVNULL)
            self.source = "nvidia-smi, 20 ms"
        except OSError:
            self.proc = None

    def stop(self, t0=None, t1=None):
        if self.thread is not None:
            self.stop_flag = True
            self.thread.join(timeout=5)
        elif self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.out.flush()
            for line in open(self.out.name).read().strip().splitlines():
                r = line.split(", ")
                try:
                    bits = sum(b for (_, b), v in zip(self.REASONS, r[5:9]) if v.strip() == "Active")
                    self.rows.append((float(r[1]), float(r[2]), float(r[3]), bits, None))
                except (ValueError, IndexError):
                    continue
            os.unlink(self.out.name)
        else:
            return None
        rows, window = self.rows, "whole sampling"
        if t0 is not None and all(r[4] is not None for r in rows):
            inside = [r for r in rows if t0 <= r[4] <= t1]
            if len(inside) >= 3:
                rows, window = inside, "timed region"
            else:
                rows, window = [r for r in rows if r[4] <= t1], "timed region and the warm-up before it"
        out = self.summary(rows)
        if out:
            out["window"] = window
        return out

    def summary(self, rows):
        if not rows:
            return None
        sm = [r[0] for r in rows]
        reasons = sorted({n for r in rows for n, b in self.REASONS if r[3] & b})
        return {"sm_mhz": statistics.median(sm), "sm_min_mhz": min(sm),
                "sm_max_mhz": max(r[1] for r in rows),
                "power_w_max": round(max(r[2] for r in rows), 1),
                "reasons": reasons, "samples": len(rows), "source": self.source}


def pick_peak(pk, region_s: float, clk):
    """The bf16 peak that applies to a kernel timed over region_s seconds.

    The burst figure (cuBLAS timed alone, full clock) unless the region is a
    second or longer and its clock record shows the power cap or a median SM
    clock below 95 % of max: then the sustained figure (cuBLAS after seconds
    under the power cap).  Returns (peak, kind)."""
    throttled = clk is not None and ("sw_power_cap" in clk["reasons"]
                                     or clk["sm_mhz"] < 0.95 * clk["sm_max_mhz"])
    if region_s >= 1.0 and throttled:
        return pk["bf16_tflops_sustained"], "sustained"
    return pk["bf16_tflops"], "burst"


def tensor_roofline(achieved: float, region_s: float, clk, traffic=None, note=None):
    pk, src = peaks()
    peak, kind = pick_peak(pk, region_s, clk)
    r = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
         "frac": achieved / peak, "traffic": traffic,
         "peak_source": f"{src} bf16 cuBLAS, {kind} (timed region {region_s:.2f} s; "
                        "burst below 1 s or at full clock without the power cap)",
         "peak_kind": kind,
         "frac_of_burst_peak": achieved / pk["bf16_tflops"],
         "frac_of_sustained_peak": achieved / pk["bf16_tflops_sustained"]}
    if note:
        r["note"] = note
    return r


def attn_source_hash() -> str:
    """sha256 (16 hex digits) over the forward attention kernel's sources."""
    csrc = os.path.join(ROOT, "block_sparse_local_raster_b200", "csrc")
    hs = hashlib.sha256()
    for f in ("ug_attn.cu", "ug_tc.cuh"):
        hs.update(open(os.path.join(csrc, f), "rb").read())
    return hs.hexdigest()[:16]


def attn_traffic_bytes(config: str):
    """DRAM bytes per attention launch from the committed ncu summary, or None
    if the kernel source changed since the counters were taken."""
    p = os.path.join(ROOT, "profiles", "attention_dram_traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    h = attn_source_hash()
    e = d.get(config)
    if not e or e.get("source_sha256_16") != h:
        return None
    return e.get("bytes_per_launch")


# ----------------------------------------------------------------------------- CPU oracle

def cpu_threads() -> int:
    """Threads the oracle's BLAS uses."""
    try:
        from threadpoolctl import threadpool_info
        n = [i["num_threads"] for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:
        return 1


def cpu_cores() -> int:
    """Host cores this process may run on (nproc)."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


class OracleArm:
    """The fp64 CPU oracle on a bounded sample of the workload."""

    def __init__(self, wl, rows_hr: int, rows_lr: int, heads, seed: int = 0):
        from oracle import hier_local_attn as O
        self.O = O
        self.g = O.Geometry.from_dict(wl.geom_dict())
        x = workloads.make_inputs(wl, seed=seed)
        self.bits = {k: v.view(torch.int16).numpy().view(np.uint16)
                     for k, v in x.items() if k != "head_scale"}
        rng = np.random.default_rng(seed)
        hr = rng.choice(self.g.N, size=min(rows_hr, self.g.N), replace=False)
        lr = rng.choice(self.g.L, size=min(rows_lr, self.g.L), replace=False) if self.g.L else []
        self.rows = np.sort(np.concatenate([hr, self.g.N + np.asarray(lr, dtype=np.int64)]))
        self.heads = list(heads)
        # useful FLOPs of the sample: visible keys of each sampled row
        T = self.g.T
        off, idx = O.window_neighbours(self.g)
        perm = O.window_first_index(self.g)
        vis = 0
        for r in self.rows:
            if r < self.g.N:
                w = perm[r] // T
                vis += (off[w + 1] - off[w]) * T + self.g.L
            else:
                vis += self.g.L
        self.flops = 4 * self.g.head_dim * vis * len(self.heads) * wl.batch

    def step(self):
        self.O.layer_forward(self.bits, self.g, self.rows, self.heads)


def run_reference(args, wl, world, rank):
    if rank != 0:
        return
    arm = OracleArm(wl, rows_hr=8, rows_lr=2, heads=[0])
    for _ in range(args.warmup):
        arm.step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        arm.step()
    dt = (time.perf_counter() - t0) / args.steps
    value = arm.flops / dt / 1e12
    sample = (f"{len(arm.rows)} query rows ({(arm.rows < arm.g.N).sum()} high-res, "
              f"{(arm.rows >= arm.g.N).sum()} low-res) x 1 head of the {wl.name} layer per step, "
              "RoPE of all keys of that head included; fp64 numpy")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "sample": sample},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cpu_threads(), "nproc": cpu_cores(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- GPU arm

def _chk(st, what):
    from block_sparse_local_raster_b200 import ug
    if st != ug.UG_OK:
        raise ug.UgError(st, what)


class LayerRunner:
    """One layer step on device-resident raster inputs `d`, launched as
    ug_layer_fwd does but call by call, so that the attention launch can be
    bracketed by its own CUDA events."""

    def __init__(self, wl, d, dev, stream):
        from block_sparse_local_raster_b200 import ug
        self.ug, self.wl, self.d, self.stream = ug, wl, d, stream
        self.plan = ug.Plan(**wl.geom_dict())
        B, N, H, D = d["q_hr"].shape
        L = self.L = wl.n_lr
        self.ws = torch.empty(self.plan.workspace_bytes(), dtype=torch.uint8, device=dev)
        self.o_hr = torch.empty_like(d["q_hr"])
        self.o_lr = torch.empty_like(d["q_lr"]) if L else None
        self.lse = torch.empty((B, H, N + L), dtype=torch.float32, device=dev)
        self.hr_bytes = hb = d["q_hr"].numel() * 2
        lb = d["q_lr"].numel() * 2
        up = lambda n: (n + 255) // 256 * 256
        ws = self.ws
        view = lambda off, nb, n: ws[off:off + nb].view(torch.bfloat16).view(B, n, H, D)
        # window-first scratch inside the workspace, same split as ug_layer_fwd
        self.q_wf, self.k_wf = view(0, hb, N), view(up(hb), hb, N)
        self.v_wf, self.o_wf = view(2 * up(hb), hb, N), view(3 * up(hb), hb, N)
        o4 = 4 * up(hb)
        self.ql = view(o4, lb, L) if L else None
        self.kl = view(o4 + up(lb), lb, L) if L else None
        # where 128-key tiles are whole window rows the attention reads v and
        # writes o in raster order (no permute of v, no unpermute of o)
        T = wl.win_h * wl.win_w
        self.vo_raster = 128 % wl.win_w == 0 and T % 128 == 0
        self.launches = 2 + (2 if L else 0) + 1 + (0 if self.vo_raster else 2)
        self.flops = useful_flops(wl)

    @staticmethod
    def launches_of(wl) -> int:
        T = wl.win_h * wl.win_w
        vo = 128 % wl.win_w == 0 and T % 128 == 0
        return 2 + (2 if wl.n_lr else 0) + 1 + (0 if vo else 2)

    def step(self, ev=None):
        ug, d, p, L = self.ug, self.d, self.plan, self.L
        _chk(p.permute_rope_window_first(d["q_hr"], self.q_wf), "permute+rope q")
        _chk(p.permute_rope_window_first(d["k_hr"], self.k_wf), "permute+rope k")
        if not self.vo_raster:
            _chk(p.permute_window_first(d["v_hr"], self.v_wf), "permute v")
        if L:
            _chk(p.rope_2d(d["q_lr"], self.ql, ug.UG_LR), "rope q_lr")
            _chk(p.rope_2d(d["k_lr"], self.kl, ug.UG_LR), "rope k_lr")
        if ev is not None:
            ev[0].record(self.stream)
        vl = d["v_lr"] if L else None
        if self.vo_raster:
            _chk(p.hier_local_attn_fwd_vo_raster(self.q_wf, self.k_wf, d["v_hr"], self.ql,
                                                 self.kl, vl, self.o_hr, self.o_lr, self.lse),
                 "attention")
        else:
            _chk(p.hier_local_attn_fwd(self.q_wf, self.k_wf, self.v_wf, self.ql, self.kl, vl,
                                       self.o_wf, self.o_lr, self.lse), "attention")
        if ev is not None:
            ev[1].record(self.stream)
        if not self.vo_raster:
            _chk(p.unpermute(self.o_wf, self.o_hr), "unpermute")

    def close(self):
        self.plan.close()


def time_steps(step, steps, warmup, dev, stream, rank, local, per_step_flush_bytes=0):
    """W untimed steps, then exactly `steps` timed ones between a barrier and
    a device synchronise on both sides, with the clocks sampled meanwhile.
    step(ev) records ev[0] / ev[1] around the kernel it wants timed alone.
    When the inputs fit in L2 (per_step_flush_bytes > 0) a buffer of that
    size is written between steps and each step is timed by its own events,
    so the flush is outside the time; otherwise an event between steps
    splits the region into steps without adding to it.  Returns (seconds per
    step, kernel seconds per launch, clock record), max over ranks, and this
    rank's per-step distribution (median, p10, p90 of the step and of the
    timed kernel, ms)."""
    clocks = ClockSampler(local) if rank == 0 else None
    if clocks:
        clocks.start()
    for _ in range(warmup):
        step()
    torch.cuda.synchronize(dev)
    flush = (torch.empty(per_step_flush_bytes, dtype=torch.uint8, device=dev)
             if per_step_flush_bytes else None)
    mk = lambda: torch.cuda.Event(enable_timing=True)
    kev = [(mk(), mk()) for _ in range(steps)]
    sev = [(mk(), mk()) for _ in range(steps)] if flush is not None else None
    bev = [mk() for _ in range(steps + 1)] if flush is None else None
    barrier()
    torch.cuda.synchronize(dev)
    t0, t1 = mk(), mk()
    h0 = time.perf_counter()
    t0.record(stream)
    for i in range(steps):
        if flush is not None:
            flush.fill_(i & 0xFF)
            sev[i][0].record(stream)
        else:
            bev[i].record(stream)
        step(kev[i])
        if flush is not None:
            sev[i][1].record(stream)
    if bev is not None:
        bev[steps].record(stream)
    t1.record(stream)
    torch.cuda.synchronize(dev)
    h1 = time.perf_counter()
    barrier()
    clk = clocks.stop(h0, h1) if clocks else None
    if sev is not None:
        sec = sum(a.elapsed_time(b) for a, b in sev) / 1e3 / steps
    else:
        sec = t0.elapsed_time(t1) / 1e3 / steps
    ksec = sum(a.elapsed_time(b) for a, b in kev) / 1e3 / steps
    per = ([a.elapsed_time(b) for a, b in sev] if sev is not None else
           [bev[i].elapsed_time(bev[i + 1]) for i in range(steps)])
    kper = [a.elapsed_time(b) for a, b in kev]
    pct = lambda v: {"median": float(np.median(v)), "p10": float(np.percentile(v, 10)),
                     "p90": float(np.percentile(v, 90))}
    dist = {"step_ms": pct(per), "kernel_ms": pct(kper)}
    return reduce_max(sec, dev), reduce_max(ksec, dev), clk, dist


def layer_record(args, wl, d, dev, stream, rank, local, steps=None, warmup=None):
    """Times the layer on device inputs d; returns (runner, record dict)."""
    r = LayerRunner(wl, d, dev, stream)
    steps = steps or args.steps
    warmup = warmup if warmup is not None else args.warmup
    flush = 0 if r.hr_bytes > L2_BYTES else 2 * L2_BYTES
    sec, attn, clk, dist = time_steps(r.step, steps, warmup, dev, stream, rank, local, flush)
    _chk(r.plan.check_error(), f"{wl.name} timed steps")
    ach = r.flops / attn / 1e12
    rec = {
        "ms_per_layer": sec * 1e3, "layer_tflops": r.flops / sec / 1e12,
        "attn_ms": attn * 1e3, "attn_tflops": ach, "steps": steps, "warmup": warmup,
        "useful_flop_per_layer": r.flops,
        "l2": ("inputs larger than L2 (each high-res tensor %.0f MB > 126 MB), no flush"
               % (r.hr_bytes / 1e6)) if not flush else
              ("inputs smaller than L2 (%.0f MB per high-res tensor): a %d MB buffer is "
               "written between steps, outside each step's events" % (r.hr_bytes / 1e6,
                                                                       flush >> 20)),
        "roofline": tensor_roofline(ach, sec * steps, clk,
                                    attn_traffic_bytes(wl.name)),
        "clocks": clk,
        "per_step_ms": dist,
    }
    return r, rec


def run_ug(args, wl, world, rank, local):
    from block_sparse_local_raster_b200 import ug
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    init_dist("nccl", world)
    stream = torch.cuda.current_stream(dev)

    host = workloads.make_inputs(wl, seed=rank)
    host.pop("head_scale", None)
    pinned = {k: v.pin_memory() for k, v in host.items()}
    d = {k: v.to(dev) for k, v in pinned.items()}
    L = wl.n_lr
    runner, rec = layer_record(args, wl, d, dev, stream, rank, local)
    plan, o_hr, o_lr, lse, ws = runner.plan, runner.o_hr, runner.o_lr, runner.lse, runner.ws
    flops = runner.flops
    sec_max = rec["ms_per_layer"] / 1e3
    attn_max = rec["attn_ms"] / 1e3

    # End to end through the public API: every step copies its inputs from
    # pinned host memory to the device, runs ug_layer_fwd and copies its
    # result back to pinned host memory.  Steps are pipelined the way a
    # serving loop would run them: copies in, compute and copies out on three
    # streams over double-buffered device inputs/outputs, so step i's
    # host-to-device copy overlaps step i-1's compute and step i-2's
    # device-to-host copy.
    h2d = sum(v.numel() * v.element_size() for v in pinned.values())
    d2h = o_hr.numel() * 2 + (o_lr.numel() * 2 if L else 0)
    s_in = torch.cuda.Stream(dev)
    s_out = torch.cuda.Stream(dev)
    bufs = [d] + [{k: torch.empty_like(v) for k, v in d.items()}]
    outs = [(o_hr, o_lr), (torch.empty_like(o_hr), torch.empty_like(o_lr) if L else None)]
    host_out = [(torch.empty_like(o_hr, device="cpu").pin_memory(),
                 torch.empty_like(o_lr, device="cpu").pin_memory() if L else None)
                for _ in range(2)]
    in_ready = [torch.cuda.Event() for _ in range(2)]
    in_free = [torch.cuda.Event() for _ in range(2)]
    out_ready = [torch.cuda.Event() for _ in range(2)]
    out_free = [torch.cuda.Event() for _ in range(2)]
    for ev in in_free + out_free:
        ev.record(stream)

    def e2e_step(i):
        k = i % 2
        bi, (oh, ol), (hh, hl) = bufs[k], outs[k], host_out[k]
        s_in.wait_event(in_free[k])
        with torch.cuda.stream(s_in):
            for name in bi:
                bi[name].copy_(pinned[name], non_blocking=True)
        in_ready[k].record(s_in)
        stream.wait_event(in_ready[k])
        stream.wait_event(out_free[k])
        _chk(plan.layer_fwd(bi["q_hr"], bi["k_hr"], bi["v_hr"], bi["q_lr"] if L else None,
                            bi["k_lr"] if L else None, bi["v_lr"] if L else None, oh, ol, lse,
                            ws, stream), "ug_layer_fwd")
        in_free[k].record(stream)
        out_ready[k].record(stream)
        s_out.wait_event(out_ready[k])
        with torch.cuda.stream(s_out):
            hh.copy_(oh, non_blocking=True)
            if L:
                hl.copy_(ol, non_blocking=True)
        out_free[k].record(s_out)

    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize(dev)
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    s_in.wait_event(e0)
    for i in range(args.e2e_steps):
        e2e_step(i)
    done = torch.cuda.Event()
    done.record(s_out)
    stream.wait_event(done)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    e2e_sec = reduce_max(e0.elapsed_time(e1) / 1e3 / args.e2e_steps, dev)
    del bufs, outs, host_out

    # The layer's backward pass on the same inputs, and the other configs,
    # timed in the same run (every rank takes the same steps).
    bwd = None
    if not args.no_backward:
        bwd = backward_record(args, wl, d, runner, dev, stream, rank, local)
    runner.close()
    del runner, d, pinned
    torch.cuda.empty_cache()
    per_config = {}
    for name in [c for c in args.per_config.split(",") if c and c != wl.name]:
        pwl = workloads.get(name)
        pd = workloads.make_inputs_on_device(pwl, seed=rank, device=dev)
        pd.pop("head_scale", None)
        steps = max(args.steps, 200) if name in ("tiny", "2K") else args.steps
        pr, prec = layer_record(args, pwl, pd, dev, stream, rank, local, steps=steps)
        prec["inputs"] = "drawn on the device (seeded CUDA generator, same distributions)"
        per_config[name] = prec
        pr.close()
        del pr, pd
        torch.cuda.empty_cache()

    if rank == 0:
        achieved = flops / attn_max / 1e12
        line = {
            "metric": METRIC,
            "value": aggregate(flops, world, sec_max) / 1e12,
            "unit": "TFLOP/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": sec_max * 1e3,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic",
            "config": {
                "workload": wl.name,
                "batch": wl.batch, "grid": [wl.grid_h, wl.grid_w],
                "window": [wl.win_h, wl.win_w], "radius": wl.radius,
                "lowres_grid": [wl.lr_h, wl.lr_w], "rho": wl.rho,
                "heads": wl.heads, "head_dim": wl.head_dim,
                "useful_flop_per_layer": flops,
                "l2": rec["l2"],
                "parallelism": f"independent layer per GPU x{world}",
            },
            "attn_ms": attn_max * 1e3,
            "attn_tflops": achieved,
            "roofline": rec["roofline"],
            "e2e": {"value": aggregate(flops, world, e2e_sec) / 1e12, "unit": "TFLOP/s",
                    "ms_per_step": e2e_sec * 1e3,
                    "how": "ug_layer_fwd per step with its host-to-device input copy and "
                           "device-to-host output copy (pinned host buffers), steps pipelined "
                           "over copy-in / compute / copy-out streams",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": LayerRunner.launches_of(wl) * args.steps,
            "clocks": rec["clocks"],
            "per_step_ms": rec["per_step_ms"],
            "per_config": per_config,
        }
        if bwd is not None:
            line["backward"] = bwd
        if not args.no_cpu_baseline and world == 1:
            arm = OracleArm(wl, rows_hr=48, rows_lr=8, heads=range(wl.heads))
            c0 = time.perf_counter()
            arm.step()
            cdt = time.perf_counter() - c0
            line["cpu_baseline"] = {
                "value": arm.flops / cdt / 1e12, "unit": "TFLOP/s", "cores": cpu_threads(),
                "nproc": cpu_cores(), "kind": "oracle",
                "sample": (f"{len(arm.rows)} query rows x {wl.heads} heads of the {wl.name} "
                           f"layer (RoPE of every key included), fp64 numpy, {cdt:.1f} s"),
                # rows are independent: the whole layer's useful FLOPs at the
                # sample's rate (an upper estimate: the sample's RoPE of every
                # key is a fixed cost that the extrapolation scales too)
                "extrapolated_ms_per_layer": flops / (arm.flops / cdt) * 1e3,
            }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


class BackwardRunner:
    """The layer's backward pass: gradients w.r.t. the raster q, k, v given
    the forward's outputs and lse.  A step recomputes the window-first
    rotated q and k (2 fused permutes with RoPE; RoPE of the global q, k),
    runs the attention backward (D, dQ, dK/dV kernels; timed alone with
    events; v, o, dO read and dv written in raster order where 128-row tiles
    are whole window rows, else 3 more permutes and 1 unpermute) and maps dq,
    dk back with the transposed RoPE and the inverse permutation.  Useful FLOPs: 2.5 x the forward's (five products per
    visible pair: S, dP, dQ, dK, dV, against the forward's two)."""

    def __init__(self, wl, d, plan, o_hr, o_lr, lse, dev):
        from block_sparse_local_raster_b200 import ug
        self.ug, self.wl, self.d, self.plan = ug, wl, d, plan
        self.o_hr, self.o_lr, self.lse = o_hr, o_lr, lse
        L = self.L = wl.n_lr
        lr = self.lr = lambda n: d[n] if L else None
        e = lambda t: torch.empty_like(t) if t is not None else None
        self.wf = {n: torch.empty_like(d["q_hr"]) for n in ("q", "k", "v", "o", "do", "dq", "dk", "dv")}
        self.ql_r, self.kl_r = e(lr("q_lr")), e(lr("k_lr"))
        self.dq_hr, self.dk_hr, self.dv_hr = e(d["q_hr"]), e(d["k_hr"]), e(d["v_hr"])
        self.dq_lr, self.dk_lr, self.dv_lr = e(lr("q_lr")), e(lr("k_lr")), e(lr("v_lr"))
        self.aws = torch.empty(plan.attn_bwd_workspace_bytes(), dtype=torch.uint8, device=dev)
        # where 128-row tiles are whole window rows the backward reads v, o, dO
        # and writes dv in raster order (no permutes of v, o, dO, no unpermute of dv)
        T = wl.win_h * wl.win_w
        self.vo_raster = 128 % wl.win_w == 0 and T % 128 == 0
        self.launches = (2 + (0 if self.vo_raster else 3) + (2 if L else 0) + 3 + 2
                         + (0 if self.vo_raster else 1) + (2 if L else 0))
        self.flops = int(2.5 * useful_flops(wl))

    def step(self, ev=None):
        ug, d, p, wf, L, lr = self.ug, self.d, self.plan, self.wf, self.L, self.lr
        _chk(p.permute_rope_window_first(d["q_hr"], wf["q"]), "q")
        _chk(p.permute_rope_window_first(d["k_hr"], wf["k"]), "k")
        if not self.vo_raster:
            _chk(p.permute_window_first(d["v_hr"], wf["v"]), "v")
            _chk(p.permute_window_first(self.o_hr, wf["o"]), "o")
            _chk(p.permute_window_first(d["do_hr"], wf["do"]), "do")
        if L:
            _chk(p.rope_2d(d["q_lr"], self.ql_r, ug.UG_LR), "q_lr")
            _chk(p.rope_2d(d["k_lr"], self.kl_r, ug.UG_LR), "k_lr")
        if ev is not None:
            ev[0].record(torch.cuda.current_stream())
        if self.vo_raster:
            _chk(p.hier_local_attn_bwd_vo_raster(
                wf["q"], wf["k"], d["v_hr"], self.ql_r, self.kl_r, lr("v_lr"), self.o_hr,
                self.o_lr, d["do_hr"], lr("do_lr"), self.lse, wf["dq"], wf["dk"], self.dv_hr,
                self.dq_lr, self.dk_lr, self.dv_lr, self.aws), "attention backward")
        else:
            _chk(p.hier_local_attn_bwd(wf["q"], wf["k"], wf["v"], self.ql_r, self.kl_r,
                                       lr("v_lr"), wf["o"], self.o_lr, wf["do"], lr("do_lr"),
                                       self.lse, wf["dq"], wf["dk"], wf["dv"], self.dq_lr,
                                       self.dk_lr, self.dv_lr, self.aws), "attention backward")
        if ev is not None:
            ev[1].record(torch.cuda.current_stream())
        _chk(p.unpermute_rope_bwd(wf["dq"], self.dq_hr), "dq")
        _chk(p.unpermute_rope_bwd(wf["dk"], self.dk_hr), "dk")
        if not self.vo_raster:
            _chk(p.unpermute(wf["dv"], self.dv_hr), "dv")
        if L:
            _chk(p.rope_2d_bwd(self.dq_lr, self.dq_lr, ug.UG_LR), "dq_lr")
            _chk(p.rope_2d_bwd(self.dk_lr, self.dk_lr, ug.UG_LR), "dk_lr")


def backward_record(args, wl, d, fwd, dev, stream, rank, local, steps=None):
    """Times the layer's backward on inputs d (adds seeded dO) with the
    forward runner's outputs and lse; returns a record dict."""
    d = dict(d)
    d.update(workloads.make_grad_outputs(wl, seed=rank + 1, device=dev))
    fwd.step()
    br = BackwardRunner(wl, d, fwd.plan, fwd.o_hr, fwd.o_lr, fwd.lse, dev)
    steps = steps or args.steps
    flush = 0 if fwd.hr_bytes > L2_BYTES else 2 * L2_BYTES
    sec, attn, clk, dist = time_steps(br.step, steps, max(3, min(args.warmup, 5)), dev, stream, rank,
                                local, flush)
    _chk(fwd.plan.check_error(), "backward timed steps")
    ach = br.flops / attn / 1e12
    return {
        "metric": "useful attention-backward TFLOP/s & ms per layer backward",
        "workload": wl.name, "steps": steps, "ms_per_layer_backward": sec * 1e3,
        "layer_backward_tflops": br.flops / sec / 1e12, "attn_bwd_ms": attn * 1e3,
        "attn_bwd_tflops": ach, "useful_flop_per_backward": br.flops,
        "gpu_launches_per_step": br.launches,
        "roofline": tensor_roofline(ach, sec * steps, clk,
                                    note="7 products executed per visible pair, 5 counted"),
        "clocks": clk,
        "per_step_ms": dist,
    }


def run_backward(args, wl, world, rank, local):
    """--op backward: the layer's backward pass alone, with its own end to
    end through ug_layer_bwd and a CPU-oracle baseline."""
    from block_sparse_local_raster_b200 import ug
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    init_dist("nccl", world)
    stream = torch.cuda.current_stream(dev)
    x = workloads.make_inputs(wl, seed=rank)
    x.pop("head_scale", None)
    x.update(workloads.make_grad_outputs(wl, seed=rank + 1))
    d = {k: v.to(dev) for k, v in x.items()}
    L = wl.n_lr
    lr = lambda n: d[n] if L else None
    fwd = LayerRunner(wl, d, dev, stream)
    fwd.step()
    br = BackwardRunner(wl, d, fwd.plan, fwd.o_hr, fwd.o_lr, fwd.lse, dev)
    flush = 0 if fwd.hr_bytes > L2_BYTES else 2 * L2_BYTES
    sec, attn, clk, dist = time_steps(br.step, args.steps, args.warmup, dev, stream, rank, local, flush)
    plan, o_hr, o_lr, lse = fwd.plan, fwd.o_hr, fwd.o_lr, fwd.lse
    _chk(plan.check_error(), "timed steps")
    # end to end: inputs (q, k, v, o, lse, do) from pinned host memory, the
    # gradients back to pinned host memory, through ug_layer_bwd
    ws = torch.empty(plan.layer_bwd_workspace_bytes(), dtype=torch.uint8, device=dev)
    host_in = {k: v.pin_memory() for k, v in x.items()}
    host_in["o_hr"], host_in["lse"] = o_hr.cpu().pin_memory(), lse.cpu().pin_memory()
    if L:
        host_in["o_lr"] = o_lr.cpu().pin_memory()
    dev_in = {"o_hr": o_hr, "lse": lse, **({"o_lr": o_lr} if L else {}), **d}
    grads = [t for t in (br.dq_hr, br.dk_hr, br.dv_hr, br.dq_lr, br.dk_lr, br.dv_lr)
             if t is not None]
    host_out = [torch.empty_like(t, device="cpu").pin_memory() for t in grads]
    e2e_steps = max(3, min(args.e2e_steps, args.steps))
    torch.cuda.synchronize(dev)
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a0.record(stream)
    for _ in range(e2e_steps):
        for k, v in host_in.items():
            dev_in[k].copy_(v, non_blocking=True)
        _chk(plan.layer_bwd(d["q_hr"], d["k_hr"], d["v_hr"], lr("q_lr"), lr("k_lr"), lr("v_lr"),
                            o_hr, o_lr, lse, d["do_hr"], lr("do_lr"), br.dq_hr, br.dk_hr,
                            br.dv_hr, br.dq_lr, br.dk_lr, br.dv_lr, ws, stream), "ug_layer_bwd")
        for h, t in zip(host_out, grads):
            h.copy_(t, non_blocking=True)
    a1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_sec = reduce_max(a0.elapsed_time(a1) / 1e3 / e2e_steps, dev)
    flops = br.flops
    if rank == 0:
        ach = flops / attn / 1e12
        line = {
            "metric": "useful attention-backward TFLOP/s & ms per layer backward", "op": "backward",
            "value": aggregate(flops, world, sec) / 1e12, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": wl.name, "useful_flop_per_backward": flops,
                       "l2": ("inputs larger than L2 (each high-res tensor %.0f MB), no flush"
                              if not flush else
                              "inputs smaller than L2 (%.0f MB per high-res tensor), flushed "
                              "between steps") % (d["q_hr"].numel() * 2 / 1e6)},
            "attn_bwd_ms": attn * 1e3, "attn_bwd_tflops": ach, "per_step_ms": dist,
            "roofline": tensor_roofline(ach, sec * args.steps, clk,
                                        note="7 products executed per visible pair, 5 counted"),
            "e2e": {"value": aggregate(flops, world, e2e_sec) / 1e12, "unit": "TFLOP/s",
                    "h2d_bytes_per_step": sum(v.numel() * v.element_size()
                                              for v in host_in.values()),
                    "d2h_bytes_per_step": sum(t.numel() * t.element_size() for t in grads)},
            "gpu_launches": br.launches * args.steps, "clocks": clk,
        }
        if not args.no_cpu_baseline and world == 1:
            line["cpu_baseline"] = backward_cpu_baseline(wl, x)
        print(json.dumps(line), flush=True)
    fwd.close()
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def backward_cpu_baseline(wl, x):
    """The oracle's attention backward, as it stands, on a bounded sample:
    dQ of 16 high-res and 4 global query rows of head 0 (each row's full
    softmax over every key it sees), rotated q/k recomputed.  Useful FLOPs of
    the sample: 2.5 x 4 d x (visible keys of the sampled rows)."""
    from oracle import hier_local_attn as O
    g = O.Geometry.from_dict(dict(wl.geom_dict(), heads=1))
    bits = {k: v[:, :, :1].contiguous().view(torch.int16).numpy().view(np.uint16)
            for k, v in x.items()}
    rng = np.random.default_rng(0)
    rows = np.sort(np.concatenate([rng.choice(g.N, 16, replace=False),
                                   g.N + rng.choice(g.L, 4, replace=False) if g.L else []])
                   ).astype(np.int64)
    vis = int(sum(O.visibility(g, O.HR_RASTER, rows[i:i + 1]).sum() for i in range(rows.size)))
    c0 = time.perf_counter()
    O.layer_backward(bits, bits, g, rows=rows, keys=np.zeros(0, dtype=np.int64))
    cdt = time.perf_counter() - c0
    flops = 2.5 * 4 * g.head_dim * vis
    return {"value": flops / cdt / 1e12, "unit": "TFLOP/s", "cores": cpu_threads(), "nproc": cpu_cores(),
            "kind": "oracle",
            "sample": (f"dq of {rows.size} query rows x 1 head of the {wl.name} layer backward "
                       f"(RoPE of every key included), fp64 numpy, {cdt:.1f} s")}


def run_warm_start(args, world, rank, local):
    """The warm-start kernel on the latent of the --config image size.
    Algorithmic bytes per launch: the low-res latent read once, the noise
    read once and the state written once (fp32).  The timed launches rotate
    over enough noise/output buffers to exceed L2."""
    from block_sparse_local_raster_b200 import ug
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    init_dist("nccl", world)
    stream = torch.cuda.current_stream(dev)
    ws = workloads.WARM_START[args.config]
    host = workloads.make_warm_start_inputs(ws, seed=rank)
    lr = host["x_lr"].to(dev)
    hr_bytes = host["noise"].numel() * 4
    nbuf = max(2, -(-3 * L2_BYTES // (2 * hr_bytes)))
    noise = [host["noise"].to(dev) for _ in range(nbuf)]
    outs = [torch.empty_like(noise[0]) for _ in range(nbuf)]
    algo = lr.numel() * 4 + 2 * hr_bytes

    def launch(i):
        st = ug.warm_start_raw(lr, noise[i % nbuf], outs[i % nbuf], ws.scale, ws.sharpen, ws.t,
                               stream)
        if st != ug.UG_OK:
            raise ug.UgError(st, "ug_warm_start")

    clocks = ClockSampler(local)
    clocks.start()
    for i in range(args.warmup):
        launch(i)
    torch.cuda.synchronize(dev)
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    h0 = time.perf_counter()
    e0.record(stream)
    for i in range(args.steps):
        launch(i)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    h1 = time.perf_counter()
    barrier()
    clk = clocks.stop(h0, h1)
    sec = reduce_max(e0.elapsed_time(e1) / 1e3 / args.steps, dev)
    # end to end: pinned host buffers in, result out, every step
    pin_lr, pin_noise = host["x_lr"].pin_memory(), host["noise"].pin_memory()
    pin_out = torch.empty_like(pin_noise).pin_memory()
    e2e_steps = max(3, min(args.e2e_steps, args.steps))
    torch.cuda.synchronize(dev)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(e2e_steps):
        lr.copy_(pin_lr, non_blocking=True)
        noise[0].copy_(pin_noise, non_blocking=True)
        launch(0)
        pin_out.copy_(outs[0], non_blocking=True)
    t1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_sec = reduce_max(t0.elapsed_time(t1) / 1e3 / e2e_steps, dev)
    pk, src = peaks()
    if rank == 0:
        gbs = algo / sec / 1e9
        line = {
            "metric": "warm-start initialisation HBM throughput", "op": "warm_start",
            "value": aggregate(algo, world, sec) / 1e9, "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": {"workload": f"warm-start {ws.name}: [{ws.batch},{ws.channels},"
                                   f"{ws.lr_h},{ws.lr_w}] x{ws.scale}, sharpen {ws.sharpen}, "
                                   f"t {ws.t}", "l2": f"rotating {nbuf} buffer pairs > L2"},
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / pk["hbm_gbs"], "traffic": None, "peak_source": src,
                         "algorithmic_bytes_per_launch": algo},
            "e2e": {"value": aggregate(algo, world, e2e_sec) / 1e9, "unit": "GB/s",
                    "h2d_bytes_per_step": lr.numel() * 4 + hr_bytes,
                    "d2h_bytes_per_step": hr_bytes},
            "gpu_launches": args.steps, "clocks": clk,
        }
        if not args.no_cpu_baseline:
            from oracle import warm_start as W
            one = (slice(0, 1), slice(0, 1))
            xs, ns = host["x_lr"][one].double().numpy(), host["noise"][one].double().numpy()
            c0 = time.perf_counter()
            W.warm_start(xs, ns, ws.scale, ws.sharpen, ws.t)
            cdt = time.perf_counter() - c0
            b1 = (xs.size + 2 * ns.size) * 4
            line["cpu_baseline"] = {"value": b1 / cdt / 1e9, "unit": "GB/s", "cores": cpu_threads(), "nproc": cpu_cores(),
                                    "kind": "oracle",
                                    "sample": f"one plane of the latent, fp64 numpy, {cdt:.2f} s"}
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def main():
    args = parse()
    world, rank, local = dist_env()
    if args.gpus != world and world > 1:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE {world}")
    if args.op == "warm_start":
        if args.impl == "reference":
            raise SystemExit("--op warm_start times the library only")
        run_warm_start(args, world, rank, local)
        return
    if args.op == "backward":
        if args.impl == "reference":
            raise SystemExit("--op backward times the library only")
        run_backward(args, workloads.get(args.config), world, rank, local)
        return
    wl = workloads.get(args.config)
    if args.impl == "reference":
        run_reference(args, wl, world, rank)
        return
    run_ug(args, wl, world, rank, local)


if __name__ == "__main__":
    main()
