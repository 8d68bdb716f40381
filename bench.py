#!/usr/bin/env python
"""Benchmark of the HASTE group-shared fixed fan-in output layer on B200.

A step is one pass of the whole hot path over one batch of synthetic input:
the dense head (forward with the BCE gradient, dWh, dXh) and the fused sparse-tail
training step (gather-once forward, BCE-with-logits gradient, dW, dX), all through
the C ABI of libhaste.so.  The fan-in plan is built once (it belongs to the
sparsity pattern, not to the batch) and stays outside the timed region.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config 670k] [--impl reference]
                  [--more 8.6m,3m,sweep16,sweep32,sweep64]

Headline workload: the 670K-label tail (B=256, d=768, L=670,208 in groups of
G=32, k=128, bf16, 4,096 head labels, 5 Zipf(1.0) positives per sample).  Other
workloads: 8.6m, 3m, sweep16/32/64 (forward + dW + dX with a given gradient),
tiny.  A single-GPU run also measures the workloads listed by --more (default:
the 8.6M and 3M steps and the three group sizes of the sweep) and reports them
under "configs" in the same line.  Multi-GPU (torchrun) runs one independent
replica of the layer per rank on its own batch (weak scaling, no collective on
the data path); the timing is the max over ranks.  Prints one JSON line on
rank 0.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "sparse-tail fwd+bwd samples/s at 670K–8.6M labels; % of B200 roofline"
UNIT = "samples/s"


# ----------------------------------------------------------------- helpers
def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            m = json.load(fh)
        return {"hbm_gbs": m["hbm_gbs"], "bf16_tflops": m["bf16_tflops"],
                "bf16_tflops_sustained": m.get("bf16_tflops_sustained", m["bf16_tflops"]), "src": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "src": "fallback"}


def algorithmic(wl):
    """Algorithmic flops and HBM bytes per launch of each kernel, and of the tail.

    Tail (per step): forward, dW and dX products 2*B*L*k flops each; compulsory
    bytes W (read) + dW (write) + group indices + X + dX + targets; the
    given-gradient workloads add the logits write and two reads of dY.
    """
    e = 2 if wl.dtype == "bf16" else 4
    B, L, k, d, n_g = wl.B, wl.L, wl.k, wl.d, wl.n_groups
    w = L * k * e
    idx = 4 * n_g * k
    x = B * d * e
    dx = B * d * 4
    tgt = 4 * (B + 1 + B * max(1, wl.positives))
    out = {}
    if wl.fused:
        out["tail_step"] = (4.0 * B * L * k, w + w + idx + x + tgt)      # forward + dW
        out["tail_dx"] = (2.0 * B * L * k, w + idx + dx)
        out["tail"] = (6.0 * B * L * k, 2 * w + idx + x + dx + tgt)
        if wl.H:
            out["head_forward"] = (2.0 * B * wl.H * d, B * d * e + wl.H * d * e + B * wl.H * e)
            out["head_dw"] = (2.0 * B * wl.H * d, B * wl.H * e + B * d * e + wl.H * d * e)
            out["head_dx"] = (2.0 * B * wl.H * d, B * wl.H * e + wl.H * d * e + dx)
    else:
        dy = B * L * e
        out["tail_forward"] = (2.0 * B * L * k, w + idx + x + B * L * e)
        out["tail_dw"] = (2.0 * B * L * k, dy + x + idx + w)
        out["tail_dx"] = (2.0 * B * L * k, dy + w + idx + dx)
        out["tail"] = (6.0 * B * L * k, 3 * w + 2 * dy + B * L * e + 3 * idx + 2 * x + dx)
    return out


# DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) of a
# kernel from one ncu capture (summaries under profiles/), valid only for the
# source file it was taken on: (config, timed region) -> (bytes, source digest).
TRAFFIC = {
    ("670k", "tail_step"): (649.0e6, "805dcd6d8ba19d47"),
    ("670k", "tail_dx"): (538.5e6, "09ba676f0abb371c"),
    ("8.6m", "tail_step"): (8.84e9, "805dcd6d8ba19d47"),
    ("8.6m", "tail_dx"): (7.01e9, "09ba676f0abb371c"),
    ("670k", "topk_score"): (187.0e6, "48974329ba8749cd"),
}
# timed region -> (source file under csrc/, kernel name in the ncu summaries)
KERNELS = {"tail_step": ("tail_v2.cu", "k_step2"), "tail_dx": ("dx_band.cu", "k_dx_band"),
           "topk_score": ("topk.cu", "k_topk")}
CSRC = os.path.join(ROOT, "structured_sparse_output_b200", "csrc")


def source_digest(kernel):
    import hashlib
    src = os.path.join(CSRC, KERNELS[kernel][0])
    if not os.path.exists(src):
        return None
    with open(src, "rb") as fh:
        return hashlib.sha256(fh.read()).hexdigest()[:16]


def traffic_of(config, kernel):
    """(bytes, where from): the captured traffic, or None when the kernel's source
    changed since the capture (or it was never captured)."""
    got = TRAFFIC.get((config, kernel))
    if got is None or kernel not in KERNELS:
        return None, "no capture of this kernel"
    if source_digest(kernel) != got[1]:
        return None, "kernel source changed since the capture"
    return got[0], f"ncu capture of {KERNELS[kernel][1]} at {config}"


# A kernel timed inside a region shorter than this runs at the burst MMA rate;
# longer regions settle at the sustained (power-capped) rate.
SUSTAINED_AFTER_S = 2.0


def use_sustained(region_ms):
    return region_ms / 1e3 >= SUSTAINED_AFTER_S


def roofline_of(flops, nbytes, ms, peaks, sustained=True):
    tf = peaks["bf16_tflops_sustained" if sustained else "bf16_tflops"]
    t_tensor = flops / (tf * 1e12)
    t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
    s = ms / 1e3
    if t_tensor >= t_hbm:
        ach = flops / s / 1e12
        return {"bound": "tensor", "achieved": round(ach, 2), "peak": tf, "unit": "TFLOP/s",
                "frac": round(ach / tf, 4)}
    ach = nbytes / s / 1e9
    return {"bound": "hbm", "achieved": round(ach, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": round(ach / peaks["hbm_gbs"], 4)}


class Clocks:
    """nvidia-smi sampling of SM clocks and throttle reasons around a region."""
    Q = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.p = None
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                       "-lms", "50", "-i", uuid], stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None
        self.marks = []

    def mark(self):
        self.marks.append(time.time())

    def stop(self):
        if self.p is not None:
            time.sleep(0.12)
            self.p.terminate()
            try:
                self.p.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.p.kill()
        self.f.flush()
        self.f.seek(0)
        rows = [r.split(", ") for r in self.f.read().strip().splitlines() if r.count(",") >= 8]
        os.unlink(self.f.name)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        sm, mx, reasons, n_in = [], None, set(), 0
        t0, t1 = (self.marks + [0, 0])[:2]
        for r in rows:
            try:
                ts = time.mktime(time.strptime(r[0].split(".")[0], "%Y/%m/%d %H:%M:%S"))
            except ValueError:
                ts = None
            inside = ts is None or (t0 - 1.0 <= ts <= t1 + 1.0)
            if not inside:
                continue
            n_in += 1
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
            except ValueError:
                pass
            for i, nm in enumerate(names):
                if r[5 + i].strip().lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": n_in}


# ------------------------------------------------------------ the workload
class Runner:
    """Device-resident inputs and the step of one workload on one GPU."""

    def __init__(self, wl, seed):
        import numpy as np
        import torch
        from structured_sparse_output_b200 import haste as H
        from structured_sparse_output_b200 import inputs as I
        self.wl, self.H, self.torch = wl, H, torch
        dt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
        self.inp = I.make_inputs(wl, seed, with_dy=not wl.fused, with_head=wl.H > 0)
        inp = self.inp

        def dev(a):
            if a.dtype == np.uint16:
                return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
            return torch.from_numpy(np.ascontiguousarray(a)).cuda()

        self.dev = dev
        t0 = time.time()
        self.plan = H.haste_plan(inp.idx, wl.G, wl.d)
        self.plan_s = time.time() - t0
        self.X, self.W = dev(inp.X), dev(inp.W)
        code = H.dtype_code(self.X)
        self.ws = torch.empty(self.plan.workspace_size(wl.B, code), dtype=torch.uint8, device="cuda")
        self.dW = torch.empty_like(self.W)
        self.dX = torch.empty((wl.B, wl.d), dtype=torch.float32, device="cuda")
        self.scale = 1.0 / wl.B
        if wl.fused:
            self.tp, self.ti = dev(inp.tail_pos[0]), dev(inp.tail_pos[1])
            self.loss = torch.zeros(2, dtype=torch.float32, device="cuda")
            if wl.H:
                self.hp, self.hi = dev(inp.head_pos[0]), dev(inp.head_pos[1])
                self.Xh, self.Wh = dev(inp.Xh), dev(inp.Wh)
                self.hws = torch.empty(H.haste_head_workspace_size(wl.B, wl.H, wl.d, code), dtype=torch.uint8,
                                       device="cuda")
                self.dYh = torch.empty((wl.B, wl.H), dtype=dt, device="cuda")
                self.dWh = torch.empty_like(self.Wh)
                self.dXh = torch.empty((wl.B, wl.d), dtype=torch.float32, device="cuda")
        else:
            self.dY = dev(inp.dY)
            self.logits = torch.empty((wl.B, wl.L), dtype=dt, device="cuda")
            self.loss = torch.zeros(2, dtype=torch.float32, device="cuda")

    def step(self):
        H, wl = self.H, self.wl
        if wl.fused:
            if wl.H:
                H.haste_head_forward(self.Xh, self.Wh, self.dYh, self.hws, self.hp, self.hi, self.scale,
                                     self.loss[1:])
                H.haste_head_backward(self.Xh, self.Wh, self.dYh, self.dWh, self.dXh, self.hws)
            H.haste_bce_step(self.plan, self.X, self.W, self.tp, self.ti, self.scale, self.loss[:1], self.dW,
                             self.dX, self.ws)
        else:
            H.haste_forward(self.plan, self.X, self.W, self.logits, self.ws)
            H.haste_backward_dw(self.plan, self.X, self.dY, self.dW, self.ws)
            H.haste_backward_dx(self.plan, self.W, self.dY, self.dX, self.ws)

    # end to end: this step's inputs come from pinned host memory, its loss (or,
    # without a loss, the dX checksum element) goes back to pinned host memory
    def e2e_setup(self):
        torch, wl = self.torch, self.wl
        pin = lambda t: t.cpu().pin_memory()
        self.h_in = [(pin(t), t) for t in ([self.X, self.tp, self.ti] if wl.fused else [self.X, self.dY])]
        if wl.fused and wl.H:
            self.h_in += [(pin(t), t) for t in (self.Xh, self.hp, self.hi)]
        self.h_out = torch.zeros(2, dtype=torch.float32).pin_memory()
        self.h2d = sum(h.numel() * h.element_size() for h, _ in self.h_in)
        self.d2h = self.h_out.numel() * self.h_out.element_size()

    def e2e_step(self):
        for h, d in self.h_in:
            d.copy_(h, non_blocking=True)
        self.step()
        src = self.loss if self.wl.fused else self.dX.view(-1)[:2]
        self.h_out.copy_(src, non_blocking=True)


def max_over_ranks(ms, device):
    """The slowest rank's time: every rank contributes its own device-timed ms."""
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_value(world, batch, steps, ms):
    """Whole-job throughput: every rank runs its own replica on its own batch of
    `batch` samples (weak scaling), the job takes the slowest rank's time."""
    return world * batch * steps / (ms / 1e3)


def timed(fn, steps, warmup, dist):
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    if dist:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    if dist:
        torch.distributed.barrier()
    ms = e0.elapsed_time(e1)
    if dist:
        ms = max_over_ranks(ms, "cuda")
    return ms


def infer_topk(run, steps, warmup, peaks, K=5, kp=4):
    """Inference scoring at the same workload: the top-K tail labels per sample by
    the two-stage top-k (the top kp of each of n_buckets buckets of whole groups,
    then the top K of the survivors), device-timed; logits never reach memory.
    With one bucket per SM and kp = 4, a top-5 label is missed only when all five
    share one bucket."""
    import torch
    H, wl = run.H, run.wl
    nb = min(wl.n_groups, torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count)
    ws = torch.empty(H.haste_topk_workspace_size(run.plan, wl.B, H.HASTE_BF16, nb, kp), dtype=torch.uint8,
                     device="cuda")
    ov = torch.empty((wl.B, K), dtype=torch.float32, device="cuda")
    oi = torch.empty((wl.B, K), dtype=torch.int32, device="cuda")
    fn = lambda: H.haste_topk(run.plan, run.X, run.W, K, kp, nb, ov, oi, ws)
    H.haste_profile_start()
    ms = timed(fn, steps, warmup, False)
    prof = H.haste_profile_stop()
    n_l, t_ms = prof.get("topk_score", (1, ms))
    flops = 2.0 * wl.B * wl.L * wl.k
    nbytes = wl.L * wl.k * 2 + 4 * wl.n_groups * wl.k + wl.B * wl.d * 2
    rf = roofline_of(flops, nbytes, t_ms / max(n_l, 1), peaks, use_sustained(ms))
    rf["kernel"] = "topk_score"
    rf["traffic"], rf["traffic_src"] = traffic_of(wl.name, "topk_score")
    return {"metric": f"top-{K} tail scoring samples/s", "value": round(wl.B * steps / (ms / 1e3), 1),
            "ms_per_call": round(ms / steps, 4), "k": K, "kp": kp, "n_buckets": nb, "exact": kp >= K,
            "roofline": rf}


# ----------------------------------------------------------- CPU baseline
def oracle_step_seconds(inp, n_sub_groups):
    """Oracle time of one step on the first n_sub_groups groups (tail) plus the
    full head, and the sub-layer size."""
    import numpy as np
    from oracle import oracle as O
    wl = inp.wl
    S = min(n_sub_groups, wl.n_groups)
    Ls = S * wl.G
    idx = inp.idx[:S]
    W = inp.W[:Ls]
    t0 = time.perf_counter()
    if wl.fused:
        rp, ids = inp.tail_pos
        keep = ids < Ls
        counts = np.array([keep[rp[b]:rp[b + 1]].sum() for b in range(wl.B)])
        srp = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
        O.bce_step(inp.X, W, idx, wl.G, srp, ids[keep], 1.0 / wl.B)
    else:
        dY = inp.dY[:, :Ls]
        O.forward(inp.X, W, idx, wl.G)
        O.backward_dw(inp.X, dY, idx, wl.G)
        O.backward_dx(W, dY, idx, wl.G, wl.d)
    t_tail = time.perf_counter() - t0
    t_head = 0.0
    if wl.fused and wl.H:
        t1 = time.perf_counter()
        O.head_step(inp.Xh, inp.Wh, inp.head_pos[0], inp.head_pos[1], 1.0 / wl.B)
        t_head = time.perf_counter() - t1
    return t_tail, t_head, S


def cpu_baseline(inp, budget_s):
    """Oracle samples/s on a bounded sample of the workload, scaled to the whole
    layer by its group count."""
    wl = inp.wl
    t_tail, t_head, S = oracle_step_seconds(inp, 16)
    S2 = int(max(16, min(wl.n_groups, 16 * max(1.0, (budget_s - t_head) / max(t_tail, 1e-3)))))
    t_tail, t_head, S2 = oracle_step_seconds(inp, S2)
    est = t_tail * wl.n_groups / S2 + t_head
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    return {"value": round(wl.B / est, 3), "unit": UNIT, "cores": int(os.environ.get("OMP_NUM_THREADS", cores)),
            "kind": "oracle",
            "sample": (f"fp64 oracle on the first {S2} of {wl.n_groups} groups "
                       f"({t_tail:.1f} s, scaled by {wl.n_groups / S2:.1f}x)"
                       + (f" + the full head ({t_head:.1f} s)" if t_head else "") + f", B={wl.B}")}


def config_of(wl, l2_note):
    c = {"workload": wl.name, "B": wl.B, "d": wl.d, "L": wl.L, "G": wl.G, "k": wl.k, "n_groups": wl.n_groups}
    if wl.fused:
        c.update({"H": wl.H, "positives": wl.positives, "zipf_alpha": wl.alpha,
                  "step": "head fwd+BCE+bwd, tail fused fwd+BCE+dW+dX"})
    else:
        c["step"] = "tail forward + dW + dX with a given upstream gradient"
    c["l2"] = l2_note
    return c


def l2_note(wl, dtype):
    wb = wl.L * wl.k * (2 if dtype == "bf16" else 4) / 1e6
    return (f"inputs larger than L2: W {wb:.0f} MB read and dW written every step (L2 126 MB)")


def est_ms(run):
    """One untimed step, timed roughly on the device: sizes the timed region."""
    import torch
    run.step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    run.step()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1)


def sgd_variant(run, steps, warmup, peaks, lr=1e-3, momentum=0.9):
    """The fused tail step with the SGD-with-momentum update in the step kernel
    (haste_bce_step_sgd), alternating two weight buffers, device-timed.  W' and
    the momentum replace the dW write: the step's compulsory bytes become W read,
    W' written, momentum read and written."""
    import torch
    H, wl = run.H, run.wl
    bufs = [run.W.clone(), torch.empty_like(run.W)]
    M = torch.zeros_like(run.W)
    state = {"i": 0}

    def fn():
        i = state["i"]
        H.haste_bce_step_sgd(run.plan, run.X, bufs[i % 2], run.tp, run.ti, run.scale, run.loss[:1], lr, momentum,
                             M, bufs[(i + 1) % 2], run.dX, run.ws)
        state["i"] = i + 1

    for _ in range(warmup):  # outside the profile: its per-step sums cover the timed steps only
        fn()
    torch.cuda.synchronize()
    H.haste_profile_start()
    ms = timed(fn, steps, 0, False)
    prof = H.haste_profile_stop()
    if H.haste_device_status() != H.HASTE_OK:
        raise SystemExit("device error word set during the fused-update timing")
    tail_ms = sum(t for k, (n, t) in prof.items() if k.startswith("tail") or k in ("xt", "dx_reduce")) / steps
    n_l, t_step = prof.get("tail_step", (1, 0.0))
    e = 2
    w = wl.L * wl.k * e
    nbytes = 4 * w + 4 * wl.n_groups * wl.k + wl.B * wl.d * e      # W, W', momentum in and out, idx, X
    rf = roofline_of(4.0 * wl.B * wl.L * wl.k, nbytes, t_step / max(n_l, 1), peaks, use_sustained(ms))
    rf["kernel"] = "tail_step"
    del bufs, M
    return {"call": "haste_bce_step_sgd", "lr": lr, "momentum": momentum, "steps": steps,
            "tail_ms_per_step": round(tail_ms, 4), "samples_per_s": round(wl.B / (tail_ms / 1e3), 1),
            "step_kernel_ms": round(t_step / max(n_l, 1), 4), "roofline": rf}


def replan_timing(run, frac=0.01, reps=5):
    """Device re-plan after rewiring a fraction of the groups (haste_plan_update):
    the changed rows are copied to the device and the inverse map is rebuilt
    there.  The new rows are other groups' rows (valid sets), so the timing sees
    a real rebuild.  Device-timed with CUDA events around the call, H2D included."""
    import numpy as np
    import torch
    wl, plan = run.wl, run.plan
    rng = np.random.default_rng(1)
    n = max(1, int(frac * wl.n_groups))
    groups = np.sort(rng.choice(wl.n_groups, n, replace=False)).astype(np.int32)
    rows = run.inp.idx[rng.permutation(groups)]
    times = []
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record()
        plan.update(groups, rows)
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
        plan.update(groups, run.inp.idx[groups])          # back to the original sets
        torch.cuda.synchronize()
    return {"call": "haste_plan_update", "groups_changed": n, "ms": round(statistics.median(times), 4),
            "full_plan_build_s": round(run.plan_s, 3)}


def measure(run, steps, warmup, dist, peaks):
    """Device-timed steps of one workload with the per-kernel profile, the
    dominant kernel's roofline, the whole tail's roofline and the clocks seen."""
    import torch
    H, wl = run.H, run.wl
    uuid = "GPU-" + str(torch.cuda.get_device_properties(torch.cuda.current_device()).uuid)
    clk = Clocks(uuid)
    time.sleep(0.2)
    for _ in range(warmup):
        run.step()
    torch.cuda.synchronize()
    H.haste_profile_start()
    clk.mark()
    ms = timed(run.step, steps, 0, dist)
    clk.mark()
    prof = H.haste_profile_stop()
    clocks = clk.stop()
    if H.haste_device_status() != H.HASTE_OK:
        raise SystemExit("device error word set during the timed region")
    sustained = use_sustained(ms)
    work = algorithmic(wl)
    dom = max((k for k in prof if k in work), key=lambda k: prof[k][1])
    n_l, tot_ms = prof[dom]
    rf = roofline_of(work[dom][0], work[dom][1], tot_ms / n_l, peaks, sustained)
    rf["kernel"] = dom
    rf["ms_per_launch"] = round(tot_ms / n_l, 4)
    rf["peak_src"] = (f"{peaks['src']} ({('sustained' if sustained else 'burst') if rf['bound'] == 'tensor' else 'copy'}"
                      f"; timed region {ms / 1e3:.2f} s)")
    rf["traffic"], rf["traffic_src"] = traffic_of(wl.name, dom)
    tail_ms = sum(prof[k][1] for k in prof if k.startswith("tail") or k in ("xt", "dx_reduce")) / steps
    tail_rf = roofline_of(work["tail"][0], work["tail"][1], tail_ms, peaks, sustained)
    total = sum(x[1] for x in prof.values())
    return {"ms": ms, "prof": prof, "clocks": clocks, "roofline": rf,
            "tail": {"ms_per_step": round(tail_ms, 4), "samples_per_s": round(wl.B / (tail_ms / 1e3), 1),
                     "roofline": tail_rf},
            "kernels": {k: {"launches": n, "ms_per_launch": round(t / n, 4), "share": round(t / total, 4)}
                        for k, (n, t) in prof.items()},
            "launches": sum(n for n, _ in prof.values())}


# -------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", default="670k")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget-s", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--more", default="8.6m,3m,sweep16,sweep32,sweep64",
                    help="further workloads measured after the headline one (single GPU only; '' for none)")
    ap.add_argument("--more-budget-ms", type=float, default=400.0, help="timed device time per further workload")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)

    from structured_sparse_output_b200 import inputs as I
    wl = I.WORKLOADS[args.config]
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dtype = "bf16" if wl.dtype == "bf16" else "f32"

    if args.impl == "reference":
        # the oracle on the host cores, rank 0 only
        if rank != 0:
            return
        inp = I.make_inputs(wl, 0, with_dy=not wl.fused, with_head=wl.H > 0)
        per_step_budget = max(0.2, 150.0 / (args.steps + args.warmup))
        t_tail, t_head, S = oracle_step_seconds(inp, 8)
        S = int(max(8, min(wl.n_groups, 8 * max(1.0, (per_step_budget - t_head) / max(t_tail, 1e-3)))))
        for _ in range(args.warmup):
            oracle_step_seconds(inp, S)
        tot = 0.0
        for _ in range(args.steps):
            t_tail, t_head, S = oracle_step_seconds(inp, S)
            tot += t_tail * wl.n_groups / S + t_head
        ms = tot / args.steps * 1e3
        value = wl.B / (ms / 1e3)
        cores = len(os.sched_getaffinity(0))
        line = {"impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3), "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": config_of(wl, "host run"),
                "cpu_baseline": {"value": round(value, 3), "unit": UNIT, "cores": cores, "kind": "oracle",
                                 "sample": f"each step: fp64 oracle on the first {S} of {wl.n_groups} groups, "
                                           f"scaled by {wl.n_groups / S:.1f}x" + (" + the full head" if wl.H else "")},
                "e2e": {"value": round(value, 3), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    import torch
    dist = world > 1
    if dist:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    else:
        torch.cuda.set_device(0)
    from structured_sparse_output_b200 import haste as H
    H.lib()
    peaks = _peaks()
    run = Runner(wl, seed=rank)       # each rank: its own batch, its own replica

    res = measure(run, args.steps, args.warmup, dist, peaks)
    ms, prof, clocks = res["ms"], res["prof"], res["clocks"]

    # end to end through the public API with host buffers
    run.e2e_setup()
    ms_e2e = timed(run.e2e_step, args.steps, args.warmup, dist)

    inference = infer_topk(run, args.steps, args.warmup, peaks) if wl.dtype == "bf16" and wl.B <= 256 else None

    value = job_value(world, wl.B, args.steps, ms)
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": dtype, "data": "synthetic",
        "config": config_of(wl, l2_note(wl, dtype)),
        "roofline": res["roofline"],
        "tail": res["tail"],
        "kernels": res["kernels"],
        "e2e": {"value": round(job_value(world, wl.B, args.steps, ms_e2e), 1), "unit": UNIT,
                "h2d_bytes_per_step": run.h2d, "d2h_bytes_per_step": run.d2h},
        "gpu_launches": res["launches"],
        "clocks": clocks,
        "plan_build_s": round(run.plan_s, 3),
        "inference": inference,
        "index_bytes": run.plan.info()[0],
    }
    if wl.fused and wl.dtype == "bf16" and wl.B <= 256:
        line["fused_update"] = sgd_variant(run, args.steps, args.warmup, peaks)
        line["replan"] = replan_timing(run)
    inp = run.inp
    if world == 1 and args.more:
        line["configs"] = {}
        del run
        torch.cuda.empty_cache()
        for name in [c for c in args.more.split(",") if c and c != args.config]:
            wlx = I.WORKLOADS[name]
            rx = Runner(wlx, seed=rank)
            steps = max(5, min(args.steps, int(round(args.more_budget_ms / max(est_ms(rx), 1e-3)))))
            rr = measure(rx, steps, args.warmup, False, peaks)
            line["configs"][name] = {
                "config": config_of(wlx, l2_note(wlx, dtype)), "steps": steps,
                "ms_per_step": round(rr["ms"] / steps, 4),
                "samples_per_s": round(wlx.B * steps / (rr["ms"] / 1e3), 1),
                "roofline": rr["roofline"], "tail": rr["tail"], "kernels": rr["kernels"],
                "gpu_launches": rr["launches"], "clocks": rr["clocks"], "plan_build_s": round(rx.plan_s, 3),
                "index_bytes": rx.plan.info()[0]}
            if wlx.fused and wlx.dtype == "bf16" and wlx.B <= 256:
                line["configs"][name]["fused_update"] = sgd_variant(rx, steps, args.warmup, peaks)
                line["configs"][name]["replan"] = replan_timing(rx)
            rx.plan.close()
            del rx
            torch.cuda.empty_cache()
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(inp, args.cpu_budget_s)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
