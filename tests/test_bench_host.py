"""Host-side arithmetic of bench.py (no GPU): the algorithmic work per kernel, the
roofline entry and the captured-traffic lookup.

The algorithmic counts follow the layer's definition ("HASTE: Hardware-Aware
Dynamic Sparse Training for Large Output Spaces", summary page, Methodology 1):
the forward, dW and dX products of the tail each take 2*B*L*k flops, and the
compulsory HBM bytes of a fused step are W read once and dW written once plus
the group indices, X, dX and the targets.
"""
import os

import pytest

import bench
from structured_sparse_output_b200 import inputs as I


def test_algorithmic_work_of_the_fused_step():
    wl = I.WORKLOADS["670k"]
    B, L, k, d, n_g = wl.B, wl.L, wl.k, wl.d, wl.n_groups
    work = bench.algorithmic(wl)
    assert work["tail"][0] == 6.0 * B * L * k
    assert work["tail_step"][0] + work["tail_dx"][0] == work["tail"][0]
    w = L * k * 2                      # bf16 weights
    tgt = 4 * (B + 1 + B * wl.positives)
    assert work["tail"][1] == 2 * w + 4 * n_g * k + B * d * 2 + B * d * 4 + tgt
    assert work["tail_dx"][1] == w + 4 * n_g * k + B * d * 4
    # the head's three products, 2*B*H*d flops each
    for key in ("head_forward", "head_dw", "head_dx"):
        assert work[key][0] == 2.0 * B * wl.H * d


def test_algorithmic_work_of_the_given_gradient_workloads():
    wl = I.WORKLOADS["sweep32"]
    B, L, k = wl.B, wl.L, wl.k
    work = bench.algorithmic(wl)
    for key in ("tail_forward", "tail_dw", "tail_dx"):
        assert work[key][0] == 2.0 * B * L * k
    dy = B * L * 2
    assert work["tail_dx"][1] == dy + L * k * 2 + 4 * wl.n_groups * k + B * wl.d * 4


def test_roofline_picks_the_slower_bound():
    peaks = {"hbm_gbs": 6000.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}
    # 1.4 TFLOP in 2 ms: tensor-bound (1 ms of MMA against 0.17 ms of HBM)
    r = bench.roofline_of(1.4e12, 1e9, 2.0, peaks)
    assert r["bound"] == "tensor" and r["peak"] == 1400.0
    assert r["achieved"] == pytest.approx(700.0) and r["frac"] == pytest.approx(0.5)
    # burst peak when asked
    assert bench.roofline_of(1.4e12, 1e9, 2.0, peaks, sustained=False)["peak"] == 1600.0
    # 12 GB in 4 ms: HBM-bound
    r = bench.roofline_of(1e9, 12e9, 4.0, peaks)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["achieved"] == pytest.approx(3000.0) and r["frac"] == pytest.approx(0.5)


def test_traffic_is_reported_only_for_the_captured_source(monkeypatch):
    digest = bench.source_digest("tail_step")
    assert digest is not None and len(digest) == 16
    monkeypatch.setattr(bench, "TRAFFIC", {("670k", "tail_step"): (123e6, digest)})
    got, src = bench.traffic_of("670k", "tail_step")
    assert got == 123e6 and src == "ncu capture of k_step2 at 670k"
    # a capture taken on another version of the kernel's source is not reported
    monkeypatch.setattr(bench, "TRAFFIC", {("670k", "tail_step"): (123e6, "0" * 16)})
    got, src = bench.traffic_of("670k", "tail_step")
    assert got is None and "changed" in src
    # nothing captured for this workload or kernel
    assert bench.traffic_of("8.6m", "tail_step")[0] is None
    assert bench.traffic_of("670k", "head_dx")[0] is None


def test_every_timed_kernel_has_a_source_file():
    for kernel, (src, name) in bench.KERNELS.items():
        assert os.path.exists(os.path.join(bench.CSRC, src)), kernel
        with open(os.path.join(bench.CSRC, src)) as fh:
            assert name in fh.read(), (kernel, name)


def test_peak_choice_follows_the_timed_region():
    # kernels timed inside a short region run at the burst rate, long ones at the
    # sustained (power-capped) rate
    assert not bench.use_sustained(140.0)
    assert bench.use_sustained(bench.SUSTAINED_AFTER_S * 1e3)


def test_job_value_counts_every_rank():
    assert bench.job_value(4, 256, 100, 50.0) == pytest.approx(4 * 256 * 100 / 0.05)
