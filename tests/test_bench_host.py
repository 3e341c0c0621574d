"""Host arithmetic of bench.py, on the CPU: the algorithmic work behind every
reported fraction, against closed forms written out here, and the roofline
entry's use of the burst peak.

Per token and head the layer's contractions are ("大块测试时训练（LaCT）技术解析"
§2.1 eqs. 2, 4-5): the apply z = [W1; W3] q^ (4 d dh) and W2 h (2 d dh); the
keys' forward [W1; W3] k^ (4 d dh) and W2^T v (2 d dh); the three gradients
(6 d dh) -- 18 d dh on a causal sequence.  Muon adds five Newton-Schulz steps
per matrix and chunk (§2.2.1 eqs. 9-10): with m = min(d, dh), p = max(d, dh),
the Gram X^T X (2 m^2 p), its square (2 m^3) and the update X B (2 m^2 p).
"""
import json

import pytest

import bench
from lact_inputs import APPLY_THEN_UPDATE, BF16, F32, RULE_GD, RULE_MOMENTUM, RULE_MUON, WORKLOADS, Workload


@pytest.mark.parametrize("idx", sorted(WORKLOADS))
def test_forward_flops_are_the_layer_contractions(idx):
    w = WORKLOADS[idx]
    BH = w.B * w.H
    want = BH * (12.0 * w.d * w.dh * w.T + 6.0 * w.d * w.dh * w.Tq)
    if w.rule == RULE_MUON:
        m, p = min(w.d, w.dh), max(w.d, w.dh)
        want += BH * w.n_chunks * 3 * 5 * (2 * m * m * p + 2 * m ** 3 + 2 * m * m * p)
    assert bench.step_flops(w) == pytest.approx(want, rel=1e-12)


def test_headline_flops_match_the_published_totals():
    """The per-configuration totals the fractions are taken of (the LM 760M
    shape: 18 d dh per token per head over 65,536 tokens and 6 heads)."""
    assert bench.step_flops(WORKLOADS[2]) == pytest.approx(2 * 6 * 32768 * 18 * 256 * 512, rel=1e-12)
    assert bench.step_flops(WORKLOADS[2]) == pytest.approx(9.28e11, rel=2e-3)
    assert bench.step_flops(WORKLOADS[3]) == pytest.approx(1.39e12, rel=3e-3)
    assert bench.step_flops(WORKLOADS[4]) == pytest.approx(1.94e12, rel=3e-3)
    assert bench.step_flops(WORKLOADS[5]) == pytest.approx(2.34e11, rel=3e-3)


@pytest.mark.parametrize("idx", [2, 3, 5])
def test_kernel_work_adds_up_to_the_step(idx):
    """The per-kernel FLOPs the roofline entries use cover the step exactly:
    key forward + gradient (or the fused key-gradient kernel) + apply."""
    w = WORKLOADS[idx]
    work = bench.kernel_work(w)
    keys = work["key_grad_umma"][1] if idx == 5 else work["fwd_key_umma"][1] + work["grad_umma"][1]
    assert keys + work["apply_fused_umma"][1] == pytest.approx(bench.step_flops(w), rel=1e-12)
    assert work["fwd_query_umma"][1] + work["apply_out_umma"][1] == pytest.approx(work["apply_fused_umma"][1])


def test_backward_flops_and_where_they_run():
    gd = WORKLOADS[2]
    fl = bench.bwd_flops(gd)
    # 42 d dh per key token (recompute 12, reverse loop 30) + 16 d dh per query token
    assert fl["layer"] == pytest.approx(gd.B * gd.H * gd.d * gd.dh * (42.0 * gd.T + 16.0 * gd.Tq), rel=1e-12)
    assert fl["ns"] == 0.0
    muon = WORKLOADS[4]
    m, n = max(muon.d, muon.dh), min(muon.d, muon.dh)
    per_step_fwd = 4 * m * n * n + 2 * n ** 3          # Gram, square, update
    per_step_vjp = 6 * m * n * n + 4 * n ** 3          # X^T Y, dB A, A dB, Y B, X T
    want = muon.B * muon.H * 3 * muon.n_chunks * 5 * (2 * per_step_fwd + per_step_vjp)
    assert bench.bwd_flops(muon)["ns"] == pytest.approx(want, rel=1e-12)
    assert bench.bwd_on_tc(gd) and bench.bwd_on_tc(WORKLOADS[3])
    assert not bench.bwd_on_tc(muon) and not bench.bwd_on_tc(WORKLOADS[1])


def test_roofline_entry_divides_by_the_burst_peak(tmp_path, monkeypatch):
    """A kernel timed alone is measured against the burst bf16 peak, with the
    sustained fraction beside it; the achieved rate is the kernel's
    algorithmic FLOPs per launch over its average launch duration."""
    monkeypatch.setattr(bench, "peaks", lambda: (6543.0, 1690.9, 1388.0, "measured"))
    monkeypatch.setattr(bench, "traffic_for", lambda name, w: None)
    w = WORKLOADS[2]
    steps = 4
    n_launch = steps * w.n_chunks
    us = 40.0
    prof = {"fwd_key_umma": (n_launch, n_launch * us / 1e3), "rule_renorm": (n_launch, n_launch * 10.0 / 1e3)}
    r = bench.roofline_entry(prof, w, steps)
    per_launch = 6.0 * w.d * w.dh * w.B * w.H * w.T / w.n_chunks
    achieved = per_launch / (us * 1e-6) / 1e12
    assert r["kernel"] == "fwd_key_umma" and r["peak"] == 1690.9
    assert r["achieved"] == pytest.approx(achieved, rel=1e-12)
    assert r["frac"] == pytest.approx(achieved / 1690.9, rel=1e-12)
    assert r["frac_of_sustained"] == pytest.approx(achieved / 1388.0, rel=1e-12)


def test_measured_peaks_file_holds_the_burst_and_sustained_figures():
    path = bench.os.path.join(bench.ROOT, "MEASURED_PEAKS.json")
    if not bench.os.path.exists(path):
        pytest.skip("no measured peaks on this machine (the bench then uses its stated fallback)")
    with open(path) as f:
        p = json.load(f)
    hbm, burst, sust, src = bench.peaks()
    assert src == "measured" and burst == p["bf16_tflops"] and sust == p["bf16_tflops_sustained"]
    assert burst > sust > 0 and hbm > 0


def test_small_workloads_fall_back_to_the_fp32_path_in_the_flop_count():
    w = Workload("x", 1, 1, 256, 256, 64, 128, 256, APPLY_THEN_UPDATE, RULE_GD, F32)
    assert bench.step_flops(w) == pytest.approx(18.0 * 64 * 128 * 256, rel=1e-12)
    wm = w.scaled(rule=RULE_MOMENTUM, dtype=BF16)
    assert bench.step_flops(wm) == bench.step_flops(w)   # the momentum rule adds no contraction
