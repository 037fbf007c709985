"""Host-side checks of the benchmark's accounting: the FLOP and byte counters
read from the index tensors agree with the oracle's own visible-set count."""

import numpy as np
import pytest

import bench
import oracle
from gen import get_workload, make_inputs, scaled

CASES = [
    ("cfg1", {}, {}),
    ("cfg2", dict(S=700, Hq=32, Hkv=2), dict(allow_future=True, ori_len_range=(0, 16))),
    ("cfg3", dict(S=300, Hq=16, topk=64), {}),
    ("cfg4", dict(seqlens=(100, 300, 37), Hq=16, cmp_topk=64, cmp_len_range=(16, 64)), dict(cmp_any=True)),
    ("cfg5", dict(S=1024, Hq=16, Hkv=4), {}),
    ("cfg4", dict(seqlens=(50, 90), Hq=8, cmp_topk=16, cmp_len_range=(2, 16), win_left=10, win_right=3), {}),
]


@pytest.mark.parametrize("name,ov,kw", CASES)
def test_flop_count_matches_oracle(name, ov, kw):
    w = scaled(name, **ov) if ov else get_workload(name)
    inp = make_inputs(w, **kw)
    c = bench.count_work(w, inp)
    p = oracle.Problem.from_inputs(w, inp)
    fwd = bwd = 0
    for tq, g in p.all_units():
        f, b = oracle.unit_flops(p, tq, g)
        fwd += f
        bwd += b
    assert c["fwd_flops"] == fwd and c["bwd_flops"] == bwd


def test_cfg1_matches_published_plan():
    """Config 1 totals: 0.526 GFLOP backward, 60.8 MB of gathered rows."""
    w = get_workload("cfg1")
    c = bench.count_work(w, make_inputs(w))
    assert abs(c["bwd_flops"] / 1e9 - 0.526) < 0.001
    assert abs(c["gathered_bytes"] / 1e6 - 60.8) < 0.1


def test_oracle_baseline_runs_briefly():
    w = scaled("cfg2", S=256, Hq=16, Hkv=1)
    r = bench.oracle_baseline(w, make_inputs(w), budget_s=0.5)
    assert r["value"] > 0 and r["cores"] >= 1 and r["kind"] == "oracle"


def test_reference_arm_line():
    class A:
        workload = "cfg1"
        override = None
        steps = 1
        warmup = 0
        step_budget = 1.0
    line = bench.run_reference(A(), rank=0)
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0
    assert bench.run_reference(A(), rank=1) is None


def test_reference_arm_reports_the_sample_and_the_gpu_arms_config():
    """ms_per_step is the measured sample; the config dict is the GPU arm's (same keys
    and values for the same workload), so the two arms compare like for like."""
    class A:
        workload = "cfg1"
        override = None
        steps = 2
        warmup = 0
        step_budget = 0.5
    line = bench.run_reference(A(), rank=0)
    w = get_workload("cfg1")
    work = bench.count_work(w, make_inputs(w))
    assert line["config"] == bench.config_of(w, work, 1, "")
    assert 400.0 <= line["ms_per_step"] <= 5000.0          # the ~0.5 s sample, not an extrapolation
    assert line["whole_backward_ms_at_sampled_rate"] > 0


def test_roofline_fractions():
    """The tensor fraction uses compulsory bytes only, so it never exceeds the
    spec fraction (whose byte count adds the gathered rows)."""
    w = get_workload("cfg1")
    work = bench.count_work(w, make_inputs(w))
    comp = bench.compulsory_bytes(w, work)
    assert comp["fwd"] < work["fwd_bytes"] and comp["bwd"] < work["bwd_main_bytes"] + comp["bwd"]
    peaks = {"bf16_tflops": 1000.0, "hbm_gbs": 5000.0}
    fr = bench.fractions(work, comp, peaks, fwd_ms=0.05, bwd_ms=0.05)
    assert fr["fwd_tensor_frac"] <= fr["fwd_gather_model_frac"]
    assert fr["bwd_tensor_frac"] <= fr["bwd_gather_model_frac"]
    # a time at exactly the spec roofline is a fraction of one
    t_ns = max(work["bwd_flops"] / 1e15, work["bwd_main_bytes"] / 5e12) * 1e3
    assert abs(bench.fractions(work, comp, peaks, 1.0, t_ns)["bwd_gather_model_frac"] - 1.0) < 1e-9
