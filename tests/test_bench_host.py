"""Host-side arithmetic of bench.py: the whole-job rate over replica ranks
and the exponential (MUFU) bound reported beside the tensor roofline."""
import os
import sys

import pytest

sys.path.insert(0, os.path.join(os.path.dirname(__file__), ".."))


def test_whole_job_rate_counts_every_rank():
    import bench
    from vision_transformer_shifted_window_b200 import synthetic as syn
    wk = bench.work(syn.WORKLOADS[3])
    one = bench.whole_job(wk, 1, 0.5)
    two = bench.whole_job(wk, 2, 0.5)
    assert two["tokens_per_s"] == pytest.approx(2 * one["tokens_per_s"])
    assert one["tokens_per_s"] == pytest.approx(16 * 112 * 112 / 0.5e-3)
    assert one["tflops"] == pytest.approx(68.05e9 / 0.5e-3 / 1e12, rel=1e-3)


def test_exp_bound_of_the_m32_workload():
    import bench
    from vision_transformer_shifted_window_b200 import synthetic as syn
    wk = bench.work(syn.WORKLOADS[3])
    assert wk["exps"] == pytest.approx(68.05e9 / 128, rel=1e-3)  # one exp per attended pair at d = 32
    eb = bench.exp_bound(wk, 148, 1965.0, 0.3)
    assert eb["bound_ms"] == pytest.approx(wk["exps"] / (16 * 148 * 1965e6) * 1e3, rel=1e-4)
    assert eb["frac"] == pytest.approx(eb["bound_ms"] / 0.3, rel=1e-3)
