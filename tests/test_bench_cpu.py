"""bench.py's host-side parts that need no GPU: the reference arm's JSON line, the
scaling of the oracle's sampled phase times to the full layer, and the L2 statement."""
import json
import subprocess
import sys
from types import SimpleNamespace

import pytest

import bench
from post_weight_quantization_20_b200.workloads import WORKLOADS

REQUIRED = {"impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
            "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
            "cpu_baseline", "e2e"}


def test_reference_arm_prints_one_contract_line():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny",
                        "--steps", "2", "--warmup", "1"], capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    out = json.loads(lines[0])
    assert REQUIRED <= set(out)
    assert out["impl"] == "reference" and out["higher_is_better"] is False
    assert out["value"] > 0 and out["cpu_baseline"]["value"] == out["value"]
    assert out["cpu_baseline"]["kind"] == "oracle" and out["cpu_baseline"]["cores"] >= 1
    assert out["e2e"] == {"value": out["value"], "unit": out["unit"], "h2d_bytes_per_step": 0,
                          "d2h_bytes_per_step": 0}


def test_sampled_phase_times_are_scaled_to_the_full_layer(monkeypatch):
    wl = WORKLOADS["opt175b"]
    l = wl.layers[2]                                   # 12288 x 49152
    m, cs, r = bench.SAMPLE_TOKENS, bench.SAMPLE_COLS, bench.SAMPLE_ROWS
    # sweep times exactly a c + b c^2 with a = 1e-5, b = 1e-9: the fit must recover it
    a, b = 1e-5, 1e-9
    times = (0.5, 2.0, a * cs / 2 + b * (cs / 2) ** 2, a * cs + b * cs ** 2, 0.01)
    got = bench.layer_ms_from_sample(times, l, wl, m, cs, r)
    C, R, N = l.cols, l.rows, wl.tokens
    want = (0.5 * (N / m) * (C / cs) ** 2 + 2.0 * (C / cs) ** 3 +
            (a * C + b * C * C) * (R / r) + 0.01 * (R / r) * (C / cs)) * 1e3
    assert got == pytest.approx(want, rel=1e-9)
    text = bench.cpu_sample_text(wl, (l, None, None, m, cs, r))
    assert "extrapolated" in text and f"{m} tokens, {cs} cols, {r} rows" in text
    # the step: one timed sample, every layer extrapolated from it, the mean per layer
    monkeypatch.setattr(bench, "oracle_phases", lambda W, X, wl_, q: times)
    step = bench.cpu_step_ms_per_layer(wl, (l, None, None, m, cs, r))
    assert step == pytest.approx(sum(bench.layer_ms_from_sample(times, x, wl, m, cs, r)
                                     for x in wl.layers) / 3, rel=1e-12)


def test_sweep_fit_stays_non_negative():
    # noise that would give a negative quadratic term falls back to a linear fit
    assert bench.sweep_model(0.6, 1.0, 100, 200, 400) == pytest.approx(2.0)
    assert bench.sweep_model(0.25, 1.0, 100, 200, 400) == pytest.approx(4.0)


def test_l2_statement_follows_the_input_size():
    assert bench.l2_note(WORKLOADS["opt125m"]).startswith("inputs larger than L2")
    assert bench.l2_note(WORKLOADS["tiny"]).startswith("inputs smaller than L2")
