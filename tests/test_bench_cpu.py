"""bench.py's host-side parts that need no GPU: the reference arm's JSON line, the
scaling of the oracle's sampled Hessian time, and the L2 statement."""
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


def test_sampled_hessian_time_is_scaled_to_the_full_token_count(monkeypatch):
    wl = WORKLOADS["opt125m"]
    m = bench.SAMPLE_TOKENS
    times = {768: (0.5, 1.0), 3072: (2.0, 3.0)}     # (Hessian s, rest s) by cols
    monkeypatch.setattr(bench, "oracle_layer", lambda W, X, wl_, q: times[X.shape[1]])
    layers = [(l, None, SimpleNamespace(shape=(m, l.cols))) for l in wl.layers]
    got = bench.cpu_step_ms_per_layer(wl, m, layers)
    scale = wl.tokens / m
    want = sum(times[l.cols][0] * scale + times[l.cols][1] for l in wl.layers) / 3 * 1e3
    assert got == pytest.approx(want, rel=1e-12)
    assert scale == 16
    assert "scaled by 16" in bench.cpu_sample_text(wl, m, layers)


def test_l2_statement_follows_the_input_size():
    assert bench.l2_note(WORKLOADS["opt125m"]).startswith("inputs larger than L2")
    assert bench.l2_note(WORKLOADS["tiny"]).startswith("inputs smaller than L2")
