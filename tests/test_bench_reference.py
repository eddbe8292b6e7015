"""The benchmark's reference arm (the CPU oracle timed on the host cores), on CPU.

Its value must be the oracle's own measured rate: the dense work of every timed pass over
the time of those passes, on the same rows as the cpu_baseline leg. A fake pass pins the
arithmetic exactly; a short real run checks that the arm and the cpu_baseline leg agree.
"""

import argparse
import io
import json
from contextlib import redirect_stdout

import bench
from structured_compressed_linear_b200.workloads import WORKLOADS


def _run_reference(layers, steps=2, warmup=1):
    args = argparse.Namespace(steps=steps, warmup=warmup)
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.run_reference(args, layers, 1, 0, 1)
    return json.loads(buf.getvalue().strip().splitlines()[-1])


def test_reference_value_is_the_sample_rate(monkeypatch):
    """Each step is one layer's pass; the arm must report the dense work of the timed passes
    over their time, and time one layer per step in rotation."""
    calls = []

    def fake_pass(prepared, rows):
        calls.append(prepared[0][0])
        return 0.25e12, 2.0           # 0.25 TFLOP of dense work in 2 s

    monkeypatch.setattr(bench, "_oracle_pass", fake_pass)
    layers = WORKLOADS[2]
    line = _run_reference(layers, steps=3, warmup=1)
    assert line["impl"] == "reference"
    assert abs(line["value"] - 0.125) < 1e-12
    assert abs(line["cpu_baseline"]["value"] - 0.125) < 1e-12
    assert abs(line["ms_per_step"] - 2000.0) < 1e-9        # the timed pass per step
    assert line["e2e"]["value"] == line["value"]
    assert calls == [layers[0], layers[0], layers[1], layers[2]]   # warm-up, then steps 0, 1, 2


def test_reference_arm_agrees_with_cpu_baseline_rate():
    layers = [WORKLOADS[1][0]]
    line = _run_reference(layers, steps=2, warmup=1)
    rate, _, _ = bench.oracle_sample_rate(bench.prepare_oracle(layers, max_rows=2048), 1.0)
    assert line["value"] > 0 and rate > 0
    # host timing noise: the same program on the same rows, so within a factor well under the
    # 27x an earlier accounting error produced
    assert 0.5 < line["value"] / rate < 2.0, (line["value"], rate)
