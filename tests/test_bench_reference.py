"""The benchmark's reference arm (the CPU oracle timed on the host cores), on CPU.

Its value must be the oracle's own measured rate: the dense work of every timed pass over
the time of those passes. A fixed fake rate pins the arithmetic exactly; a short real run
checks that the arm and the cpu_baseline leg's measurement agree.
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
    """Each step repeats its sample for ~budget seconds; the arm must report the rate those
    repeats ran at, not one pass's work over all of their time."""
    calls = []

    def fake_rate(prepared, budget, rows=None):
        calls.append(budget)
        return 0.125, 2.0, 32          # TFLOP/s over 2 s of repeated passes of 32 rows

    monkeypatch.setattr(bench, "oracle_sample_rate", fake_rate)
    line = _run_reference([WORKLOADS[1][0]], steps=3, warmup=1)
    assert line["impl"] == "reference"
    assert abs(line["value"] - 0.125) < 1e-12
    assert abs(line["cpu_baseline"]["value"] - 0.125) < 1e-12
    assert abs(line["ms_per_step"] - 2000.0) < 1e-9        # the timed sample per step
    assert line["e2e"]["value"] == line["value"]
    assert len(calls) == 4


def test_reference_arm_agrees_with_cpu_baseline_rate():
    layers = [WORKLOADS[1][0]]
    line = _run_reference(layers, steps=2, warmup=1)
    rate, _, _ = bench.oracle_sample_rate(bench.prepare_oracle(layers, max_rows=2048), 1.0)
    assert line["value"] > 0 and rate > 0
    # host timing noise: the same program on the same rows, so within a factor well under the
    # 27x an earlier accounting error produced
    assert 0.5 < line["value"] / rate < 2.0, (line["value"], rate)
