"""Host-side checks of the seeded workloads and of the parity metric (no GPU)."""

import numpy as np
import pytest
import torch

from structured_compressed_linear_b200.workloads import WORKLOADS, make_inputs, instance_seed
from tests._parity import row_normalised_max_err


def test_workload_shapes_are_valid_ss1_layers():
    for wid, layers in WORKLOADS.items():
        for L in layers:
            assert L.K % L.BK == 0 and L.N % L.BN == 0 and L.BK % L.c == 0, L
            assert L.BK <= 256
    assert len(WORKLOADS[4]) == 24 and len(WORKLOADS[5]) == 19


def test_inputs_deterministic_and_distinct():
    L = WORKLOADS[2][1].with_M(64)
    X1, W1 = make_inputs(L)
    X2, W2 = make_inputs(L)
    assert torch.equal(X1, X2) and torch.equal(W1, W2)
    assert X1.dtype == torch.bfloat16 and X1.shape == (64, 768) and W1.shape == (768, 384)
    seeds = {instance_seed(L) for ws in WORKLOADS.values() for L in ws}
    assert len(seeds) == sum(len(ws) for ws in WORKLOADS.values())


def test_outlier_rows():
    L = WORKLOADS[3][1].with_M(1000)
    X, Wc = make_inputs(L)
    rn = X.float().abs().amax(dim=1)
    assert int((rn > 12).sum()) >= 9          # ~1% of rows scaled x20
    bound = 1.0 / np.sqrt(L.K)
    assert float(Wc.float().abs().max()) <= bound * 1.01


def test_parity_metric():
    ref = np.array([[1.0, -2.0, 0.5], [100.0, 0.0, 1.0]])
    y = ref.copy()
    y[0, 1] += 0.02
    y[1, 2] += 1.0
    assert abs(row_normalised_max_err(y, ref) - 0.01) < 1e-12
    assert row_normalised_max_err(ref, ref) == 0.0


def test_bench_layer_selection():
    """bench.py runs a workload's largest row count by default and any of its row counts on request."""
    import importlib.util
    import os
    from tests.conftest import ROOT
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    # default: the Llama-3-8B projections at the prefill row count, both compressions
    wid, layers = bench.select_layers(None, None)
    assert wid == 4 and len(layers) == 8 and {L.M for L in layers} == {4096} and {L.c for L in layers} == {2, 8}
    _, layers = bench.select_layers(2, None)
    assert len(layers) == 4 and {L.M for L in layers} == {8192}
    _, layers = bench.select_layers(4, None)
    assert {L.M for L in layers} == {4096} and len(layers) == 8
    _, layers = bench.select_layers(4, 1)
    assert {L.M for L in layers} == {1} and len(layers) == 8
    with pytest.raises(SystemExit):
        bench.select_layers(4, 3)
    _, layers = bench.select_layers(4, None, "4096x14336c2")
    assert [(L.K, L.N, L.c, L.M) for L in layers] == [(4096, 14336, 2, 4096)]
    with pytest.raises(SystemExit):
        bench.select_layers(4, None, "1x1c2")


def test_bench_work_matches_hand_values():
    """The benchmark's per-layer work against values worked out by hand from the metric's
    definition: actual flops = 2 M N K / c plus the M (N / BN) K (1 - 1/c) sketch additions,
    bytes = 2 (M K + N K / c + M N) for bf16 (GFLOP and MB, rounded as written)."""
    import importlib.util
    import os
    from structured_compressed_linear_b200.workloads import Layer
    from tests.conftest import ROOT
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    cases = [  # (M, K, N, c, BK, GFLOP, MB)
        (16384, 1280, 3840, 4, 128, 40.7, 170.2),
        (16384, 1280, 1280, 4, 128, 13.6, 84.7),
        (16384, 1280, 5120, 4, 128, 54.3, 213.0),
        (4096, 4096, 4096, 2, 256, 69.0, 83.9),
        (4096, 4096, 1024, 2, 256, 17.2, 46.1),
        (4096, 4096, 14336, 2, 256, 241.5, 209.7),
        (4096, 4096, 4096, 8, 256, 17.65, 71.3),
        (4096, 4096, 1024, 8, 256, 4.4, 43.0),
    ]
    for M, K, N, c, BK, gflop, mb in cases:
        L = Layer("hand", M, K, N, c, BK, 128, "bf16", "normal", "normal_002", 0)
        dense, actual, byts = bench.layer_work(L)
        assert dense == 2.0 * M * N * K
        assert abs(actual / 1e9 - gflop) <= 0.05, (M, K, N, c, actual)
        assert abs(byts / 1e6 - mb) <= 0.05, (M, K, N, c, byts)
    # exactly, in powers of two: Llama 4096 x 4096 at M = 4096, c = 8, BK = 256 (32 N-blocks):
    # 2 * 2^36 / 8 = 2^34 products, 2^12 * 32 * 2^12 * 7/8 = 7 * 2^26 additions;
    # bytes 2 * (2^24 + 2^21 + 2^24)
    L = Layer("hand", 4096, 4096, 4096, 8, 256, 128, "bf16", "normal", "normal_002", 0)
    _, actual, byts = bench.layer_work(L)
    assert actual == 2 ** 34 + 7 * 2 ** 26 and byts == 2 * (2 ** 24 + 2 ** 21 + 2 ** 24)


def _bench_module():
    import importlib.util
    import os
    from tests.conftest import ROOT
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    return bench


def test_traffic_record_only_for_its_layers_and_code(tmp_path):
    """DRAM counters are reported for the layers and the kernel code they were taken on, no others."""
    import json
    bench = _bench_module()
    sources = ["ss1_tc3.cu", "ptx_sm100.cuh", "ss1_internal.cuh"]
    rec = {"TC": {"layers": [bench.layer_key(L) for L in WORKLOADS[2]], "dram_bytes_per_step": 1,
                  "sources": sources, "source_hash": bench.source_hash(sources)}}
    p = tmp_path / "dram_traffic.json"
    p.write_text(json.dumps(rec))
    assert bench.traffic_record("TC", WORKLOADS[2], str(p)) is not None
    assert bench.traffic_record("TC", WORKLOADS[3], str(p)) is None
    assert bench.traffic_record("TC", [L.with_M(4096) for L in WORKLOADS[2]], str(p)) is None
    assert bench.traffic_record("SMALLM", WORKLOADS[2], str(p)) is None
    rec["TC"]["source_hash"] = "0" * 16          # the kernel's code changed since the capture
    p.write_text(json.dumps(rec))
    assert bench.traffic_record("TC", WORKLOADS[2], str(p)) is None


def test_source_hash_ignores_comments_only():
    bench = _bench_module()
    a = 'int f() { return 1; }  // one\n/* block\n comment */\nconst char* s = "a // b /* c */";\n'
    b = '// header\nint f() { return 1; }\n\nconst char* s = "a // b /* c */";  /* tail */\n'
    c = 'int f() { return 2; }\nconst char* s = "a // b /* c */";\n'
    assert bench.code_only(a) == bench.code_only(b)
    assert bench.code_only(a) != bench.code_only(c)
    assert '"a // b /* c */"' in bench.code_only(a)


def test_fp32_layers_use_the_alu_peak():
    """The fp32 workload runs on the CUDA cores: its roofline is the FP32 ALU peak, not the bf16
    tensor peak (148 SMs x 128 lanes x 2 flops x 1.965 GHz = 74.4 TFLOP/s)."""
    bench = _bench_module()
    peaks = {"bf16_tflops": 1628.3, "hbm_gbs": 6542.7}
    assert abs(bench.compute_peak_tflops(WORKLOADS[1][0], peaks) - 74.4) < 0.05
    assert bench.compute_peak_tflops(WORKLOADS[2][0], peaks) == 1628.3
