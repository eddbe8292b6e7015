"""The benchmark's DRAM-traffic record (profiles/dram_traffic.json), on CPU.

`roofline.traffic` in the benchmark line comes from an ncu capture stored with the layers it
was taken on and a hash of the capturing kernel's code (comments and blank lines excluded). The
record must be used only while both still hold, so that a stale capture reads as null.
"""

import json

import bench
from structured_compressed_linear_b200.workloads import WORKLOADS


def test_code_only_ignores_comments_and_blank_lines():
    a = 'int x = 1;  // one\n\n/* a\n block */int y = 2;\nconst char* s = "// kept";\n'
    b = 'int x = 1;\nint y = 2;\n// another comment\nconst char* s = "// kept";\n'
    assert bench.code_only(a) == bench.code_only(b)
    assert '"// kept"' in bench.code_only(a)
    assert bench.code_only("int x = 1;") != bench.code_only("int x = 2;")


def _layers():
    return [L for L in WORKLOADS[4] if L.M == 4096]


def _record(tmp_path, **change):
    with open(bench.os.path.join(bench.ROOT, "profiles", "dram_traffic.json")) as f:
        d = json.load(f)
    d["TC"].update(change)
    p = tmp_path / "traffic.json"
    p.write_text(json.dumps(d))
    return str(p)


def test_record_holds_only_for_its_layers_and_code(tmp_path):
    layers = _layers()
    good = _record(tmp_path, source_hash=bench.source_hash(["ss1_tc3.cu", "ptx_sm100.cuh", "ss1_internal.cuh"]),
                   sources=["ss1_tc3.cu", "ptx_sm100.cuh", "ss1_internal.cuh"])
    rec = bench.traffic_record("TC", layers, path=good)
    assert rec is not None and rec["dram_bytes_per_step"] == sum(
        x["dram_read"] + x["dram_write"] for x in rec["per_launch"])
    assert bench.traffic_record("TC", layers, path=_record(tmp_path, source_hash="0" * 16)) is None
    assert bench.traffic_record("TC", layers[:-1], path=good) is None
    assert bench.traffic_record("TC", [L.with_M(2048) for L in layers], path=good) is None
    assert bench.traffic_record("DEC", layers, path=good) is None
