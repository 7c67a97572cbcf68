"""The bench's roofline denominators: measured figures are taken where the peaks file has
them, in either shape, and the fallback fills whatever it lacks; a missing or unreadable
file gives the fallback."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _write(tmp_path, obj):
    p = tmp_path / "MEASURED_PEAKS.json"
    p.write_text(obj if isinstance(obj, str) else json.dumps(obj))
    return str(p)


def test_plain_numbers(tmp_path):
    pk, src = bench.peaks(_write(tmp_path, {"hbm_gbs": 6540.0, "bf16_tflops": 1610.6,
                                            "bf16_tflops_sustained": 1395.0, "clocks": "x"}))
    assert set(src.values()) == {"measured"}
    assert pk == {"hbm_gbs": 6540.0, "bf16_tflops": 1610.6, "bf16_tflops_sustained": 1395.0}


def test_value_objects_and_missing_keys(tmp_path):
    pk, src = bench.peaks(_write(tmp_path, {"hbm_gbs": {"value": 6500, "unit": "GB/s"}, "bf16_tflops": "n/a"}))
    assert src == {"hbm_gbs": "measured", "bf16_tflops": "fallback", "bf16_tflops_sustained": "fallback"}
    assert pk["hbm_gbs"] == 6500.0
    assert pk["bf16_tflops"] == bench.FALLBACK_PEAKS["bf16_tflops"]
    assert pk["bf16_tflops_sustained"] == bench.FALLBACK_PEAKS["bf16_tflops_sustained"]


def test_unreadable_or_absent_file(tmp_path):
    fb = {k: "fallback" for k in bench.FALLBACK_PEAKS}
    assert bench.peaks(_write(tmp_path, "{not json"))[1] == fb
    assert bench.peaks(_write(tmp_path, [1, 2, 3]))[1] == fb
    assert bench.peaks(str(tmp_path / "absent.json")) == (dict(bench.FALLBACK_PEAKS), fb)
