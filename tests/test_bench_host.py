"""Host-side helpers of bench.py that need no GPU: the roofline denominators
and the kernel-code hash that keys the recorded DRAM traffic."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_peaks_measured_file_used_when_well_formed(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.load_peaks() == (bench.FALLBACK_PEAKS, "fallback")
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps(
        {"hbm_gbs": 6540.2, "bf16_tflops": 1632.8, "notes": "x"}))
    peaks, src = bench.load_peaks()
    assert src == "measured"
    assert peaks["hbm_gbs"] == 6540.2 and peaks["bf16_tflops"] == 1632.8
    assert peaks["bf16_tflops_sustained"] == bench.FALLBACK_PEAKS["bf16_tflops_sustained"]


def test_peaks_fall_back_on_a_malformed_file(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    for text in ("{", json.dumps({"hbm": 1}), json.dumps({"hbm_gbs": "fast", "bf16_tflops": 1}),
                 json.dumps([1, 2])):
        (tmp_path / "MEASURED_PEAKS.json").write_text(text)
        assert bench.load_peaks() == (bench.FALLBACK_PEAKS, "fallback")


def test_source_hash_ignores_comments_only():
    code = "int f(int a) {\n    return a + 1;   // one\n}\n/* block\n comment */\n"
    same = "int f(int a) {\n    return a + 1;\n}\n"
    other = "int f(int a) {\n    return a + 2;\n}\n"
    assert bench._strip_comments(code) == bench._strip_comments(same)
    assert bench._strip_comments(code) != bench._strip_comments(other)
    assert len(bench.kernel_source_hash()) == 16


def test_recorded_traffic_keyed_by_current_code():
    """Every row of profiles/dram_traffic.txt names a kernel of a workload;
    rows taken on the current kernel code are returned, others are not."""
    cur = bench.kernel_source_hash()
    with open(bench.TRAFFIC_FILE) as f:
        rows = [l.split() for l in f if l.strip() and not l.startswith("#")]
    assert rows
    for k, w, b, h in (r[:4] for r in rows):
        got = bench.recorded_traffic(k, w)
        assert (got == float(b)) if h == cur else (got is None or got != float(b))
