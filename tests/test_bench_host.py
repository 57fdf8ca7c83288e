"""Host logic of bench.py that decides what the JSON line reports: the peak
denominators (measured file, per-key fallback) and the committed DRAM
traffic figure, which is reported only while the kernel's code is the code
it was captured on.  CPU only."""
import json
import os
import shutil

import pytest

import bench

CSRC = os.path.join(bench.ROOT, "fp8_microscaling_quantization_b200", "csrc")


@pytest.fixture
def root(tmp_path, monkeypatch):
    shutil.copytree(CSRC, tmp_path / "fp8_microscaling_quantization_b200" / "csrc")
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    return tmp_path


def test_peaks_fall_back_without_the_measured_file(root):
    peaks, kind = bench.load_peaks()
    assert kind == "fallback"
    for k, v in bench.FALLBACK_PEAKS.items():
        assert peaks[k] == v and peaks["sources"][k] == "fallback"


def test_peaks_take_each_measured_key_and_fall_back_per_key(root):
    (root / "MEASURED_PEAKS.json").write_text(json.dumps(
        {"hbm_gbs": {"value": 7012.5, "unit": "GB/s"}, "bf16_tflops": "n/a", "bf16_tflops_sustained": -1}))
    peaks, kind = bench.load_peaks()
    assert kind == "measured"
    assert peaks["hbm_gbs"] == 7012.5 and peaks["sources"]["hbm_gbs"] == "measured"
    assert peaks["bf16_tflops"] == bench.FALLBACK_PEAKS["bf16_tflops"]
    assert peaks["sources"]["bf16_tflops"] == "fallback"
    assert peaks["bf16_tflops_sustained"] == bench.FALLBACK_PEAKS["bf16_tflops_sustained"]


def test_peaks_without_a_measured_hbm_figure_are_labelled_fallback(root):
    (root / "MEASURED_PEAKS.json").write_text(json.dumps({"bf16_tflops": 1700}))
    peaks, kind = bench.load_peaks()
    assert kind == "fallback" and peaks["bf16_tflops"] == 1700.0
    assert peaks["sources"]["bf16_tflops"] == "measured"


def test_unreadable_peaks_file_falls_back(root):
    (root / "MEASURED_PEAKS.json").write_text("{not json")
    assert bench.load_peaks()[1] == "fallback"


def _edit(root, name, old, new):
    p = root / "fp8_microscaling_quantization_b200" / "csrc" / name
    s = p.read_text()
    assert old in s
    p.write_text(s.replace(old, new, 1))


def test_source_hash_ignores_comments_and_layout_but_not_code(root):
    h0 = bench.kernel_source_hash("cache")
    _edit(root, "cache.cu", "// Row-resident fake-quant", "/* an added note */   // Row-resident   fake-quant")
    assert bench.kernel_source_hash("cache") == h0
    _edit(root, "cache.cu", "constexpr int RPW = 32 / S;", "constexpr int RPW = 32 /  S;\n\n")
    assert bench.kernel_source_hash("cache") == h0
    _edit(root, "cache.cu", "constexpr int RPW = 32 /  S;", "constexpr int RPW = 16 / S;")
    assert bench.kernel_source_hash("cache") != h0
    # a shared header is part of every family built from it
    g0, n0 = bench.kernel_source_hash("gemm"), bench.kernel_source_hash("nvfp4")
    _edit(root, "formats.cuh", "namespace bsq {", "namespace bsq {\nconstexpr int kUnusedProbe = 1;")
    assert bench.kernel_source_hash("gemm") != g0 and bench.kernel_source_hash("nvfp4") != n0


def test_traffic_is_reported_only_while_the_code_matches(root):
    ents = {
        "a": {"family": "cache", "bytes_per_launch": 1000, "source_hash": bench.kernel_source_hash("cache")},
        "b": {"family": "kv", "bytes_per_launch": 234, "source_hash": bench.kernel_source_hash("kv")},
        "c": {"family": "nope", "bytes_per_launch": 5, "source_hash": "0"},
    }
    (root / "profiles" / "dram_traffic.json").write_text(json.dumps({"kernels": ents}))
    assert bench.traffic_from_profiles("a") == 1000
    assert bench.traffic_from_profiles("a", "b") == 1234
    assert bench.traffic_from_profiles("a", "missing") is None
    assert bench.traffic_from_profiles("c") is None
    _edit(root, "kv_cache.cu", "namespace bsq {", "namespace bsq {\nconstexpr int kUnusedProbe = 1;")
    assert bench.traffic_from_profiles("a") == 1000
    assert bench.traffic_from_profiles("a", "b") is None


def test_committed_traffic_entries_name_known_families():
    with open(os.path.join(bench.ROOT, "profiles", "dram_traffic.json")) as f:
        kernels = json.load(f)["kernels"]
    assert kernels
    for key, ent in kernels.items():
        assert ent["family"] in bench.KERNEL_SOURCES, key
        # read and write are per launch, each averaged (and rounded) over the captured launches
        assert abs(ent["bytes_per_launch"] - ent["dram_read_bytes"] - ent["dram_write_bytes"]) <= 1, key
