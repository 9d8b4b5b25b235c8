"""Host-side pieces of the benchmark that decide what its JSON line reports,
checked on CPU: the DRAM-traffic record is used only while every source it
was captured from is unchanged, the clock summary reads nvidia-smi's CSV
rows (median clock, throttle reasons) as the timing rules require, and the
peaks come from the measured file when it is there."""
import hashlib
import json
import os

import bench


def _tree(tmp_path, sources, record_sources):
    csrc = tmp_path / "block_sparse_attention_kap_b200" / "csrc"
    csrc.mkdir(parents=True)
    for name, text in sources.items():
        (csrc / name).write_text(text)
    prof = tmp_path / "profiles"
    prof.mkdir()
    rec = {"kernels": {"k<1>": {"dram_read_bytes": 1000, "dram_write_bytes": 24,
                                "sources_sha256_16": record_sources}}}
    (prof / "traffic_gqa_128k.json").write_text(json.dumps(rec))
    return tmp_path


def _h(text):
    return hashlib.sha256(text.encode()).hexdigest()[:16]


def test_traffic_record_used_while_sources_match(tmp_path, monkeypatch):
    root = _tree(tmp_path, {"a.cu": "kernel A", "b.h": "header"}, {"a.cu": _h("kernel A"), "b.h": _h("header")})
    monkeypatch.setattr(bench, "ROOT", str(root))
    assert bench.recorded_traffic("k<1>") == 1024


def test_traffic_record_dropped_when_a_source_changed(tmp_path, monkeypatch):
    root = _tree(tmp_path, {"a.cu": "kernel A, edited", "b.h": "header"},
                 {"a.cu": _h("kernel A"), "b.h": _h("header")})
    monkeypatch.setattr(bench, "ROOT", str(root))
    assert bench.recorded_traffic("k<1>") is None


def test_traffic_record_dropped_when_missing(tmp_path, monkeypatch):
    root = _tree(tmp_path, {"a.cu": "kernel A"}, {"a.cu": _h("kernel A"), "gone.h": _h("x")})
    monkeypatch.setattr(bench, "ROOT", str(root))
    assert bench.recorded_traffic("k<1>") is None          # a listed source no longer exists
    assert bench.recorded_traffic("other<2>") is None      # no record for this kernel


def _sampler_with_rows(tmp_path, rows):
    f = tmp_path / "clocks.csv"
    f.write_text("".join(r + "\n" for r in rows))

    class _Done:                       # stands in for the finished nvidia-smi process
        pass

    s = bench.ClockSampler(0)
    s.proc = _Done()
    s.file = open(f, "r+")
    return s


def test_clock_summary_median_and_reasons(tmp_path):
    rows = [
        "0, 1965, 1965, 300.5, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, 1912, 1965, 910.2, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1530, 1965, 980.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
    ]
    out = _sampler_with_rows(tmp_path, rows).summary()
    assert out["sm_mhz"] == 1912.0 and out["sm_max_mhz"] == 1965.0
    assert out["sm_min_mhz"] == 1530.0 and out["power_w_max"] == 980.0
    assert out["reasons"] == ["sw_power_cap"] and out["samples"] == 3


def test_clock_summary_flags_thermal_and_hw_slowdown(tmp_path):
    rows = ["0, 1400, 1965, 700.0, 0x48, Active, Not Active, Active, Not Active"]
    out = _sampler_with_rows(tmp_path, rows).summary()
    assert out["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]


def test_clock_summary_without_samples(tmp_path):
    out = _sampler_with_rows(tmp_path, ["garbage"]).summary()
    assert out["sm_mhz"] is None and out["reasons"] == ["no samples"]


def test_peaks_come_from_the_measured_file(tmp_path, monkeypatch):
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps(
        {"hbm_gbs": 6000.0, "bf16_tflops": 1500.0, "bf16_tflops_sustained": 1300.0}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.load_peaks() == (6000.0, 1500.0, 1300.0, "measured")
    os.remove(tmp_path / "MEASURED_PEAKS.json")
    hbm, tc, sus, kind = bench.load_peaks()
    assert kind == "fallback" and (hbm, tc, sus) == (6650.0, 1590.0, 1400.0)
