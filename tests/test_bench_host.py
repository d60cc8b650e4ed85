"""Host logic of bench.py on CPU: a committed ncu traffic record is used only for
the workload it was taken on and only while the kernel source it names still
hashes to the recorded value; the peaks fall back to the stated figures when the
measured file is absent; the reference arm (the oracle) prints the contract's
line and refuses fewer than three warm-up steps."""

import hashlib
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _tree(tmp_path, source_text, recorded_text, workload="swin_t_s1_b8"):
    csrc = tmp_path / "shifted_window_attention_sw_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cu").write_text(source_text)
    (tmp_path / "profiles").mkdir()
    rec = {"k_kernel": {"bytes_per_launch": 123, "source": "k.cu", "workload": workload,
                        "sha256": hashlib.sha256(recorded_text.encode()).hexdigest()}}
    (tmp_path / "profiles" / "ncu_traffic.json").write_text(json.dumps(rec))


def test_traffic_record_used_while_source_unchanged(tmp_path, monkeypatch):
    _tree(tmp_path, "kernel v1", "kernel v1")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_record("k_kernel", "swin_t_s1_b8")["bytes_per_launch"] == 123


def test_traffic_record_dropped_after_a_source_change(tmp_path, monkeypatch):
    _tree(tmp_path, "kernel v2", "kernel v1")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_record("k_kernel", "swin_t_s1_b8") is None


def test_traffic_record_dropped_for_another_workload(tmp_path, monkeypatch):
    _tree(tmp_path, "kernel v1", "kernel v1")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_record("k_kernel", "swin_t_s3_b32") is None
    assert bench.traffic_record("other_kernel", "swin_t_s1_b8") is None


def test_committed_records_name_existing_sources_and_workloads():
    with open(os.path.join(ROOT, "profiles", "ncu_traffic.json")) as f:
        rec = json.load(f)
    assert rec
    for name, entry in rec.items():
        src = os.path.join(ROOT, "shifted_window_attention_sw_b200", "csrc", entry["source"])
        assert os.path.isfile(src), name
        assert entry["workload"] in bench.WORKLOADS, name
        assert entry["bytes_per_launch"] > 0
        assert len(entry["dram_read_bytes"]) == len(entry["dram_write_bytes"]) >= 1


def test_peaks_fall_back_when_the_measured_file_is_absent(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    peaks, src = bench.load_peaks()
    assert src == "fallback"
    assert peaks == bench.FALLBACK_PEAKS


def test_peaks_read_from_the_measured_file(tmp_path, monkeypatch):
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6500.0, "bf16_tflops": 1600.0}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    peaks, src = bench.load_peaks()
    assert src == "measured"
    assert peaks["hbm_gbs"] == pytest.approx(6500.0)


def _reference_line(*extra):
    import subprocess
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                        "swin_t_s1_small_f32", *extra], capture_output=True, text=True, timeout=600,
                       env=dict(os.environ, CUDA_VISIBLE_DEVICES=""))
    return r


def test_reference_arm_line_contract():
    # the oracle timed as the reference arm (small workload, a few seconds): one JSON
    # line with the arm's metric and unit, its own value as cpu_baseline and e2e, and
    # no host<->device bytes
    r = _reference_line("--steps", "1", "--warmup", "3")
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["metric"] == bench.METRIC and line["unit"] == "tokens/s"
    assert line["higher_is_better"] is True
    assert (line["steps"], line["warmup"]) == (1, 3)
    assert line["value"] > 0
    assert line["config"]["workload"] == "swin_t_s1_small_f32"
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"]
    assert cb["value"] == pytest.approx(line["value"])
    e2e = line["e2e"]
    assert e2e["value"] == pytest.approx(line["value"]) and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_reference_arm_refuses_fewer_than_three_warmup_steps():
    r = _reference_line("--steps", "1", "--warmup", "1")
    assert r.returncode != 0
