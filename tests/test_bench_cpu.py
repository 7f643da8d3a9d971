"""Host logic of bench.py that needs no GPU: the measured-peak loader and its fallback, the
comment-insensitive kernel-source hash that guards recorded ncu traffic, the traffic lookup, the
reference arm's JSON line (run on a bounded sample: one step, one warm-up), and its no-op on
non-zero ranks."""

import json
import types

import pytest

import bench


def _tree(tmp_path, attention_text, device_text="// helpers\nint x;\n"):
    csrc = tmp_path / "candidate_isolated_jagged_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "attention.cu").write_text(attention_text)
    (csrc / "jca_device.cuh").write_text(device_text)
    (tmp_path / "profiles").mkdir()
    return tmp_path


def test_peaks_measured_and_fallback(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    p = bench.load_peaks()
    assert p["source"] == "fallback" and p["hbm_gbs"] == bench.FALLBACK_PEAKS["hbm_gbs"]
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6000, "bf16_tflops": 1500}))
    p = bench.load_peaks()
    assert p["source"] == "measured" and p["hbm_gbs"] == 6000.0
    assert p["bf16_tflops_sustained"] == 1500.0      # absent: the burst figure stands in


def test_source_hash_ignores_comments_not_code(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(_tree(tmp_path, "int f() { return 1; }  // one\n")))
    h0 = bench.kernel_source_sha()
    (tmp_path / "candidate_isolated_jagged_b200/csrc/attention.cu").write_text(
        "/* a block\n comment */\nint  f()  {\n  return 1;   // other words\n}\n")
    assert bench.kernel_source_sha() == h0
    (tmp_path / "candidate_isolated_jagged_b200/csrc/attention.cu").write_text(
        "int f() { return 2; }\n")
    assert bench.kernel_source_sha() != h0


def test_profiled_traffic_needs_a_matching_hash(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(_tree(tmp_path, "int f();\n")))
    assert bench.profiled_traffic("k") is None                      # no summary
    sha = bench.kernel_source_sha()
    (tmp_path / "profiles" / "k.md").write_text(
        f"source_sha256_16: {sha}\ndram_bytes_per_launch: 1234567\n")
    assert bench.profiled_traffic("k") == 1234567.0
    (tmp_path / "profiles" / "k.md").write_text(
        "source_sha256_16: 0000000000000000\ndram_bytes_per_launch: 1234567\n")
    assert bench.profiled_traffic("k") is None                      # stale capture


def test_reference_arm_is_a_no_op_off_rank_zero(capsys):
    args = types.SimpleNamespace(gpus=2, steps=1, warmup=3)
    assert bench.run_reference(args, rank=1) == 0
    assert capsys.readouterr().out == ""


@pytest.mark.timeout(600)
def test_reference_arm_line(capsys):
    args = types.SimpleNamespace(gpus=1, steps=1, warmup=1)
    assert bench.run_reference(args, rank=0) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC
    assert line["value"] > 0 and line["unit"] == "TFLOP/s" and line["higher_is_better"] is True
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]
