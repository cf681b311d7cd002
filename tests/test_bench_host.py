"""Host-side logic of bench.py that needs no GPU: the ncu traffic records in
profiles/ (read back only while the kernel source is unchanged), the peaks
file, and the reference arm's bounded sampling of the oracle."""

import json
import os

import pytest

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("summary,algorithmic", [
    ("w4r_gemv_gpt2_m1.md", bench.body_bytes()),
    ("w4r_step_gpt2_m1.md", bench.body_bytes() + bench.head_bytes()),
    ("w4r_gemv_3p8b_4layers_m1.md", 290193408),
    ("w4_gemv_pageformat_3p8b_4layers_m8.md", 290193408),
    ("i8r_head_gpt2_m1.md", bench.head_bytes()),
    ("w4_gemv_pageformat_gpt2_m1.md", bench.body_bytes()),
    ("i8_rows_pageformat_gpt2_head_m1.md", bench.head_bytes()),
    ("i8t_head_gpt2_m1.md", bench.head_bytes()),
    ("i8t_head_gpt2_m8.md", bench.head_bytes()),
])
def test_committed_profiles_are_machine_readable(summary, algorithmic):
    """Each summary names its kernel's source, a 16-hex-digit hash and the
    DRAM bytes of one launch, at least the algorithmic bytes (nothing can be
    read fewer times than once)."""
    fields = {}
    for line in open(os.path.join(ROOT, "profiles", summary)):
        if ":" in line and line.startswith("    "):
            k, v = line.strip().split(":", 1)
            fields[k.strip()] = v.strip()
    assert os.path.exists(os.path.join(ROOT, fields["source"]))
    assert len(fields["source_sha256_16"]) == 16
    int(fields["source_sha256_16"], 16)
    assert algorithmic <= int(fields["dram_bytes_per_launch"]) <= 1.05 * algorithmic


def test_traffic_is_dropped_when_the_source_changes(tmp_path, monkeypatch):
    (tmp_path / "profiles").mkdir()
    (tmp_path / "src").mkdir()
    src = tmp_path / "src" / "k.cu"
    src.write_text("kernel A\n")
    import hashlib
    h = hashlib.sha256(src.read_bytes()).hexdigest()[:16]
    (tmp_path / "profiles" / "k.md").write_text(
        "# k\n\n    kernel: k\n    source: src/k.cu\n    source_sha256_16: %s\n    dram_bytes_per_launch: 1234\n" % h)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profiled_traffic("k.md") == 1234
    src.write_text("kernel B\n")
    assert bench.profiled_traffic("k.md") is None
    assert bench.profiled_traffic("missing.md") is None


def test_peaks_fall_back_when_the_file_is_absent(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    p = bench.measured_peaks()
    assert p["_source"] == "fallback" and p["hbm_gbs"] > 0
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 7000.0, "bf16_tflops": 1600.0}))
    p = bench.measured_peaks()
    assert p["_source"] == "measured" and p["hbm_gbs"] == 7000.0


def test_reference_arm_samples_when_whole_steps_do_not_fit(monkeypatch):
    """With a tiny budget every timed step runs one op of the 49 (round robin)
    and the value counts exactly the bytes processed."""
    calls = []
    fake_ops = [(1000 * (j + 1), (lambda j=j: calls.append(j))) for j in range(49)]
    monkeypatch.setattr(bench, "_oracle_inputs", lambda: fake_ops)
    monkeypatch.setattr(bench, "REFERENCE_BUDGET_S", 0.0)

    class A:
        steps = 5
        warmup = 1
    line = bench.run_reference(A(), 1, 0)
    timed = calls[1:]  # the first call of each op list is the untimed estimate step
    assert len(calls) == 49 + 5
    assert timed[-5:] == [0, 1, 2, 3, 4]
    assert line["impl"] == "reference" and line["steps"] == 5
    assert "5 steps of 1 of the 49 ops" in line["cpu_baseline"]["sample"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def test_reference_arm_runs_whole_steps_when_they_fit(monkeypatch):
    calls = []
    fake_ops = [(10, (lambda j=j: calls.append(j))) for j in range(49)]
    monkeypatch.setattr(bench, "_oracle_inputs", lambda: fake_ops)

    class A:
        steps = 3
        warmup = 1
    line = bench.run_reference(A(), 1, 0)
    assert len(calls) == 49 * 4
    assert "3 full decode steps" in line["cpu_baseline"]["sample"]
    assert bench.run_reference(A(), 2, 1) is None  # only rank 0 runs it
