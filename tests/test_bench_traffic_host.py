"""Host tests of the bench's bookkeeping around the roofline fields: the DRAM
traffic stored from an ncu capture is reported only while the code of the
kernel's sources is the code that was captured (comments and whitespace may
change), and the peaks come from the measured file, else the stated
fallback. No GPU needed."""
import json
import os
import shutil
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


def test_code_only_drops_comments_and_whitespace():
    src = "int a = 1; /* block\n comment */ int b; // line comment\n  return a  +\tb;"
    assert bench._code_only(src) == "inta=1;intb;returna+b;"


def fake_root(tmp_path):
    csrc = tmp_path / "weight_only_quantization_group_b200" / "csrc"
    csrc.mkdir(parents=True)
    for name in bench.KERNEL_SOURCES["gemv_rows_kernel"]:
        shutil.copy(os.path.join(bench.ROOT, "weight_only_quantization_group_b200", "csrc", name), csrc / name)
    (tmp_path / "profiles").mkdir()
    return csrc


def test_traffic_follows_the_code_not_the_comments(tmp_path, monkeypatch):
    csrc = fake_root(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h = bench.kernel_source_hash()
    assert h == bench.kernel_source_hash()
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(
        {"gemv_rows_kernel": {"dram_bytes_per_launch": 12345, "source_hash": h}}))
    assert bench.profiled_traffic("gemv_rows_kernel") == 12345
    # a comment and reflowed whitespace: same code, same traffic
    f = csrc / bench.KERNEL_SOURCES["gemv_rows_kernel"][0]
    f.write_text("// a new comment\n" + f.read_text().replace("\n", "\n\n", 3))
    assert bench.kernel_source_hash() == h
    assert bench.profiled_traffic("gemv_rows_kernel") == 12345
    # a code change: the stored traffic no longer describes the kernel
    f.write_text(f.read_text() + "\nstatic int extra_symbol = 0;\n")
    assert bench.kernel_source_hash() != h
    assert bench.profiled_traffic("gemv_rows_kernel") is None
    # no entry, or no file: nothing reported
    assert bench.profiled_traffic("some_other_kernel") is None
    (tmp_path / "profiles" / "traffic.json").unlink()
    assert bench.profiled_traffic("gemv_rows_kernel") is None


def test_peaks_measured_else_fallback(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    p = bench.load_peaks()
    assert p["source"] == "fallback" and p["hbm_gbs"] == bench.FALLBACK_HBM_GBS
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6000.5, "bf16_tflops": 1500.0}))
    p = bench.load_peaks()
    assert p["source"] == "measured" and p["hbm_gbs"] == 6000.5 and p["bf16_tflops_sustained"] == 1500.0
