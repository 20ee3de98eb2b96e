"""Host-side helpers of bench.py that decide what the bench line reports:
the captured DRAM traffic is reported only for the GEMM build it was taken
from, and the issue bound of the instruction-bound rows only for the quantizer
build whose instructions were counted."""
import shutil

import bench


def _section(text):
    a = text.index("namespace gemm {")
    b = text.index("// ------------------------------------------------------------------ W4A16")
    return a, b


def test_gemm_hash_covers_the_gemm_section_and_the_ptx_header(tmp_path, monkeypatch):
    src = bench.GEMM_SOURCE
    shutil.copy(src, tmp_path / "q4_gemm.cu")
    shutil.copy(src.parent / "q4_ptx.cuh", tmp_path / "q4_ptx.cuh")
    monkeypatch.setattr(bench, "GEMM_SOURCE", tmp_path / "q4_gemm.cu")
    h0 = bench.gemm_source_hash()
    assert h0 == bench.gemm_source_hash()
    text = (tmp_path / "q4_gemm.cu").read_text()
    a, b = _section(text)
    # an edit after the GEMM section (another kernel) keeps the hash
    (tmp_path / "q4_gemm.cu").write_text(text + "\n// another kernel\n")
    assert bench.gemm_source_hash() == h0
    # an edit inside it, or in the PTX header, changes it
    (tmp_path / "q4_gemm.cu").write_text(text[:b] + "// edit\n" + text[b:])
    assert bench.gemm_source_hash() != h0
    (tmp_path / "q4_gemm.cu").write_text(text)
    (tmp_path / "q4_ptx.cuh").write_text((tmp_path / "q4_ptx.cuh").read_text() + "\n")
    assert bench.gemm_source_hash() != h0


def test_roofline_traffic_only_for_the_captured_build(monkeypatch):
    cur = bench.gemm_source_hash()
    monkeypatch.setattr(bench, "GEMM_TRAFFIC", {"bytes": 123, "source_sha256_16": cur})
    assert bench.roofline_traffic(None)[0] == 123
    monkeypatch.setattr(bench, "GEMM_TRAFFIC", {"bytes": 123, "source_sha256_16": "0" * 16})
    assert bench.roofline_traffic(None)[0] is None
    assert bench.roofline_traffic(77)[0] == 77           # given on the command line


def test_issue_bound_arithmetic_and_gating(monkeypatch):
    cur = bench.issue_sources_hash()
    monkeypatch.setattr(bench, "ISSUE_COUNTS", {"sources_sha256_16": cur, "row": 592 * 1965})
    r = bench.issue_bound("row", 2.0, 148)
    # 592 * 1965 warp instructions on 148 SMs x 4 schedulers at 1965 MHz take 1 us
    assert abs(r["issue_bound_us"] - 1.0) < 1e-12 and abs(r["frac"] - 0.5) < 1e-12
    assert r["bound"] == "alu"
    monkeypatch.setattr(bench, "ISSUE_COUNTS", {"sources_sha256_16": "0" * 16, "row": 1})
    assert "issue_bound_us" not in bench.issue_bound("row", 2.0, 148)
