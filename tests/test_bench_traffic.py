"""CPU: bench.py reports a stored DRAM-traffic capture of the pass kernel only for the kernel
sources it was taken on, scaled from the captured stack to the 64-layer pass by the ratio of
the algorithmic bytes."""

import importlib.util
import json
import os
import shutil

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_traffic_under_test", os.path.join(ROOT, "bench.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    return b


def test_capture_is_scaled_and_guarded(tmp_path, monkeypatch):
    b = _bench()
    prof = {"source_sha256": b.pass_kernel_source_hash(), "layers": 8,
            "per_m": {"17": {"dram_read_bytes": 1000, "dram_write_bytes": 24}}}
    path = tmp_path / "traffic.json"
    path.write_text(json.dumps(prof))
    monkeypatch.setattr(b, "TRAFFIC_PROFILE", str(path))
    want = 1024 * b.pass_alg_bytes(17, 64) / b.pass_alg_bytes(17, 8)
    assert b.measured_traffic(17, 64) == pytest.approx(want)
    assert b.measured_traffic(1, 64) is None                 # no capture at this M
    assert b.measured_traffic(17, 8) is None                 # only the full 64-layer pass is reported
    prof["layers"] = 64
    path.write_text(json.dumps(prof))
    assert b.measured_traffic(17, 64) == pytest.approx(1024)
    prof["source_sha256"] = "0" * 64                         # the kernel changed since the capture
    path.write_text(json.dumps(prof))
    assert b.measured_traffic(17, 64) is None


def test_source_hash_ignores_comments_only(tmp_path, monkeypatch):
    b = _bench()
    for rel in b.PASS_KERNEL_SOURCES:
        dst = tmp_path / rel
        dst.parent.mkdir(parents=True, exist_ok=True)
        shutil.copy(os.path.join(ROOT, rel), dst)
    monkeypatch.setattr(b, "ROOT", str(tmp_path))
    h0 = b.pass_kernel_source_hash()
    assert h0 == _bench().pass_kernel_source_hash()          # the copy hashes like the tree
    first = tmp_path / b.PASS_KERNEL_SOURCES[0]
    text = first.read_text()
    first.write_text("// a comment\n" + text.replace("\n", "\n  ", 3) + "\n/* another */\n")
    assert b.pass_kernel_source_hash() == h0                 # comments and whitespace do not count
    first.write_text(text + "\nstatic int a_new_line_of_code = 0;\n")
    assert b.pass_kernel_source_hash() != h0
