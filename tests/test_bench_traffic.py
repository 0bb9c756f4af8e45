"""bench.py's roofline.traffic: the committed DRAM capture of a workload is used only while its
hash of the attention kernel's sources matches the current sources, and a capture of a smaller
launch is scaled to the bench's launch by algorithmic bytes.  CPU only."""

import importlib.util
import json
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def load_bench():
    spec = importlib.util.spec_from_file_location("bench_traffic_mod", os.path.join(ROOT, "bench.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def test_committed_captures_match_the_kernel_sources():
    b = load_bench()
    h = b.kernel_source_hash()
    for name in ("mixed", "long-user-history"):
        rec = json.load(open(os.path.join(ROOT, "profiles", f"bat_attn_tc_{name}_traffic.json")))
        assert rec["kernel_sha256_16"] == h, f"{name}: capture taken on other kernel sources"
        ratio = rec["dram_bytes_per_launch"] / rec["alg_bytes_per_launch"]
        assert 0.95 <= ratio <= 1.2, f"{name}: measured/algorithmic {ratio}"


def test_traffic_scales_by_algorithmic_bytes(tmp_path, monkeypatch):
    b = load_bench()
    prof = tmp_path / "profiles"
    prof.mkdir()
    current = b.kernel_source_hash()
    rec = {"dram_bytes_per_launch": 3.15e9, "alg_bytes_per_launch": 3.0e9, "kernel_sha256_16": current}
    (prof / "bat_attn_tc_toy_traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(b, "ROOT", str(tmp_path))
    # The kernel sources stay those of the real tree.
    monkeypatch.setattr(b, "kernel_source_hash", lambda: current)
    assert abs(b.traffic_per_launch("toy", 90e9) - 94.5e9) < 1e3
    assert b.traffic_per_launch("absent", 90e9) is None
    rec["kernel_sha256_16"] = "0000000000000000"
    (prof / "bat_attn_tc_toy_traffic.json").write_text(json.dumps(rec))
    assert b.traffic_per_launch("toy", 90e9) is None
