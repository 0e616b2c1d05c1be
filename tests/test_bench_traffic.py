"""The bench's roofline bookkeeping, host logic only (no GPU): the stored ncu
DRAM traffic is reported only where it applies (the kernel sources it was
captured on, comment edits aside, and the workload whose launch it measured),
and the algorithmic bytes and flops of a pass follow their definitions (one
read of K and V; 4 d flop per visible (token, query) pair, counted here by
brute force)."""

import json
import os

import bench
from kv_cache_eviction_scores_b200 import workloads as W


def _write(tmp_path, entry):
    p = tmp_path / "traffic.json"
    p.write_text(json.dumps({"k_tc_pass1": entry}))
    return str(p)


def test_traffic_only_for_its_sources_and_workload(tmp_path, monkeypatch):
    spec = W.config_spec(3)
    entry = {"bytes_per_launch": 123456789,
             "csrc_sha256": bench.source_hash(bench.KERNEL_SRC["k_tc_pass1"]),
             "workload": bench.workload_desc(spec)}
    monkeypatch.setattr(bench, "TRAFFIC_FILE", _write(tmp_path, entry))
    assert bench.traffic_for("k_tc_pass1", spec) == 123456789.0
    # another workload: its launch moves other bytes
    assert bench.traffic_for("k_tc_pass1", W.config_spec(2)) is None
    # another kernel, or no entry
    assert bench.traffic_for("k_tc_pass2_pair", spec) is None
    # sources changed since the capture
    monkeypatch.setattr(bench, "TRAFFIC_FILE", _write(tmp_path, dict(entry, csrc_sha256="0" * 64)))
    assert bench.traffic_for("k_tc_pass1", spec) is None
    # an entry without a workload is not trusted either
    bare = {k: v for k, v in entry.items() if k != "workload"}
    monkeypatch.setattr(bench, "TRAFFIC_FILE", _write(tmp_path, bare))
    assert bench.traffic_for("k_tc_pass1", spec) is None


def test_source_hash_ignores_comments_only(tmp_path, monkeypatch):
    src = tmp_path / "k.cu"
    monkeypatch.setattr(bench, "CSRC", str(tmp_path))
    src.write_text("// header\nint f() {\n  return 1;  // one\n}\n")
    h0 = bench.source_hash(("k.cu",))
    src.write_text("// another header\n\nint f() {\n  return 1;  // the value one\n}\n")
    assert bench.source_hash(("k.cu",)) == h0
    src.write_text("// header\nint f() {\n  return 2;  // one\n}\n")
    assert bench.source_hash(("k.cu",)) != h0


def test_stored_traffic_names_its_workload():
    with open(os.path.join(os.path.dirname(bench.TRAFFIC_FILE), "ncu_traffic.json")) as f:
        d = json.load(f)
    for kernel, e in d.items():
        assert kernel in bench.KERNEL_SRC
        assert e["workload"] == bench.workload_desc(W.config_spec(3))
        assert e["bytes_per_launch"] == e["dram_read"] + e["dram_write"]


def test_visible_elements_by_brute_force():
    # window query i (0-based) sits at position L - w + i and sees tokens 0 .. L - w + i
    spec = W.Spec("tiny", B=2, Hq=4, Hkv=2, d=8, lengths=[9, 13], window=3, pool=1,
                  keep=[2, 3], dtype="f32")
    brute = 0
    for L in spec.lengths:
        for i in range(spec.window):
            brute += sum(1 for j in range(L) if j <= L - spec.window + i)
    assert bench.visible_elements(spec) == brute * spec.Hq


def test_roofline_of_a_tensor_pass():
    spec = W.config_spec(3)
    us = 200.0
    r = bench.roofline("k_tc_pass2_pair", spec, us, 6650.0, 1590.0, 1965.0)
    nbytes = sum(spec.lengths) * spec.Hkv * spec.d * 2 * 2  # one read of K and V, bf16
    assert nbytes == 536870912
    assert abs(r["achieved"] - nbytes / (us * 1e-6) / 1e9) < 1e-6
    assert abs(r["frac"] - r["achieved"] / 6650.0) < 1e-12
    flops = 4 * spec.d * bench.visible_elements(spec)
    assert abs(r["tensor"]["achieved"] - flops / (us * 1e-6) / 1e12) < 1e-9
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
