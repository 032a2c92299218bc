"""The bench's recorded DRAM traffic (CPU): reported only while the kernel
sources it was captured on are unchanged."""
import json
import os

import bench


def test_recorded_traffic_is_reported_only_for_current_sources():
    path = os.path.join(bench.ROOT, "profiles", "indexer_topk_decode_b64_t128k.json")
    with open(path) as f:
        rec = json.load(f)
    if rec["kernel_source_hash"] == bench.kernel_source_hash():
        assert bench.recorded_traffic("decode_b64_t128k") == float(rec["dram_bytes_per_call"])
    else:                                                   # captured on other kernel sources: not reported
        assert bench.recorded_traffic("decode_b64_t128k") is None
    assert bench.recorded_traffic("no_such_workload") is None


def test_recorded_traffic_is_null_once_a_kernel_source_changes(tmp_path, monkeypatch):
    pkg = tmp_path / "compressed_sparse_attention_quant_b200"
    (pkg / "csrc").mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    for rel in bench.KERNEL_SOURCES:
        src = os.path.join(bench.ROOT, "compressed_sparse_attention_quant_b200", rel)
        (pkg / rel).write_bytes(open(src, "rb").read())
    rec = json.load(open(os.path.join(bench.ROOT, "profiles", "indexer_topk_decode_b64_t128k.json")))
    rec["kernel_source_hash"] = bench.kernel_source_hash()          # a record taken on these sources
    (tmp_path / "profiles" / "indexer_topk_decode_b64_t128k.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.recorded_traffic("decode_b64_t128k") == float(rec["dram_bytes_per_call"])
    edited = pkg / bench.KERNEL_SOURCES[-1]
    edited.write_bytes(edited.read_bytes() + b"\n// edited\n")
    assert bench.recorded_traffic("decode_b64_t128k") is None
