"""Host-side bookkeeping of bench.py (no GPU): the DRAM-traffic figures are
keyed to each kernel's own sources."""

import json

import bench


def test_kernel_source_lists_name_existing_files():
    pkg = bench.ROOT / "test_sequence_layers_02_b200" / "csrc"
    for key, files in bench._KERNEL_SOURCES.items():
        for f in files:
            assert (pkg / f).exists(), (key, f)
    # the tensor-core and decode kernels share one translation unit
    assert bench._kernel_hash("scan_tc") == bench._kernel_hash("decode_step")
    assert bench._kernel_hash("scan_cluster") != bench._kernel_hash("scan_tc")


def test_traffic_is_null_once_a_kernels_sources_differ(tmp_path, monkeypatch):
    f = tmp_path / "traffic.json"
    f.write_text(json.dumps({"csrc_hash": "x", "kernels": {
        "scan_tc": {"bytes_per_head_token": 500.0, "sources_hash": bench._kernel_hash("scan_tc")},
        "scan_cluster": {"bytes_per_head_token": 800.0, "sources_hash": "0" * 16},
    }}))
    monkeypatch.setattr(bench, "PROFILE_TRAFFIC", f)
    assert bench._traffic("scan_tc", 1000) == 500000
    assert bench._traffic("scan_cluster", 1000) is None      # sources changed since
    assert bench._traffic("decode_step", 1000) is None       # never captured
