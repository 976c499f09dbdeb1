"""Host-side arithmetic of the benchmark (no GPU): algorithmic bytes, the roofline's traffic record and
the whole-job throughput."""
import json
import os

import bench


def test_algorithmic_bytes_of_the_llama_shaped_head():
    # centroids c*d*2 + token rows p*b*d*2 + C2T rows p*b*4 + h d*2 + the token 4
    assert bench.algorithmic_bytes(128256, 2048, 8016, 16, 512) == 66424836
    # INT4 rows: d/2 code bytes + d/16 scale bytes per centroid
    assert bench.algorithmic_bytes(128256, 2048, 8016, 16, 512, crow_bytes=1024 + 128) == \
        8016 * 1152 + 512 * 16 * 2048 * 2 + 512 * 16 * 4 + 2048 * 2 + 4


def test_traffic_record_is_used_only_for_the_kernels_it_was_taken_on(monkeypatch):
    with open(os.path.join(bench.PROFILE_DIR, "decode_b1_llama1b.json")) as f:
        rec = json.load(f)
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: rec["kernel_source_hash"])
    assert bench.measured_traffic("decode_b1_llama1b") == rec["dram_bytes_per_launch"]
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "0" * 16)
    assert bench.measured_traffic("decode_b1_llama1b") is None
    assert bench.measured_traffic("no_such_profile") is None


def test_traffic_record_is_consistent():
    # the committed ncu record names the source hash it was taken on (bench.py reports its
    # traffic only while that hash matches the tree) and its read + write bytes add up
    with open(os.path.join(bench.PROFILE_DIR, "decode_b1_llama1b.json")) as f:
        rec = json.load(f)
    assert len(rec["kernel_source_hash"]) == 16 and int(rec["kernel_source_hash"], 16) >= 0
    assert rec["dram_bytes_per_launch"] == rec["dram_bytes_read_per_launch"] + rec["dram_bytes_write_per_launch"]
    assert "hash_note" not in rec


def test_job_throughput_uses_the_slowest_rank():
    # 2 ranks x 1000 steps in 50 ms (the slower rank's time) = 40000 tokens/s
    assert bench.job_throughput(50.0, 1000, 2) == 40000.0
