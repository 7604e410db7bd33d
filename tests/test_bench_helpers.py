"""bench.py helpers that need no GPU: kernels per C-ABI call, and the DRAM
traffic it reports only from an ncu summary taken on the current sources."""
from __future__ import annotations

import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_two_kernel_split_k_counts_both_launches():
    assert bench.kernels_per_call("dense_nlanes_bn64_st8_gsplit_2k") == 2
    assert bench.kernels_per_call("dense_nlanes_bn64_st4_gsplit_2k_x2") == 2
    assert bench.kernels_per_call("dense_nlanes_bn64_st8_gsplit") == 1
    assert bench.kernels_per_call("dense_mlanes_pair_bn192_st6_f") == 1


def _summary(tmp_path, workload, variant, source_hash, dram):
    d = tmp_path / "profiles"
    d.mkdir(exist_ok=True)
    (d / f"{variant}__{workload}.txt").write_text(
        f"ncu summary: test\nkernel_source_hash: {source_hash}\ndram_bytes_per_launch: {dram}\n")


def test_traffic_only_from_a_summary_of_the_current_sources(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "abc123")
    _summary(tmp_path, "w", "v", "abc123", 1234)
    assert bench.ncu_traffic("w", "v") == 1234.0
    _summary(tmp_path, "w", "v", "stale", 1234)
    assert bench.ncu_traffic("w", "v") is None
    assert bench.ncu_traffic("w", "missing") is None


def test_committed_summaries_name_their_traffic(tmp_path):
    # every committed summary of the current sources states its DRAM bytes
    prof = os.path.join(ROOT, "profiles")
    h = bench.kernel_source_hash()
    for fn in os.listdir(prof):
        text = open(os.path.join(prof, fn)).read()
        if f"kernel_source_hash: {h}" in text:
            assert "dram_bytes_per_launch:" in text, fn
