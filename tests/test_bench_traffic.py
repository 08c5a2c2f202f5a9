"""The DRAM traffic that bench.py reports comes from the committed ncu summary of the
indexer call, and only while that summary was taken on the current sources of the kernel
(no GPU): the summary's source hash matches today's files, an edit to one of the listed
sources turns the figure off, and the figure is per launch, close to the call's
algorithmic bytes (a summary far above them would mean re-reads)."""

import json
import os

import bench
from long_context_compressed_layer_b200 import build as b

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SUMMARY = os.path.join(ROOT, "profiles", "indexer_topk_csa_decode_pro_1m.json")


def test_summary_matches_the_current_kernel_sources():
    d = json.load(open(SUMMARY))
    assert d["sources"] and all(
        os.path.exists(os.path.join(b.HERE, "csrc", f)) for f in d["sources"])
    assert d["sources_sha"] == b.sources_sha(d["sources"])
    got = bench.ncu_traffic()
    assert got is not None and got["dram_bytes_per_launch"] == (
        d["dram_bytes_read_per_launch"] + d["dram_bytes_write_per_launch"])
    # per launch of the 1M workload's call: within a few % of its algorithmic bytes
    assert 1.0 <= got["dram_bytes_per_launch"] / got["algorithmic_bytes_per_launch"] < 1.1


def test_an_edited_source_turns_the_figure_off(monkeypatch):
    real = b.sources_sha
    monkeypatch.setattr(b, "sources_sha", lambda files=None: "0" * 16 if files else real())
    assert bench.ncu_traffic() is None


def test_no_summary_means_no_figure(monkeypatch, tmp_path):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.ncu_traffic() is None
