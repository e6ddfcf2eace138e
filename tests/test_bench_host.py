"""Host-side helpers of bench.py (CPU only): the hash of the CUDA sources'
code, which decides whether the committed ncu traffic figures still apply,
and the reading of those figures."""
import os
import shutil
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


@pytest.fixture()
def tree(tmp_path, monkeypatch):
    """A copy of the CUDA sources and of the traffic summary under a temporary root."""
    src = os.path.join(ROOT, "flash_attention_tiled_b200", "csrc")
    dst = tmp_path / "flash_attention_tiled_b200" / "csrc"
    shutil.copytree(src, dst, ignore=shutil.ignore_patterns("*.so", "*.o"))
    (tmp_path / "profiles").mkdir()
    shutil.copy(os.path.join(ROOT, "profiles", "dram_traffic__bench_calls.md"), tmp_path / "profiles")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    return tmp_path


def _edit(path, old, new):
    text = path.read_text()
    assert old in text
    path.write_text(text.replace(old, new, 1))


def test_source_hash_ignores_comments_and_whitespace(tree):
    before = bench.source_sha()
    f = tree / "flash_attention_tiled_b200" / "csrc" / "merge_lse.cuh"
    _edit(f, "// One warp per row;", "// (reworded) One warp per row;")
    _edit(f, "#pragma once\n", "#pragma once\n\n/* a new block comment */\n\n")
    assert bench.source_sha() == before


def test_source_hash_follows_code(tree):
    before = bench.source_sha()
    f = tree / "flash_attention_tiled_b200" / "csrc" / "merge_lse.cuh"
    _edit(f, "constexpr int kMergeWarps = 8;", "constexpr int kMergeWarps = 4;")
    assert bench.source_sha() != before


def test_traffic_figures_apply_only_to_the_profiled_code(tree):
    summary = tree / "profiles" / "dram_traffic__bench_calls.md"
    text = summary.read_text()
    # point the summary at the copied sources' hash: the figures are read back
    lines = [ln for ln in text.splitlines() if not ln.startswith("source-sha256:")]
    summary.write_text("\n".join(lines + [f"source-sha256: {bench.source_sha()}", ""]))
    tr = bench.profiled_traffic()
    assert set(tr) >= {"prefill", "paged", "long", "contig"}
    assert all(v > 0 for v in tr.values())
    # a code change retires them
    _edit(tree / "flash_attention_tiled_b200" / "csrc" / "merge_lse.cuh",
          "constexpr int kMergeWarps = 8;", "constexpr int kMergeWarps = 4;")
    assert bench.profiled_traffic() == {}


def test_traffic_summary_missing_reads_as_none(tree):
    os.remove(tree / "profiles" / "dram_traffic__bench_calls.md")
    assert bench.profiled_traffic() == {}
