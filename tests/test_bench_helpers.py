"""CPU checks of the benchmark's bookkeeping: the kernel-code identity that guards the committed
ncu traffic figures, and the lookup of those figures."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _with_sources(monkeypatch, tmp_path, texts):
    paths = []
    for i, t in enumerate(texts):
        p = tmp_path / f"src{i}.cu"
        p.write_text(t)
        paths.append(str(p))
    monkeypatch.setattr(bench, "KERNEL_SOURCES", paths)
    return bench.kernel_source_hash()


def test_source_identity_ignores_comments_and_blank_lines(monkeypatch, tmp_path):
    base = _with_sources(monkeypatch, tmp_path, ["int a = 1;\n/* note */\nint b = 2;  // two\n", "x();\n"])
    same = _with_sources(monkeypatch, tmp_path, ["int a = 1;\n\n\nint b = 2;\n// another note\n", "x();  \n"])
    assert base == same


def test_source_identity_changes_with_code_in_any_file(monkeypatch, tmp_path):
    base = _with_sources(monkeypatch, tmp_path, ["int a = 1;\n", "x();\n"])
    assert _with_sources(monkeypatch, tmp_path, ["int a = 2;\n", "x();\n"]) != base
    assert _with_sources(monkeypatch, tmp_path, ["int a = 1;\n", "y();\n"]) != base
    # a string that contains "//" is code, not a comment
    assert _with_sources(monkeypatch, tmp_path, ['s("a//b");\n', "x();\n"]) != \
        _with_sources(monkeypatch, tmp_path, ['s("a//c");\n', "x();\n"])


def test_committed_traffic_matches_the_current_kernels():
    with open(bench.TRAFFIC_FILE) as f:
        d = json.load(f)
    for kernel in ("gemm", "quant_down"):
        t = bench.stored_traffic(kernel, bench.DEFAULT_WORKLOAD)
        assert t is not None and t == d[kernel][bench.DEFAULT_WORKLOAD]["dram_bytes_per_launch"]


def test_traffic_is_null_for_other_code(monkeypatch, tmp_path):
    _with_sources(monkeypatch, tmp_path, ["int changed = 1;\n"])
    assert bench.stored_traffic("gemm", bench.DEFAULT_WORKLOAD) is None
