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


def test_committed_traffic_is_reported_only_for_the_code_it_was_measured_on():
    """The stored DRAM traffic of a kernel is returned exactly when its capture's code identity
    equals the current kernel code's; otherwise the benchmark reports null (stale counters)."""
    with open(bench.TRAFFIC_FILE) as f:
        d = json.load(f)
    current = bench.kernel_source_hash()
    for kernel in ("gemm", "quant_down", "gemm_int4", "quant_down_int4"):
        e = d[kernel][bench.DEFAULT_WORKLOAD]
        t = bench.stored_traffic(kernel, bench.DEFAULT_WORKLOAD)
        if e["source_sha256"] == current:
            assert t == e["dram_bytes_per_launch"]
        else:
            assert t is None


def test_traffic_is_null_for_other_code(monkeypatch, tmp_path):
    _with_sources(monkeypatch, tmp_path, ["int changed = 1;\n"])
    assert bench.stored_traffic("gemm", bench.DEFAULT_WORKLOAD) is None
