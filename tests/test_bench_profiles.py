"""The bench's roofline `traffic` comes from a committed ncu summary only for the workload that summary was
captured on, and only while the summary's recorded kernel-source hash matches the current sources."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _summary_workload(path):
    """The `--workload` a summary's commands run (the default workload when they name none)."""
    for line in open(path):
        if "python bench.py" in line:
            parts = line.split()
            return parts[parts.index("--workload") + 1] if "--workload" in parts else bench.DEFAULT_WORKLOAD
    raise AssertionError(f"{path}: no bench command")


def test_each_summary_is_keyed_by_the_workload_its_commands_run():
    for workload, path in bench.PROFILED_WORKLOADS.items():
        assert os.path.exists(path), path
        assert workload in bench.WORKLOADS
        assert _summary_workload(path) == workload, path


def test_traffic_is_null_for_a_workload_without_its_own_summary():
    src = bench.kernel_source_hash()
    for workload in ("prefix_paged_alibi_fp16", "long_alibi_left_bf16"):
        assert bench.profiled_traffic(workload, src) is None
    assert bench.profiled_traffic("mla_spec_qs4_bf16", bench.kernel_source_hash(bench.MLA_KERNEL_SOURCES)) is None


def test_traffic_is_null_when_the_kernel_source_changed():
    assert bench.profiled_traffic("varlen_causal_bf16", "0" * 16) is None
