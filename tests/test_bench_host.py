"""Host logic of bench.py that needs no GPU: the committed DRAM-traffic table
is honoured only while the kernel sources it was measured on are unchanged."""
import json
import os
import shutil

import pytest

import bench


def _copy_tree(tmp_path):
    root = tmp_path / "repo"
    shutil.copytree(os.path.join(bench.ROOT, "profiles"), root / "profiles")
    shutil.copytree(os.path.join(bench.ROOT, "long_context_bidirectional_b200", "csrc"),
                    root / "long_context_bidirectional_b200" / "csrc")
    return root


def test_traffic_table_entries_name_their_sources():
    with open(os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        table = json.load(f)
    assert table
    for kernel, per_workload in table.items():
        for workload, ent in per_workload.items():
            assert ent["bytes_per_launch"] > 0
            assert ent["sources"] and len(ent["sources_sha256_16"]) == 16
            for name in ent["sources"]:
                assert os.path.exists(os.path.join(bench.ROOT, "long_context_bidirectional_b200", "csrc", name))


def test_traffic_is_dropped_once_a_source_changes(tmp_path, monkeypatch):
    root = _copy_tree(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(root))
    with open(root / "profiles" / "traffic.json") as f:
        table = json.load(f)
    kernel, per_workload = next(iter(table.items()))
    workload, ent = next(iter(per_workload.items()))
    in_copy = bench.committed_traffic(kernel, workload)
    monkeypatch.undo()
    # the copy is byte-identical: the entry holds there exactly when it holds in the repository
    assert in_copy == bench.committed_traffic(kernel, workload)
    monkeypatch.setattr(bench, "ROOT", str(root))
    src = root / "long_context_bidirectional_b200" / "csrc" / ent["sources"][-1]
    src.write_bytes(src.read_bytes() + b"\n// edited\n")
    assert bench.committed_traffic(kernel, workload) is None


def test_unknown_kernel_or_workload_has_no_traffic():
    assert bench.committed_traffic("no_such_kernel<0>", "s32768_h32_d128_qsig4") is None
    assert bench.committed_traffic("attn_pair_kernel<0>", "no_such_workload") is None


class _FakeLib:
    ATTN_KERNEL_SINGLE, ATTN_KERNEL_PAIR = 1, 2

    def __init__(self, choice):
        self.choice = choice

    def attn_kernel_for(self, d, skv):
        return self.choice


@pytest.mark.parametrize("choice,mode,name", [
    (2, 0, "attn_pair_kernel<0>"), (2, 1, "attn_pair_kernel<1>"),
    (1, 0, "attn_fwd_kernel<128, 0, 0>"), (1, 1, "attn_fwd_kernel<128, 1, 0>"), (1, 2, "attn_fwd_kernel<128, 2, 0>"),
])
def test_kernel_names_match_the_launch_list(choice, mode, name):
    assert bench.attn_kernel_name(_FakeLib(choice), 128, 4096, mode) == name


def test_merge_kernel_names():
    assert bench.merge_kernel_name(128, 8, "float") == "attn_merge_pipe_kernel<128, float>"
    assert bench.merge_kernel_name(128, 16, "float") == "attn_merge_pipe_kernel<128, float>"
    assert bench.merge_kernel_name(64, 17, "float") == "attn_merge_kernel<64, float>"
