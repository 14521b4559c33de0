"""Host logic of bench.py that needs no GPU: the DRAM-traffic figure it reports for the
streaming kernel is taken from a committed ncu summary only while that summary was captured
on the streaming kernel's current sources."""
import json
import os
import shutil

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture()
def tree(tmp_path, monkeypatch):
    """A copy of the sources and of the traffic record, with bench.py pointed at it."""
    import sys
    sys.path.insert(0, ROOT)
    import bench
    shutil.copytree(os.path.join(ROOT, "store_kv_attention_b200", "csrc"), tmp_path / "store_kv_attention_b200" / "csrc")
    shutil.copytree(os.path.join(ROOT, "include"), tmp_path / "include")
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    sha = bench.kernel_source_sha()
    rec = {"int4_2b": {"source_sha": sha, "dram_bytes_per_launch": 12345}}
    (tmp_path / "profiles" / "stream_kernel_traffic.json").write_text(json.dumps(rec))
    return bench, tmp_path


def _touch(path):
    with open(path, "a") as f:
        f.write("\n// edited\n")


def test_record_is_used_for_current_sources(tree):
    bench, _ = tree
    assert bench.recorded_traffic("int4_2b") == 12345
    assert bench.recorded_traffic("int8_b16") is None  # no capture for that workload


@pytest.mark.parametrize("rel", ["store_kv_attention_b200/csrc/k_stream_tc.cu",
                                 "store_kv_attention_b200/csrc/tc_ptx.cuh",
                                 "store_kv_attention_b200/csrc/tl_internal.cuh",
                                 "include/tl_storeh.h"])
def test_edit_to_streaming_sources_voids_record(tree, rel):
    bench, root = tree
    _touch(root / rel)
    assert bench.recorded_traffic("int4_2b") is None


@pytest.mark.parametrize("rel", ["store_kv_attention_b200/csrc/k_proj_tc.cu",
                                 "store_kv_attention_b200/csrc/cluster_ptx.cuh",
                                 "store_kv_attention_b200/csrc/k_append.cu"])
def test_edit_elsewhere_keeps_record(tree, rel):
    bench, root = tree
    _touch(root / rel)
    assert bench.recorded_traffic("int4_2b") == 12345

