"""bench.py reports counter-measured DRAM bytes only for the workload they were
captured on, and only while the kernel sources hash as they did at the capture:
a changed kernel gets `traffic: null` until its counters are taken again."""
import os
import shutil

import pytest

import bench


def test_every_traffic_entry_names_existing_sources():
    for key, t in bench.TRAFFIC.items():
        assert t["bytes"] > 0, key
        for f in t["sources"]:
            assert os.path.exists(os.path.join(bench.ROOT, "unified_sparse_attention_b200", "csrc", f)), (key, f)


def test_traffic_withheld_off_the_captured_workload():
    for key in bench.TRAFFIC:
        assert bench.traffic(key, False) is None


@pytest.mark.parametrize("key", sorted(bench.TRAFFIC))
def test_traffic_withheld_once_a_hashed_source_changes(key, tmp_path, monkeypatch):
    in_tree = bench.traffic(key, True)
    src = os.path.join(bench.ROOT, "unified_sparse_attention_b200", "csrc")
    dst = tmp_path / "unified_sparse_attention_b200" / "csrc"
    shutil.copytree(src, dst)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic(key, True) == in_tree   # the copy hashes like the tree it came from
    for f in bench.TRAFFIC[key]["sources"]:
        path = dst / f
        original = path.read_bytes()
        path.write_bytes(original + b"\n")
        assert bench.traffic(key, True) is None, f
        path.write_bytes(original)
    # a missing source withholds it too
    (dst / bench.TRAFFIC[key]["sources"][0]).unlink()
    assert bench.traffic(key, True) is None
