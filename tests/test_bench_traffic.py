"""The bench reports a kernel's DRAM traffic only while its sources are the ones the counters
were captured from (profiles/traffic.json keys each entry by a hash of those sources)."""
import json
import os
import shutil

import bench


def _tree(tmp_path):
    """A copy of the kernel sources and the committed traffic file under tmp_path."""
    src = os.path.join(bench.ROOT, "shifted_sparse_attention_fwd_b200", "csrc")
    dst = tmp_path / "shifted_sparse_attention_fwd_b200" / "csrc"
    shutil.copytree(src, dst)
    (tmp_path / "profiles").mkdir()
    shutil.copy(os.path.join(bench.ROOT, "profiles", "traffic.json"), tmp_path / "profiles")
    return dst


def test_traffic_follows_the_sources(tmp_path, monkeypatch):
    csrc = _tree(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    with open(tmp_path / "profiles" / "traffic.json") as f:
        table = json.load(f)["llama7b_n8192_g2048"]
    for kernel, entry in table.items():
        # the committed counters belong to the committed sources
        assert bench.kernel_source_hash(kernel) == entry["source_hash"], kernel
        assert bench.load_traffic(kernel, "llama7b_n8192_g2048") == entry["bytes_per_launch"]
    # editing a kernel's own source makes its counters stale, and only its own
    with open(csrc / "s2_bwd_pre.cuh", "a") as f:
        f.write("\n// edited\n")
    assert bench.load_traffic("s2_bwd_pre", "llama7b_n8192_g2048") is None
    assert bench.load_traffic("s2_fwd", "llama7b_n8192_g2048") == table["s2_fwd"]["bytes_per_launch"]
    # a shared header makes every kernel's counters stale
    with open(csrc / "s2_device.cuh", "a") as f:
        f.write("\n// edited\n")
    assert all(bench.load_traffic(k, "llama7b_n8192_g2048") is None for k in table)


def test_no_traffic_for_unknown_workload_or_missing_file(tmp_path, monkeypatch):
    _tree(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.load_traffic("s2_fwd", "no_such_workload") is None
    os.remove(tmp_path / "profiles" / "traffic.json")
    assert bench.load_traffic("s2_fwd", "llama7b_n8192_g2048") is None
