"""Host-side pieces of bench.py that need no GPU: the digest that decides
whether recorded DRAM traffic still describes the kernels, and the lookup."""

import os
import shutil
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _copy_tree(tmp_path):
    dst = tmp_path / "tensor_layer_reconciliation_b200" / "csrc"
    shutil.copytree(os.path.join(ROOT, "tensor_layer_reconciliation_b200", "csrc"), dst)
    return dst


def test_digest_ignores_comments_but_not_code(tmp_path, monkeypatch):
    base = bench._kernel_source_digest()
    csrc = _copy_tree(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench._kernel_source_digest() == base
    f = csrc / "tp_common.cuh"
    text = f.read_text()
    f.write_text("// a new comment line\n/* and a block\n   comment */\n" + text.replace("\n", "\n\n", 3))
    assert bench._kernel_source_digest() == base          # comments and blank space only
    f.write_text(text.replace("kWaitLimitNs = 2000000000ull", "kWaitLimitNs = 1000000000ull"))
    assert bench._kernel_source_digest() != base          # code changed


def test_profiled_traffic_lookup():
    assert bench._profiled_traffic("no_such_workload", "tensor") is None
    for (workload, path), (nbytes, digest, summary) in bench.PROFILED_TRAFFIC.items():
        assert nbytes > 0 and len(digest) == 16
        assert os.path.exists(os.path.join(ROOT, summary)), summary
        if digest == bench._kernel_source_digest():
            assert bench._profiled_traffic(workload, path) == nbytes
