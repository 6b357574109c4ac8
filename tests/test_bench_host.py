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
    for (workload, path), (nbytes, digest, capture) in bench.PROFILED_TRAFFIC.items():
        assert nbytes > 0 and len(digest) == 16
        assert workload in capture and "kernel" in capture, capture   # names kernel and workload
        if digest == bench._kernel_source_digest():
            assert bench._profiled_traffic(workload, path) == nbytes


def test_configs_to_run():
    args = type("A", (), {"config": "all", "weights": "bf16"})()
    assert bench._configs_to_run(args) == bench.BENCH_CONFIGS
    assert bench.BENCH_CONFIGS[0] == bench.HEADLINE_CONFIG
    args.weights = "mxfp8"                              # MXFP8 shards run every workload
    assert bench._configs_to_run(args) == bench.BENCH_CONFIGS
    args.config, args.weights = "prefill_n4", "bf16"
    assert bench._configs_to_run(args) == ["prefill_n4"]


def test_sample_cols_cover_chunk_edges():
    cols = bench._sample_cols(5120, 4, 40, seed=3)
    for c in range(4):
        assert {c * 1280, c * 1280 + 1279} <= set(cols.tolist())
    assert cols.min() >= 0 and cols.max() < 5120 and len(set(cols.tolist())) == len(cols)


def test_reference_arm_config_keys_match_gpu_arm():
    cfg = bench.get_config("decode_n2")
    args = type("A", (), {"weights": "bf16", "variant": "auto"})()
    ref_keys = set(bench._config_keys(cfg, 1, args))
    assert {"workload", "n_ranks", "tokens", "hidden", "points", "l2", "weights",
            "variant", "parallelism"} <= ref_keys


def test_oracle_parity_counts_on_the_cpu():
    """The bench's parity leg on a stand-in workload whose outputs are the
    oracle's own (all counts zero), then with one output flipped by one bf16
    unit at a non-fragile position (counted as differing and not fragile)."""
    import numpy as np
    import torch

    import oracle
    from workloads import KIND_RESIDUAL, KIND_W, KIND_X, point_tensor

    cfg = bench.get_config("tiny")
    outs = []
    for p in cfg.points:
        bits = [point_tensor(cfg, p, kd).view(torch.int16).numpy().view(np.uint16)
                for kd in (KIND_X, KIND_W, KIND_RESIDUAL)]
        ref = oracle.reconcile(cfg.n_ranks, cfg.hidden, *bits)
        outs.append(torch.from_numpy(ref["out"].view(np.int16).copy()).view(torch.bfloat16))

    class Stand:
        def __init__(self):
            self.cfg, self.device, self.weights = cfg, torch.device("cpu"), "bf16"

        def out(self, i):
            return outs[i]

    st = bench.oracle_parity(Stand(), threads=2)
    assert st["outputs_differing"] == 0 and st["max_abs"] == 0.0 and st["rel_l2"] == 0.0
    assert st["within_tolerance"] and st["sampled_outputs"] > 0
    col = int(bench._sample_cols(cfg.hidden, cfg.n_ranks, 40, seed=len(cfg.name))[0])
    o = outs[0].view(torch.int16)
    o[0, col] += 1                                    # one unit of the last place
    st = bench.oracle_parity(Stand(), threads=2)
    assert st["outputs_differing"] == 1
    assert st["differing_not_fragile"] in (0, 1) and st["max_abs"] > 0
    assert st["rel_l2"] > 0
