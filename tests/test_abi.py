"""The C-ABI library: loads, exports every function include/*.h declares, and
rejects bad host-side arguments before touching the GPU. Runs without a GPU."""

import ctypes
import glob
import os
import re

import pytest

import oracle
from helpers import golden_rows

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        names += re.findall(r"TP_API\s+[\w\s\*]+?\b(tp_\w+)\s*\(", text)
    return sorted(set(names))


def test_library_exports_every_declared_symbol():
    import tensor_layer_reconciliation_b200 as tlr
    declared = _declared()
    assert len(declared) >= 12
    lib = ctypes.CDLL(tlr.LIB_PATH)
    for name in declared:
        assert hasattr(lib, name), name
    assert sorted(tlr.EXPORTED) == declared


def test_ring_bytes_matches_pages_and_oracle():
    import tensor_layer_reconciliation_b200 as tlr
    for n, m, h, e, pts, want in golden_rows("ring_bytes.txt"):
        assert tlr.tp_ring_bytes(int(n), int(m), int(h), int(e), int(pts)) == int(want)
    for n in range(1, 9):
        for m, h, pts in [(1, 5120, 128), (32, 5120, 128), (64, 4096, 96), (4096, 5120, 1)]:
            assert tlr.tp_ring_bytes(n, m, h, 2, pts) == oracle.ring_bytes(n, m, h, 2, pts)
    assert tlr.tp_ring_bytes(0, 1, 8, 2, 1) == 0
    assert tlr.tp_ring_bytes(2, -1, 8, 2, 1) == 0


def test_status_strings():
    import tensor_layer_reconciliation_b200 as tlr
    for s in range(6):
        assert tlr.tp_status_string(s)
    assert tlr.tp_status_string(99) == "unknown status"


@pytest.mark.parametrize("args,status", [
    ((0, 1, 1024, 256), 1),        # N < 1
    ((9, 1, 1024, 256), 1),        # N > 8
    ((3, 1, 1024, 256), 1),        # K % N
    ((2, 1, 1000, 256), 1),        # (K/N) % 8
    ((2, 1, 1024, 252), 1),        # (H/N) % 8
    ((2, -1, 1024, 256), 1),       # negative max_tokens
])
def test_plan_create_rejects_bad_shapes(args, status):
    import tensor_layer_reconciliation_b200 as tlr
    st, h = tlr.tp_plan_create(*args)
    assert st == status and h is None


def test_plan_create_rejects_dtype_and_null():
    import tensor_layer_reconciliation_b200 as tlr
    from tensor_layer_reconciliation_b200 import _lib
    st, _ = tlr.tp_plan_create(2, 1, 1024, 256, dtype=7)
    assert st == tlr.TP_ERR_UNSUPPORTED
    assert _lib.LIB.tp_plan_create(None, 2, 1, 1024, 256, 0) == tlr.TP_ERR_INVALID


def test_null_plan_everywhere():
    import tensor_layer_reconciliation_b200 as tlr
    INV = tlr.TP_ERR_INVALID
    assert tlr.tp_plan_set_variant(None, 0, 0) == INV
    assert tlr.tp_plan_workspace_bytes(None, 4) == 0
    assert tlr.tp_plan_kernel_variant(None, 4) == -1
    assert tlr.tp_plan_launches(None, 4) == -1
    assert tlr.tp_plan_mxfp8_bytes(None)[0] == INV
    assert tlr.tp_pack_weights_mxfp8(None, 16, 32, 48, 0) == INV
    assert tlr.tp_rowlinear_reconcile_mxfp8(None, 16, 32, 48, 64, 80, 1, 0, 0) == INV
    assert tlr.tp_plan_mxfp8_workspace_bytes(None, 4) == 0
    assert tlr.tp_plan_nvfp4_bytes(None)[0] == INV
    assert tlr.tp_pack_weights_nvfp4(None, 16, 32, 48, 0) == INV
    assert tlr.tp_plan_nvfp4_workspace_bytes(None, 4) == 0
    assert tlr.tp_rowlinear_reconcile_nvfp4(None, 16, 32, 48, 64, 80, 1, 0, 0) == INV
    assert tlr.tp_pack_weights(None, 16, 32, 0) == INV
    assert tlr.tp_rowlinear_reconcile(None, 16, 32, 48, 64, 1, 0, 0) == INV
    assert tlr.tp_rowlinear_partials(None, 16, 32, 48, 1, 0) == INV
    assert tlr.tp_ring_reduce(None, 16, 32, 48, 1, 0) == INV
    assert tlr.tp_device_error_flags(None)[0] == INV
    assert tlr.tp_ring_rank_workspace_bytes(None, 4) == 0
    assert tlr.tp_ring_allreduce_ranks(None, [16, 32], 48, [64, 80], [96, 112], 0, 2, 1, 0, 0) == INV
    tlr.tp_plan_destroy(None)          # NULL-safe


def test_product_does_not_import_oracle():
    pkg = os.path.join(ROOT, "tensor_layer_reconciliation_b200")
    for f in glob.glob(os.path.join(pkg, "**", "*"), recursive=True):
        if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
            text = open(f).read()
            assert not re.search(r"^\s*(import|from)\s+oracle", text, re.M), f
            assert "liboracle" not in text and "oracle.c" not in text, f


@pytest.mark.parametrize("scheme", ["ring", "naive", "sharp"])
def test_allreduce_bytes_matches_oracle(scheme):
    """The library's all-reduce byte model (host code) against the oracle's
    message count, over rank counts, shapes and bad arguments."""
    import oracle
    import tensor_layer_reconciliation_b200 as tlr
    code = {"ring": tlr.TP_ALLREDUCE_RING, "naive": tlr.TP_ALLREDUCE_NAIVE,
            "sharp": tlr.TP_ALLREDUCE_SWITCH}[scheme]
    for n in range(0, 10):
        for m, h, e, pts in [(1, 5120, 2, 128), (32, 5120, 2, 128), (3, 840, 4, 7), (0, 5, 2, 1),
                             (64, 4096, 2, 96), (5, 7, 1, 3), (2, -1, 2, 1)]:
            assert tlr.tp_allreduce_bytes(code, n, m, h, e, pts) == \
                oracle.allreduce_bytes(scheme, n, m, h, e, pts), (n, m, h, e, pts)
    assert tlr.tp_allreduce_bytes(code, 4, 1, 5120, 2, 128) == \
        oracle.allreduce_bytes(scheme, 4, 1, 5120, 2, 128)
    assert tlr.tp_allreduce_bytes(9, 4, 1, 5120, 2, 128) == 0


@pytest.mark.parametrize("scheme", ["ring", "naive", "sharp"])
def test_moe_combine_bytes_matches_oracle(scheme):
    """The library's MoE-combine byte model (host code) against the oracle's
    buffer-by-buffer count, with and without the local accumulation."""
    import tensor_layer_reconciliation_b200 as tlr
    code = {"ring": tlr.TP_ALLREDUCE_RING, "naive": tlr.TP_ALLREDUCE_NAIVE,
            "sharp": tlr.TP_ALLREDUCE_SWITCH}[scheme]
    for n in range(0, 10):
        for m, h, e, k in [(1, 5120, 2, 8), (64, 4096, 2, 8), (3, 840, 4, 1), (0, 5, 2, 2),
                           (5, 7, 1, 3), (2, -1, 2, 2), (4, 16, 2, 0)]:
            for local in (0, 1):
                assert tlr.tp_moe_combine_bytes(code, n, m, h, e, k, local) == \
                    oracle.moe_combine_bytes(scheme, n, m, h, e, k, bool(local)), (n, m, h, e, k, local)
    assert tlr.tp_moe_combine_bytes(code, 4, 1, 16, 2, 2, 2) == 0
