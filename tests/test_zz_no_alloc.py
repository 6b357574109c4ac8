"""The entry point for callers that cannot allocate device memory.

tp_rowlinear_reconcile_noalloc takes no workspace: the partials it stages go
to a fixed scratch array inside the library. Its result must equal that of
tp_rowlinear_reconcile with a caller-supplied workspace, call after call
(the array keeps the previous call's contents, so two calls in a row with
different inputs are compared), and a call that would need more scratch
than the array holds must be refused before anything is launched.

This file is collected last so that a run stopping at the first failure has
already run every other test.
"""

import pytest
import torch

from gpu_util import inputs

pytestmark = pytest.mark.gpu


def _ptr(t):
    return t.data_ptr()


def test_noalloc_matches_workspace_entry_point_twice():
    import tensor_layer_reconciliation_b200 as tlr
    dev = torch.device("cuda")
    n, m, k, h = 4, 32, 1024, 512          # 32 tokens: the tensor-core path stages partials
    plan = tlr.Plan(n, m, k, h)            # AUTO
    need = plan.workspace_bytes(m)
    assert need > 0, "the case must exercise the staged (scratch-using) path"
    stream = torch.cuda.current_stream().cuda_stream
    for call, seed in enumerate((11, 12)):
        x, w, r = inputs(n, m, k, h, seed, dev)
        wp = plan.pack_weights(w)
        out_ref = torch.empty(m, h, dtype=torch.bfloat16, device=dev)
        ws = torch.zeros(need, dtype=torch.uint8, device=dev)
        st = tlr.tp_rowlinear_reconcile(plan.handle, _ptr(x), _ptr(wp), _ptr(r), _ptr(out_ref), m,
                                        _ptr(ws), stream)
        assert st == tlr.TP_OK
        out = torch.full((m, h), float("nan"), dtype=torch.bfloat16, device=dev)
        st = tlr.tp_rowlinear_reconcile_noalloc(plan.handle, _ptr(x), _ptr(wp), _ptr(r), _ptr(out),
                                                m, stream)
        assert st == tlr.TP_OK
        torch.cuda.synchronize()
        assert plan.device_error_flags() == 0
        # same kernels on the same inputs: identical bits
        assert torch.equal(out.view(torch.int16), out_ref.view(torch.int16)), f"call {call}"


def test_noalloc_single_token_fold_twice():
    """One token: the tensor-core kernel folds in place, using counters at
    the start of the scratch array that each call must leave at zero."""
    import tensor_layer_reconciliation_b200 as tlr
    dev = torch.device("cuda")
    n, m, k, h = 2, 1, 4096, 1024
    plan = tlr.Plan(n, m, k, h)            # AUTO
    assert plan.launches(m) == 1 and plan.workspace_bytes(m) > 0
    stream = torch.cuda.current_stream().cuda_stream
    for call, seed in enumerate((21, 22)):
        x, w, r = inputs(n, m, k, h, seed, dev)
        wp = plan.pack_weights(w)
        ref = plan.reconcile(x, wp, r)
        out = torch.full((m, h), float("nan"), dtype=torch.bfloat16, device=dev)
        st = tlr.tp_rowlinear_reconcile_noalloc(plan.handle, _ptr(x), _ptr(wp), _ptr(r), _ptr(out),
                                                m, stream)
        assert st == tlr.TP_OK
        torch.cuda.synchronize()
        assert plan.device_error_flags() == 0
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16)), f"call {call}"


def test_noalloc_fused_path_needs_no_scratch():
    import tensor_layer_reconciliation_b200 as tlr
    dev = torch.device("cuda")
    n, m, k, h = 2, 1, 512, 256            # the fused exact path stages nothing
    plan = tlr.Plan(n, m, k, h, variant="exact")
    assert plan.workspace_bytes(m) == 0
    x, w, r = inputs(n, m, k, h, 13, dev)
    wp = plan.pack_weights(w)
    ref = plan.reconcile(x, wp, r)
    out = torch.empty_like(ref)
    st = tlr.tp_rowlinear_reconcile_noalloc(plan.handle, _ptr(x), _ptr(wp), _ptr(r), _ptr(out), m,
                                            torch.cuda.current_stream().cuda_stream)
    assert st == tlr.TP_OK
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))


def test_noalloc_zero_tokens_tensor_plan():
    """Zero tokens with the tensor-core variant chosen explicitly: nothing to
    launch, TP_OK, and no work-size arithmetic on an empty token range."""
    import tensor_layer_reconciliation_b200 as tlr
    plan = tlr.Plan(4, 8, 1024, 512, variant="tensor")
    st = tlr.tp_rowlinear_reconcile_noalloc(plan.handle, 0, 0, 0, 0, 0,
                                            torch.cuda.current_stream().cuda_stream)
    assert st == tlr.TP_OK
    assert plan.launches(0) == 0 and plan.workspace_bytes(0) == 0


def test_noalloc_staged_exact_twice():
    """The exact variant with staged partials: its partials go through the
    scratch array and a ring kernel; bit-identical to the workspace form."""
    import tensor_layer_reconciliation_b200 as tlr
    dev = torch.device("cuda")
    n, m, k, h = 4, 3, 1024, 512
    plan = tlr.Plan(n, m, k, h, variant="exact", staged=True)
    assert plan.workspace_bytes(m) > 0
    stream = torch.cuda.current_stream().cuda_stream
    for call, seed in enumerate((41, 42)):
        x, w, r = inputs(n, m, k, h, seed, dev)
        wp = plan.pack_weights(w)
        ref = plan.reconcile(x, wp, r)
        out = torch.full((m, h), float("nan"), dtype=torch.bfloat16, device=dev)
        st = tlr.tp_rowlinear_reconcile_noalloc(plan.handle, _ptr(x), _ptr(wp), _ptr(r), _ptr(out),
                                                m, stream)
        assert st == tlr.TP_OK
        torch.cuda.synchronize()
        assert plan.device_error_flags() == 0
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16)), f"call {call}"


def test_noalloc_refuses_more_than_its_scratch():
    import tensor_layer_reconciliation_b200 as tlr
    n, m, k, h = 4, 4096, 1024, 5120       # N*M*H*2 = 168 MB > 16 MiB
    plan = tlr.Plan(n, m, k, h)
    assert plan.workspace_bytes(m) > 16 << 20
    # refused on the host before any pointer is touched or any kernel launched
    st = tlr.tp_rowlinear_reconcile_noalloc(plan.handle, 256, 512, 768, 1024, m, 0)
    assert st == tlr.TP_ERR_WORKSPACE
    assert tlr.tp_rowlinear_reconcile_noalloc(None, 256, 512, 768, 1024, 1, 0) == tlr.TP_ERR_INVALID
