"""The ring all-reduce as a protocol between ranks that each hold their own
buffers (tp_ring_allreduce_ranks), on one GPU with all N ranks in one
cooperative launch.

* Every rank's output equals the oracle's message-by-message ring plus the
  residual, bit for bit, for N = 1 .. 8, with token counts and widths that
  leave ragged slices per CTA, and equals tp_ring_reduce's output.
* The same workspaces serve several calls in a row (the step flags only
  grow; each call takes its base from them).
* A rank that never runs: the others' bounded waits on its flags run out,
  the device error word shows bit 1, the kernel returns, and the context
  stays usable (a full call afterwards is correct).
"""

import numpy as np
import pytest
import torch

import oracle
from gpu_util import draw
from helpers import u16

pytestmark = pytest.mark.gpu


def _partials(n, m, h, seed, dev):
    return [draw((m, h), 1.0, seed, 10 + r, dev) for r in range(n)]


def _expected(n, h, parts, res):
    p = np.stack([u16(t) for t in parts])
    red, _ = oracle.ring(n, h, p)
    return oracle.residual(u16(res), red)


@pytest.mark.parametrize("n,m,h", [(1, 3, 64), (2, 1, 5120), (2, 5, 1024), (3, 7, 4104),
                                   (4, 32, 5120), (5, 2, 640), (8, 64, 4096), (8, 3, 1088),
                                   (7, 1, 7 * 8)])
def test_protocol_matches_oracle_ring(n, m, h):
    import tensor_layer_reconciliation_b200 as tlr
    dev = torch.device("cuda")
    plan = tlr.Plan(n, m, 8 * n, h)
    parts = _partials(n, m, h, 300 + n * 10 + m, dev)
    res = draw((m, h), 1.0, 300 + m, 1, dev)
    outs, _ = plan.ring_allreduce_ranks(parts, res)
    ring = plan.ring_reduce(torch.stack(parts), res)
    torch.cuda.synchronize()
    assert plan.device_error_flags() == 0
    want = _expected(n, h, parts, res)
    for r, o in enumerate(outs):
        assert np.array_equal(u16(o), want), f"rank {r}"
    assert np.array_equal(u16(ring), want)


def test_protocol_workspaces_serve_many_calls():
    import tensor_layer_reconciliation_b200 as tlr
    dev = torch.device("cuda")
    n, m, h = 4, 9, 2048
    plan = tlr.Plan(n, m, 8 * n, h)
    ws = outs = None
    for call in range(4):
        parts = _partials(n, m, h, 400 + call, dev)
        res = draw((m, h), 1.0, 400 + call, 1, dev)
        outs, ws = plan.ring_allreduce_ranks(parts, res, outs=outs, workspaces=ws)
        torch.cuda.synchronize()
        assert plan.device_error_flags() == 0
        want = _expected(n, h, parts, res)
        for r, o in enumerate(outs):
            assert np.array_equal(u16(o), want), (call, r)


def test_protocol_absent_rank_times_out_and_context_survives():
    import tensor_layer_reconciliation_b200 as tlr
    dev = torch.device("cuda")
    n, m, h = 4, 2, 1024
    plan = tlr.Plan(n, m, 8 * n, h)
    parts = _partials(n, m, h, 500, dev)
    res = draw((m, h), 1.0, 500, 1, dev)
    assert plan.device_error_flags(reset=True) == 0
    # ranks 0..2 only: rank 3's flags are never set, so waits on them run out
    outs, ws = plan.ring_allreduce_ranks(parts, res, launch_ranks=3, wait_limit_ns=20_000_000)
    torch.cuda.synchronize()
    flags = plan.device_error_flags(reset=True)
    assert flags & 2, flags
    # the context is usable: zero the flag blocks and run the whole group
    for w in ws:
        w.zero_()
    outs, ws = plan.ring_allreduce_ranks(parts, res, outs=outs, workspaces=ws)
    torch.cuda.synchronize()
    assert plan.device_error_flags() == 0
    want = _expected(n, h, parts, res)
    for o in outs:
        assert np.array_equal(u16(o), want)


def test_protocol_rejects_bad_arguments():
    import tensor_layer_reconciliation_b200 as tlr
    dev = torch.device("cuda")
    n, m, h = 2, 2, 256
    plan = tlr.Plan(n, m, 16, h)
    parts = _partials(n, m, h, 600, dev)
    res = draw((m, h), 1.0, 600, 1, dev)
    need = plan.ring_rank_workspace_bytes(m)
    ws = [torch.zeros(need, dtype=torch.uint8, device=dev) for _ in range(n)]
    outs = [torch.full((m, h), 7.0, dtype=torch.bfloat16, device=dev) for _ in range(n)]
    P = [t.data_ptr() for t in parts]
    O = [t.data_ptr() for t in outs]
    W = [t.data_ptr() for t in ws]
    s = torch.cuda.current_stream().cuda_stream
    h_ = plan.handle
    assert tlr.tp_ring_allreduce_ranks(h_, P, res.data_ptr(), O, W, 0, 3, m, 0, s) == tlr.TP_ERR_INVALID
    assert tlr.tp_ring_allreduce_ranks(h_, P, res.data_ptr(), O, W, 1, 2, m, 0, s) == tlr.TP_ERR_INVALID
    assert tlr.tp_ring_allreduce_ranks(h_, P, res.data_ptr(), O, W, 0, 2, m + 1, 0, s) == tlr.TP_ERR_INVALID
    assert tlr.tp_ring_allreduce_ranks(h_, [P[0] + 2, P[1]], res.data_ptr(), O, W, 0, 2, m, 0,
                                       s) == tlr.TP_ERR_ALIGN
    assert tlr.tp_ring_allreduce_ranks(h_, P, res.data_ptr(), [O[0], O[0]], W, 0, 2, m, 0,
                                       s) == tlr.TP_ERR_INVALID       # two ranks, one output
    assert tlr.tp_ring_allreduce_ranks(h_, P, res.data_ptr(), [P[1], O[1]], W, 0, 2, m, 0,
                                       s) == tlr.TP_ERR_INVALID       # output over an input
    assert tlr.tp_ring_allreduce_ranks(h_, P, res.data_ptr(), O, [W[0], None], 0, 2, m, 0,
                                       s) == tlr.TP_ERR_INVALID
    assert tlr.tp_ring_allreduce_ranks(h_, P, 0, O, W, 0, 2, m, 0, s) == tlr.TP_ERR_INVALID
    assert tlr.tp_ring_allreduce_ranks(h_, P, res.data_ptr(), O, W, 0, 2, 0, 0, s) == tlr.TP_OK
    assert tlr.tp_ring_allreduce_ranks(None, P, res.data_ptr(), O, W, 0, 2, m, 0, s) == tlr.TP_ERR_INVALID
    torch.cuda.synchronize()
    for o in outs:
        assert bool(torch.all(o == 7.0))                # nothing launched
