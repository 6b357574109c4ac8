"""Host-side argument checks of every compute entry point, and guard zones
around the buffers of every kernel path.

Fault injection on the host: misaligned pointers (TP_ERR_ALIGN), an output
that overlaps an input or the workspace (TP_ERR_INVALID), a missing workspace
(TP_ERR_WORKSPACE), token counts outside [0, max_tokens] (TP_ERR_INVALID)
and shard widths the MXFP8 path has no form for (TP_ERR_UNSUPPORTED). Each
call must return its status with nothing launched: the output, filled with a
sentinel beforehand, is unchanged after the stream has drained, and the
device error word stays clear. The C ABI carries no workspace size, so a
workspace that is present but short cannot be seen there; the torch binding
checks the size and raises (tested below).

Guard zones: the output and the workspace of the tensor-core path (one and
three tokens with a k-split, 32 tokens without), of the CTA-pair path and
of the MXFP8 kernel sit between sentinel-filled guards that no kernel may
write; the guarded call must also give the same bits as an unguarded one.
"""

import pytest
import torch

from gpu_util import inputs

pytestmark = pytest.mark.gpu

SENT = 0x7BCD
N, M, K, H = 4, 4, 1024, 128         # tensor cores, K split 4 ways, a ring kernel: a workspace


@pytest.fixture(scope="module")
def setup():
    import tensor_layer_reconciliation_b200 as tlr
    dev = torch.device("cuda")
    plan = tlr.Plan(N, M, K, H)       # AUTO: tensor cores, staged partials
    x, w, r = inputs(N, M, K, H, 77, dev)
    wp = plan.pack_weights(w)
    need = plan.workspace_bytes(M)
    assert need > 0
    ws = torch.zeros(need + 64, dtype=torch.uint8, device=dev)
    torch.cuda.synchronize()
    return tlr, plan, x, wp, r, ws, dev


def _sentinel(numel, dev):
    return torch.full((numel,), SENT, dtype=torch.int16, device=dev)


def _untouched(buf, plan):
    torch.cuda.synchronize()
    assert bool(torch.all(buf == SENT)), "a refused call wrote its output"
    assert plan.device_error_flags() == 0


def _stream():
    return torch.cuda.current_stream().cuda_stream


def test_reconcile_rejects_misaligned(setup):
    tlr, plan, x, wp, r, ws, dev = setup
    out = _sentinel(M * H + 8, dev)
    o = out.data_ptr()
    args = dict(x=x.data_ptr(), w=wp.data_ptr(), r=r.data_ptr(), o=o, ws=ws.data_ptr())
    for key in args:
        bad = dict(args)
        bad[key] += 2                                   # bf16-aligned, not 16-byte aligned
        st = tlr.tp_rowlinear_reconcile(plan.handle, bad["x"], bad["w"], bad["r"], bad["o"], M,
                                        bad["ws"], _stream())
        assert st == tlr.TP_ERR_ALIGN, key
        st = tlr.tp_rowlinear_reconcile_noalloc(plan.handle, bad["x"], bad["w"], bad["r"],
                                                bad["o"], M, _stream())
        assert st == (tlr.TP_OK if key == "ws" else tlr.TP_ERR_ALIGN), key
        if key == "ws":                                  # that call ran: refill the sentinel
            torch.cuda.synchronize()
            out.fill_(SENT)
    _untouched(out, plan)


def test_reconcile_rejects_overlap(setup):
    tlr, plan, x, wp, r, ws, dev = setup
    out = _sentinel(M * H, dev)
    big = _sentinel(M * K + M * H + 64, dev)             # x with room for an out inside it
    big_x = big[:M * K]
    overlaps = {
        "out in x": (big.data_ptr(), big.data_ptr() + 16, r.data_ptr(), ws.data_ptr()),
        "out in residual": (x.data_ptr(), r.data_ptr(), r.data_ptr(), ws.data_ptr()),
        "out in weights": (x.data_ptr(), wp.data_ptr() + 1024, r.data_ptr(), ws.data_ptr()),
        "out in workspace": (x.data_ptr(), ws.data_ptr(), r.data_ptr(), ws.data_ptr()),
    }
    big_x.copy_(x.view(torch.int16).view(-1))
    for name, (px, po, pr, pws) in overlaps.items():
        st = tlr.tp_rowlinear_reconcile(plan.handle, px, wp.data_ptr(), pr, po, M, pws, _stream())
        assert st == tlr.TP_ERR_INVALID, name
    # the no-alloc form: the output may not overlap its inputs either
    st = tlr.tp_rowlinear_reconcile_noalloc(plan.handle, big.data_ptr(), wp.data_ptr(), r.data_ptr(),
                                            big.data_ptr() + 16, M, _stream())
    assert st == tlr.TP_ERR_INVALID
    _untouched(out, plan)
    torch.cuda.synchronize()
    assert bool(torch.all(big[M * K:] == SENT))
    assert torch.equal(big_x, x.view(torch.int16).view(-1))


def test_reconcile_rejects_missing_workspace_and_token_counts(setup):
    tlr, plan, x, wp, r, ws, dev = setup
    out = _sentinel(M * H, dev)
    args = (x.data_ptr(), wp.data_ptr(), r.data_ptr(), out.data_ptr())
    assert tlr.tp_rowlinear_reconcile(plan.handle, *args, M, 0, _stream()) == tlr.TP_ERR_WORKSPACE
    for tokens in (M + 1, -1):
        assert tlr.tp_rowlinear_reconcile(plan.handle, *args, tokens, ws.data_ptr(),
                                          _stream()) == tlr.TP_ERR_INVALID
        assert tlr.tp_rowlinear_reconcile_noalloc(plan.handle, *args, tokens,
                                                  _stream()) == tlr.TP_ERR_INVALID
        assert tlr.tp_rowlinear_partials(plan.handle, args[0], args[1], out.data_ptr(), tokens,
                                         _stream()) == tlr.TP_ERR_INVALID
        assert tlr.tp_ring_reduce(plan.handle, ws.data_ptr(), args[2], out.data_ptr(), tokens,
                                  _stream()) == tlr.TP_ERR_INVALID
    # null tensors with tokens > 0
    assert tlr.tp_rowlinear_reconcile(plan.handle, 0, args[1], args[2], args[3], M, ws.data_ptr(),
                                      _stream()) == tlr.TP_ERR_INVALID
    assert tlr.tp_rowlinear_reconcile(plan.handle, args[0], args[1], 0, args[3], M, ws.data_ptr(),
                                      _stream()) == tlr.TP_ERR_INVALID
    # tokens = 0 launches nothing and needs no pointer at all
    assert tlr.tp_rowlinear_reconcile(plan.handle, 0, 0, 0, 0, 0, 0, _stream()) == tlr.TP_OK
    _untouched(out, plan)


def test_binding_rejects_short_workspace(setup):
    tlr, plan, x, wp, r, ws, dev = setup
    short = torch.zeros(plan.workspace_bytes(M) - 256, dtype=torch.uint8, device=dev)
    out = _sentinel(M * H, dev)
    with pytest.raises(ValueError):
        plan.reconcile(x, wp, r, out=out.view(torch.bfloat16).view(M, H), workspace=short)
    _untouched(out, plan)


def test_partials_rejects_misaligned_and_overlap(setup):
    tlr, plan, x, wp, r, ws, dev = setup
    parts = _sentinel(N * M * H + 8, dev)
    p = parts.data_ptr()
    s = _stream()
    assert tlr.tp_rowlinear_partials(plan.handle, x.data_ptr() + 2, wp.data_ptr(), p, M, s) == tlr.TP_ERR_ALIGN
    assert tlr.tp_rowlinear_partials(plan.handle, x.data_ptr(), wp.data_ptr() + 2, p, M, s) == tlr.TP_ERR_ALIGN
    assert tlr.tp_rowlinear_partials(plan.handle, x.data_ptr(), wp.data_ptr(), p + 2, M, s) == tlr.TP_ERR_ALIGN
    assert tlr.tp_rowlinear_partials(plan.handle, x.data_ptr(), wp.data_ptr(), x.data_ptr(), M,
                                     s) == tlr.TP_ERR_INVALID
    assert tlr.tp_rowlinear_partials(plan.handle, x.data_ptr(), wp.data_ptr(), wp.data_ptr() + 4096,
                                     M, s) == tlr.TP_ERR_INVALID
    assert tlr.tp_rowlinear_partials(plan.handle, x.data_ptr(), wp.data_ptr(), 0, M, s) == tlr.TP_ERR_INVALID
    _untouched(parts, plan)


def test_ring_reduce_rejects_misaligned_and_overlap(setup):
    tlr, plan, x, wp, r, ws, dev = setup
    parts = torch.zeros(N * M * H, dtype=torch.int16, device=dev)
    out = _sentinel(M * H + 8, dev)
    s = _stream()
    pp, pr, po = parts.data_ptr(), r.data_ptr(), out.data_ptr()
    for a, b, c in ((pp + 2, pr, po), (pp, pr + 2, po), (pp, pr, po + 2)):
        assert tlr.tp_ring_reduce(plan.handle, a, b, c, M, s) == tlr.TP_ERR_ALIGN
    assert tlr.tp_ring_reduce(plan.handle, pp, pr, pp + 256, M, s) == tlr.TP_ERR_INVALID
    assert tlr.tp_ring_reduce(plan.handle, pp, pr, pr, M, s) == tlr.TP_ERR_INVALID
    assert tlr.tp_ring_reduce(plan.handle, 0, pr, po, M, s) == tlr.TP_ERR_INVALID
    _untouched(out, plan)


def test_mxfp8_rejects_bad_arguments(setup):
    tlr, plan, x, wp, r, ws, dev = setup
    w = torch.randn(H, K, device=dev).to(torch.bfloat16)
    q, sc = plan.pack_weights_mxfp8(w)
    need = plan.mxfp8_workspace_bytes(M)
    assert need > 0
    mws = torch.zeros(need, dtype=torch.uint8, device=dev)
    out = _sentinel(M * H + 8, dev)
    s = _stream()
    base = [x.data_ptr(), q.data_ptr(), sc.data_ptr(), r.data_ptr(), out.data_ptr()]
    for i in range(5):
        bad = list(base)
        bad[i] += 2
        assert tlr.tp_rowlinear_reconcile_mxfp8(plan.handle, *bad, M, mws.data_ptr(), s) == tlr.TP_ERR_ALIGN, i
    assert tlr.tp_rowlinear_reconcile_mxfp8(plan.handle, *base, M, mws.data_ptr() + 2, s) == tlr.TP_ERR_ALIGN
    for i in (0, 1, 2, 3):                               # out overlapping x, codes, scales, residual
        bad = list(base)
        bad[4] = base[i]
        assert tlr.tp_rowlinear_reconcile_mxfp8(plan.handle, *bad, M, mws.data_ptr(), s) == tlr.TP_ERR_INVALID, i
    bad = list(base)
    bad[4] = mws.data_ptr()
    assert tlr.tp_rowlinear_reconcile_mxfp8(plan.handle, *bad, M, mws.data_ptr(), s) == tlr.TP_ERR_INVALID
    assert tlr.tp_rowlinear_reconcile_mxfp8(plan.handle, *base, M, 0, s) == tlr.TP_ERR_WORKSPACE
    assert tlr.tp_rowlinear_reconcile_mxfp8(plan.handle, *base, M + 1, mws.data_ptr(), s) == tlr.TP_ERR_INVALID
    assert tlr.tp_rowlinear_reconcile_mxfp8(plan.handle, *base, -1, mws.data_ptr(), s) == tlr.TP_ERR_INVALID
    # packing: misaligned or overlapping shard buffers
    assert tlr.tp_pack_weights_mxfp8(plan.handle, w.data_ptr(), q.data_ptr() + 2, sc.data_ptr(), s) == tlr.TP_ERR_ALIGN
    assert tlr.tp_pack_weights_mxfp8(plan.handle, w.data_ptr(), q.data_ptr(), sc.data_ptr() + 2, s) == tlr.TP_ERR_ALIGN
    assert tlr.tp_pack_weights_mxfp8(plan.handle, w.data_ptr(), q.data_ptr(), q.data_ptr(), s) == tlr.TP_ERR_INVALID
    _untouched(out, plan)


# ------------------------------------------------------------ guard zones --

GUARD = 4096     # int16 elements on each side (8 KB)


def _guarded(numel, dev):
    buf = torch.full((GUARD + numel + GUARD,), SENT, dtype=torch.int16, device=dev)
    return buf, buf[GUARD:GUARD + numel]


def _guards_intact(buf, numel):
    torch.cuda.synchronize()
    return bool(torch.all(buf[:GUARD] == SENT)) and bool(torch.all(buf[GUARD + numel:] == SENT))


@pytest.mark.parametrize("n,m,k,h,variant", [
    (2, 1, 8192, 512, "auto"),      # one token: K split across CTAs, folded in the kernel
    (4, 3, 2048, 640, "auto"),      # three tokens: K split, fp32 parts, ring kernel for parts
    (8, 32, 1024, 4096, "auto"),    # 32 tokens, 256 units (>= one per SM): no split, bf16 partials
    (8, 300, 1024, 4224, "auto"),   # CTA pairs (2-SM MMA), ragged token tile and H-tile pair
    (8, 32, 1024, 4096, "cluster"), # folded on chip in clusters of 8
    (2, 1, 5120, 5120, "cluster"),  # clusters of 2 ranks x 3 K parts
])
def test_guard_zones_tensor_paths(n, m, k, h, variant):
    import tensor_layer_reconciliation_b200 as tlr
    dev = torch.device("cuda")
    x, w, r = inputs(n, m, k, h, 600 + m, dev)
    plan = tlr.Plan(n, m, k, h, variant=variant)
    wp = plan.pack_weights(w)
    ref = plan.reconcile(x, wp, r)
    obuf, o = _guarded(m * h, dev)
    need = (plan.workspace_bytes(m) + 1) // 2
    wbuf, ws = _guarded(need, dev)
    ws.zero_()                       # fold counters at zero, the partials region anything
    plan.reconcile(x, wp, r, out=o.view(torch.bfloat16).view(m, h), workspace=ws)
    assert _guards_intact(obuf, m * h) and _guards_intact(wbuf, need)
    assert torch.equal(o, ref.view(torch.int16).view(-1))
    assert plan.device_error_flags() == 0


@pytest.mark.parametrize("n,m,k,h", [(2, 1, 2048, 512), (4, 4, 1024, 256), (8, 64, 1024, 4096)])
def test_guard_zones_mxfp8(n, m, k, h):
    import tensor_layer_reconciliation_b200 as tlr
    dev = torch.device("cuda")
    x, w, r = inputs(n, m, k, h, 700 + m, dev)
    plan = tlr.Plan(n, m, k, h)
    q, sc = plan.pack_weights_mxfp8(w)
    ref = plan.reconcile_mxfp8(x, q, sc, r)
    obuf, o = _guarded(m * h, dev)
    need = (plan.mxfp8_workspace_bytes(m) + 1) // 2
    wbuf, ws = _guarded(need, dev)
    ws.zero_()
    plan.reconcile_mxfp8(x, q, sc, r, out=o.view(torch.bfloat16).view(m, h),
                         workspace=ws if need else None)
    assert _guards_intact(obuf, m * h) and _guards_intact(wbuf, need)
    assert torch.equal(o, ref.view(torch.int16).view(-1))
    # the shards themselves, packed into guarded buffers
    qb, sb = plan.mxfp8_bytes()
    qbuf = torch.full((GUARD * 2 + qb + GUARD * 2,), 0x5A, dtype=torch.uint8, device=dev)
    sbuf = torch.full((GUARD * 2 + sb + GUARD * 2,), 0x5A, dtype=torch.uint8, device=dev)
    st = tlr.tp_pack_weights_mxfp8(plan.handle, w.data_ptr(), qbuf.data_ptr() + GUARD * 2,
                                   sbuf.data_ptr() + GUARD * 2, _stream())
    assert st == tlr.TP_OK
    torch.cuda.synchronize()
    for buf, nb, ref_t in ((qbuf, qb, q), (sbuf, sb, sc)):
        assert bool(torch.all(buf[:GUARD * 2] == 0x5A)) and bool(torch.all(buf[GUARD * 2 + nb:] == 0x5A))
        assert torch.equal(buf[GUARD * 2:GUARD * 2 + nb], ref_t)
    assert plan.device_error_flags() == 0
