"""S2-S4 on the GPU given identical partials: bit-exact against the oracle's
message-by-message ring, for N = 1..8 and several shapes, and the bf16 add of
the ring kernel against the oracle's on all 2^32 pairs of bf16 patterns."""

import numpy as np
import pytest
import torch

import oracle
from helpers import from_u16, u16

pytestmark = pytest.mark.gpu


def _ring_gpu(plan, p_u16, r_u16):
    dev = torch.device("cuda")
    p = from_u16(p_u16).to(dev)
    r = from_u16(r_u16).to(dev)
    out = plan.ring_reduce(p, r)
    torch.cuda.synchronize()
    return u16(out)


@pytest.mark.parametrize("n", range(1, 9))
@pytest.mark.parametrize("m,hc", [(1, 8), (3, 64), (32, 640), (2, 1280)])
def test_ring_bitexact(n, m, hc):
    import tensor_layer_reconciliation_b200 as tlr
    h = n * hc
    rng = np.random.default_rng(n * 1000 + m * 7 + hc)
    p = oracle.bf16_rne((rng.standard_normal((n, m, h)) * 2).astype(np.float32))
    r = oracle.bf16_rne(rng.standard_normal((m, h)).astype(np.float32))
    plan = tlr.Plan(n, m, 8 * n, h)
    red, _ = oracle.ring(n, h, p)
    want = oracle.residual(r, red)
    assert np.array_equal(_ring_gpu(plan, p, r), want)


def test_ring_fold_order_golden_on_gpu():
    import tensor_layer_reconciliation_b200 as tlr
    from helpers import golden_rows
    (row,) = golden_rows("ring_order_n3.txt")
    vals = [float(v) for v in row]
    n, hc = 3, 8
    h = n * hc
    p = np.stack([np.full((1, h), oracle.bf16_rne(np.float32(v)), np.uint16) for v in vals[:3]])
    r = np.zeros((1, h), np.uint16)
    got = oracle.f32(_ring_gpu(tlr.Plan(n, 1, 8 * n, h), p, r))[0]
    for c in range(n):
        assert np.all(got[c * hc:(c + 1) * hc] == vals[3 + c])


def test_bf16_add_exhaustive():
    """Every (a, b) pair of bf16 patterns: the ring kernel at N = 2 with a
    residual of -0 (which leaves a sum unchanged) computes bf16(a + b); the
    oracle's add is compared on all 2^32 pairs, NaN compared as NaN."""
    import tensor_layer_reconciliation_b200 as tlr
    dev = torch.device("cuda")
    na = 1024                                   # a-values per slice
    h = na * 65536                              # one column per (a, b) pair
    plan = tlr.Plan(2, 1, 16, h)
    b_all = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    fb = oracle.f32(b_all)
    res = torch.full((1, h), -0.0, dtype=torch.bfloat16, device=dev)
    out = torch.empty(1, h, dtype=torch.bfloat16, device=dev)
    parts = torch.empty(2, 1, h, dtype=torch.bfloat16, device=dev)
    for a0 in range(0, 65536, na):
        a = np.arange(a0, a0 + na, dtype=np.uint32).astype(np.uint16)
        pa = np.repeat(a, 65536)
        pb = np.tile(b_all, na)
        parts[0, 0].copy_(from_u16(pa))
        parts[1, 0].copy_(from_u16(pb))
        plan.ring_reduce(parts, res, out=out)
        got = u16(out)[0]
        s32 = (oracle.f32(a)[:, None] + fb[None, :]).astype(np.float32).reshape(-1)
        want = oracle.bf16_rne(s32)
        nan_w = (want & 0x7F80) == 0x7F80
        nan_w &= (want & 0x7F) != 0
        nan_g = ((got & 0x7F80) == 0x7F80) & ((got & 0x7F) != 0)
        assert np.array_equal(nan_g, nan_w), a0
        assert np.array_equal(got[~nan_w], want[~nan_w]), a0
