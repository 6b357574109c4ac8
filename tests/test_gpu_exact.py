"""Parity of the CUDA path against the oracle, element by element.

The exact variant (CUDA cores, k-ascending fp32 FMA chain per partial) must
match the oracle bit for bit in the partials and in the output, fused or
staged, on shapes that span several CTAs with ragged tails in H (CTA rows),
in K (the last 64-column TMA block) and in M (the token tile), and on the
edge cases: N = 1, odd N, N = 8, K/N below one block, M = 0, W = 0,
integer-valued inputs, and swapped shards at N = 2.
"""

import numpy as np
import pytest
import torch

import oracle
from gpu_util import gpu_point, inputs, oracle_point
from helpers import from_u16, u16

pytestmark = pytest.mark.gpu

SHAPES = [            # N, M, K, H
    (2, 1, 1024, 256),    # the tiny workload's shape
    (2, 1, 400, 1200),    # H % rows-per-CTA != 0; K/N = 200 = 3 blocks + 8 columns
    (1, 1, 64, 64),       # one rank: no ring
    (3, 2, 48, 48),       # odd N; K/N = 16, less than one block
    (8, 3, 512, 256),     # N = 8, token tile of 4 with one token past the end
    (4, 9, 2048, 512),    # two token tiles of 8, the second ragged
    (2, 33, 320, 160),    # many token tiles
    (4, 1, 17408, 5120),  # the full down-projection width at N = 4
]


@pytest.fixture(scope="module")
def dev():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch.device("cuda")


@pytest.mark.parametrize("staged", [False, True])
@pytest.mark.parametrize("shape", SHAPES, ids=[f"N{n}M{m}K{k}H{h}" for n, m, k, h in SHAPES])
def test_exact_bitwise(shape, staged, dev):
    import tensor_layer_reconciliation_b200 as tlr
    n, m, k, h = shape
    seed = 100 + sum(shape)
    x, w, r = inputs(n, m, k, h, seed, dev)
    plan = tlr.Plan(n, m, k, h)
    out, parts, _ = gpu_point(plan, x, w, r, staged=staged)
    ref = oracle_point(n, h, x.cpu(), w.cpu(), r.cpu())
    assert np.array_equal(parts, ref["partials"])
    assert np.array_equal(out, ref["out"])


def test_generator_same_bits_on_gpu(dev):
    x, w, r = inputs(2, 3, 256, 64, 5, dev)
    xc, wc, rc = inputs(2, 3, 256, 64, 5, "cpu")
    assert torch.equal(x.cpu(), xc) and torch.equal(w.cpu(), wc) and torch.equal(r.cpu(), rc)


def test_zero_tokens_launches_nothing(dev):
    import tensor_layer_reconciliation_b200 as tlr
    plan = tlr.Plan(2, 4, 256, 64)
    x = torch.empty(0, 256, dtype=torch.bfloat16, device=dev)
    r = torch.empty(0, 64, dtype=torch.bfloat16, device=dev)
    wp = torch.zeros(plan.packed_numel, dtype=torch.bfloat16, device=dev)
    out = plan.reconcile(x, wp, r)
    assert out.shape == (0, 64)


def test_weight_zero_gives_residual(dev):
    import tensor_layer_reconciliation_b200 as tlr
    n, m, k, h = 4, 5, 512, 256
    x, _, r = inputs(n, m, k, h, 9, dev)
    w = torch.zeros(h, k, dtype=torch.bfloat16, device=dev)
    out, _, _ = gpu_point(tlr.Plan(n, m, k, h), x, w, r)
    assert torch.equal(from_u16(out).float(), r.cpu().float())


def test_integer_inputs_exact(dev):
    import tensor_layer_reconciliation_b200 as tlr
    n, m, k, h = 4, 3, 256, 64
    g = torch.Generator().manual_seed(3)
    xi = torch.randint(-1, 2, (m, k), generator=g)
    wi = torch.randint(-1, 2, (h, k), generator=g)
    ri = torch.randint(-8, 9, (m, h), generator=g)
    out, _, _ = gpu_point(tlr.Plan(n, m, k, h), xi.to(dev, torch.bfloat16),
                          wi.to(dev, torch.bfloat16), ri.to(dev, torch.bfloat16))
    assert torch.equal(from_u16(out).long(), xi @ wi.T + ri)


def test_swapped_shards_n2_bit_identical(dev):
    import tensor_layer_reconciliation_b200 as tlr
    n, m, k, h = 2, 2, 512, 256
    x, w, r = inputs(n, m, k, h, 4, dev)
    ks = k // n
    xs = torch.cat([x[:, ks:], x[:, :ks]], 1).contiguous()
    ws = torch.cat([w[:, ks:], w[:, :ks]], 1).contiguous()
    plan = tlr.Plan(n, m, k, h)
    a, _, _ = gpu_point(plan, x, w, r)
    b, _, _ = gpu_point(plan, xs, ws, r)
    assert np.array_equal(a, b)


def test_guard_zones_untouched(dev):
    """Output and workspace sit between sentinel-filled guards that no kernel may write."""
    import tensor_layer_reconciliation_b200 as tlr
    n, m, k, h = 2, 3, 400, 1200
    x, w, r = inputs(n, m, k, h, 6, dev)
    plan = tlr.Plan(n, m, k, h, variant="exact", staged=True)
    wp = plan.pack_weights(w)
    g = 4096
    sentinel = torch.tensor(0x7BCD, dtype=torch.int16)
    obuf = torch.full((g + m * h + g,), 0x7BCD, dtype=torch.int16, device=dev)
    out = obuf[g:g + m * h].view(torch.bfloat16).view(m, h)
    need = plan.workspace_bytes(m) // 2
    wbuf = torch.full((g + need + g,), 0x7BCD, dtype=torch.int16, device=dev)
    ws = wbuf[g:g + need]
    plan.reconcile(x, wp, r, out=out, workspace=ws)
    torch.cuda.synchronize()
    for buf, n_in in ((obuf, m * h), (wbuf, need)):
        assert torch.all(buf[:g].cpu() == sentinel) and torch.all(buf[g + n_in:].cpu() == sentinel)
    ref = oracle_point(n, h, x.cpu(), w.cpu(), r.cpu())
    assert np.array_equal(u16(out), ref["out"])


def test_subnormal_product_added_with_one_rounding(dev):
    """The oracle's pin of the accumulate step (a product below the fp32
    normal range, added to the running sum with one rounding) on the exact
    kernel: the partial, and with a zero residual the output, is 0x0181
    (rounding the product first would give 0x0182)."""
    import tensor_layer_reconciliation_b200 as tlr
    from test_oracle_reconcile import FMA_PIN_W, FMA_PIN_X
    n, m, k, h = 1, 1, 8, 8
    xb = np.zeros((m, k), dtype=np.uint16)
    wb = np.zeros((h, k), dtype=np.uint16)
    xb[0, :4] = FMA_PIN_X
    wb[0, :4] = FMA_PIN_W
    x, w = from_u16(xb).to(dev), from_u16(wb).to(dev)
    r = torch.zeros(m, h, dtype=torch.bfloat16, device=dev)
    for staged in (False, True):
        out, parts, _ = gpu_point(tlr.Plan(n, m, k, h), x, w, r, staged=staged)
        assert int(parts[0, 0, 0]) == 0x0181 and int(out[0, 0]) == 0x0181
