"""MXFP8 weight shards on the GPU against the oracle.

* Quantisation (S0) is byte work: the codes and scales must equal the
  oracle's bit for bit, on Gaussian weights and on blocks that run through
  every finite bf16 magnitude under several block maxima (subnormal E4M3
  codes, midpoints, saturation at 448, tiny and huge scales).
* The reconciliation (S1-S4) over the shards is compared with the oracle's
  reconciliation over the dequantised weights under the same rule as the
  tensor-core path: the kernel sums in its own order, so a partial lying
  within 2^-19 * sum|x*w| of a bf16 rounding boundary may round either way;
  every output none of whose partials is that close is bit-identical. For
  at most 8 tokens the block-scaled form splits each activation into two
  E4M3 terms, exact except for values far below their run's maximum; the
  margin then grows by the bound on that split (helpers.x_split_error_bound).
"""

import numpy as np
import pytest
import torch

import oracle
from gpu_util import inputs
from helpers import from_u16, mx_scales_as_stored, u16, x_split_error_bound
from test_gpu_tensor import check_against_oracle

pytestmark = pytest.mark.gpu


def _plan(n, m, k, h):
    import tensor_layer_reconciliation_b200 as tlr
    return tlr.Plan(n, m, k, h)


def _quantize_on_gpu(n, w):
    h, k = w.shape
    plan = _plan(n, 1, k, h)
    q, sc = plan.pack_weights_mxfp8(w)
    torch.cuda.synchronize()
    ks = k // n
    return q.cpu().numpy().reshape(n, h, ks), sc.cpu().numpy()


@pytest.mark.parametrize("n,h,k,seed", [(1, 64, 256, 1), (2, 96, 1024, 2), (4, 128, 2048, 3),
                                        (8, 64, 4096, 4)])
def test_mx_quantize_gaussian_bit_exact(n, h, k, seed):
    dev = torch.device("cuda")
    _, w, _ = inputs(n, 1, k, h, seed, dev)
    q, sc = _quantize_on_gpu(n, w)
    q_ref, sc_ref = oracle.mx_quantize(n, u16(w))
    assert np.array_equal(sc, mx_scales_as_stored(sc_ref))
    assert np.array_equal(q, q_ref)


@pytest.mark.parametrize("amax_bits", [0x3F80, 0x3FFF, 0x3E40, 0x0780, 0x7F7F, 0x0001, 0x3B00])
def test_mx_quantize_every_magnitude(amax_bits):
    """Blocks of 31 bf16 values with |v| <= A plus A itself, for every finite
    |v| <= A and both signs: all element conversions the block maximum A allows."""
    amax = float(oracle.f32(np.array([amax_bits], dtype=np.uint16))[0])
    pats = np.arange(0, 0x7F80, dtype=np.uint32).astype(np.uint16)          # finite magnitudes
    vals = oracle.f32(pats)
    keep = pats[vals <= amax]
    both = np.concatenate([keep, keep | 0x8000]).astype(np.uint16)
    nb = (len(both) + 30) // 31
    blocks = np.zeros((nb, 32), dtype=np.uint16)
    flat = np.zeros(nb * 31, dtype=np.uint16)
    flat[:len(both)] = both
    blocks[:, 1:] = flat.reshape(nb, 31)
    blocks[:, 0] = amax_bits
    rows = 8
    per_row = (nb + rows - 1) // rows
    per_row = (per_row + 7) // 8 * 8                                         # K/N % 8 for the plan
    w = np.zeros((rows * per_row, 32), dtype=np.uint16)
    w[:nb] = blocks
    w = np.ascontiguousarray(w.reshape(rows, per_row * 32))
    q, sc = _quantize_on_gpu(1, from_u16(w).cuda())
    q_ref, sc_ref = oracle.mx_quantize(1, w)
    assert np.array_equal(sc, mx_scales_as_stored(sc_ref))
    assert np.array_equal(q, q_ref)


SHAPES = [             # N, M, K, H
    (2, 1, 1024, 512),      # one token: K split, folded in the kernel
    (4, 2, 2048, 640),      # two tokens, H % 128 != 0
    (8, 3, 4096, 1024),     # three tokens: K split, fp32 parts, split ring kernel
    (1, 4, 512, 256),       # N = 1
    (2, 1, 17408, 5120),    # the down-projection of the decode example, full size
    (2, 1, 1152, 384),      # K/N = 576: the last 128-column stage lies half past K/N (block-scaled)
    (2, 5, 1152, 256),      # five tokens, the same half stage, K split and the split ring kernel
    (8, 64, 1024, 4096),    # 64 tokens, 256 units: bf16 partials and the ring kernel
    (2, 300, 1024, 512),    # 256-token tiles with a K split: parts and the split ring kernel
    (8, 300, 1024, 4224),   # 256-token tiles, no split: bf16 partials and the ring kernel
]
CLUSTER = [                 # the CLUSTER variant: ranks (x K parts) folded on chip
    (8, 64, 1024, 4096),    # clusters of 8
    (3, 40, 768, 6504),     # clusters of 3, ragged H tile and tokens
    (2, 1, 5120, 5120),     # 2 ranks x 3 K parts
]
CASES = [("auto", s) for s in SHAPES] + [("cluster", s) for s in CLUSTER]
IDS = [f"{v}-N{n}M{m}K{k}H{h}" for v, (n, m, k, h) in CASES]


@pytest.mark.parametrize("variant,shape", CASES, ids=IDS)
def test_mx_reconcile_against_oracle(variant, shape):
    import tensor_layer_reconciliation_b200 as tlr
    n, m, k, h = shape
    dev = torch.device("cuda")
    x, w, r = inputs(n, m, k, h, 900 + sum(shape), dev)
    plan = tlr.Plan(n, m, k, h, variant=variant)
    q, sc = plan.pack_weights_mxfp8(w)
    out = plan.reconcile_mxfp8(x, q, sc, r)
    torch.cuda.synchronize()
    assert plan.device_error_flags() == 0
    ks = k // n
    q_ref, sc_ref = oracle.mx_quantize(n, u16(w))
    assert np.array_equal(q.cpu().numpy().reshape(n, h, ks), q_ref)
    w_deq = oracle.mx_dequant_bf16(n, q_ref, sc_ref)
    ref = oracle.reconcile(n, h, u16(x), w_deq, u16(r), threads=8)
    ref["res"] = u16(r)
    if m <= 8:   # the block-scaled form splits the activations: widen the margin by that bound
        ref["pabs"] = ref["pabs"] + x_split_error_bound(n, u16(x), w_deq) * 2.0 ** 19
    got = u16(out)
    # the kernel does not expose its partials: check outputs with the rule's bound
    fp, fo, mx, rl2 = check_against_oracle(got, ref["partials"], ref, n, outputs_only=True)
    print(f"{shape}: fragile partials {fp}, outputs touched {fo}, max abs {mx:.3g}, rel L2 {rl2:.3g}")


def test_mx_limits():
    import tensor_layer_reconciliation_b200 as tlr
    plan48 = _plan(2, 1, 96, 256)                        # K/N = 48: not whole 32-weight blocks
    assert tlr.tp_plan_mxfp8_bytes(plan48.handle)[0] == tlr.TP_ERR_UNSUPPORTED
    plan96 = _plan(1, 1, 96, 256)                        # K/N = 96: 32-weight runs, not 64-column blocks
    assert tlr.tp_plan_mxfp8_bytes(plan96.handle)[0] == tlr.TP_ERR_UNSUPPORTED
    assert tlr.tp_rowlinear_reconcile_mxfp8(plan96.handle, 256, 512, 768, 1024, 1280, 1, 0,
                                            0) == tlr.TP_ERR_UNSUPPORTED
    plan = tlr.Plan(8, 64, 1024, 4096, variant="cluster")
    assert plan.mxfp8_workspace_bytes(64) == 0           # folds in clusters: nothing staged
    assert _plan(8, 64, 1024, 4096).mxfp8_workspace_bytes(64) > 0   # AUTO: staged partials
    assert _plan(2, 1, 1024, 512).mxfp8_workspace_bytes(1) > 0      # k-split parts and counters
