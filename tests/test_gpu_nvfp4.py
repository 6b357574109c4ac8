"""NVFP4 weight shards on the GPU against the oracle.

* Quantisation (S0) is byte work: codes, block scales and the second-level
  exponent must equal the oracle's bit for bit, on Gaussian weights and on
  blocks that run through every finite bf16 magnitude under several block
  maxima (E2M1 midpoints and saturation, E4M3 subnormal block scales, zero
  blocks).
* The reconciliation (S1-S4) over the shards is compared with the oracle's
  reconciliation over the dequantised weights under the tensor-core rule: a
  partial within 2^-19 * sum|x*w| of a bf16 rounding boundary may round
  either way; every output none of whose partials is that close is
  bit-identical.
"""

import numpy as np
import pytest
import torch

import oracle
from gpu_util import inputs
from helpers import from_u16, nv_scales_as_stored, u16
from test_gpu_tensor import check_against_oracle

pytestmark = pytest.mark.gpu


def _quantize_on_gpu(n, w):
    import tensor_layer_reconciliation_b200 as tlr
    h, k = w.shape
    plan = tlr.Plan(n, 1, k, h)
    q, sc = plan.pack_weights_nvfp4(w)
    torch.cuda.synchronize()
    return q.cpu().numpy().reshape(n, h, k // n // 2), sc.cpu().numpy()


def _amax_bits(w_u16):
    return int((np.asarray(w_u16) & 0x7FFF).max())


@pytest.mark.parametrize("n,h,k,seed", [(1, 64, 256, 1), (2, 96, 1024, 2), (4, 128, 2048, 3),
                                        (8, 64, 4096, 4)])
def test_nv_quantize_gaussian_bit_exact(n, h, k, seed):
    dev = torch.device("cuda")
    _, w, _ = inputs(n, 1, k, h, seed, dev)
    q, sc = _quantize_on_gpu(n, w)
    q_ref, sc_ref, g = oracle.nvfp4_quantize(n, u16(w))
    assert np.array_equal(sc, nv_scales_as_stored(sc_ref, g, _amax_bits(u16(w))))
    assert np.array_equal(q, q_ref)


@pytest.mark.parametrize("amax_bits", [0x3F80, 0x3FFF, 0x3E40, 0x0780, 0x7F7F, 0x0001, 0x3B00])
def test_nv_quantize_every_magnitude(amax_bits):
    """Blocks of 15 bf16 values with |v| <= A plus A itself, for every finite
    |v| <= A and both signs, and one block of zeros per row."""
    amax = float(oracle.f32(np.array([amax_bits], dtype=np.uint16))[0])
    pats = np.arange(0, 0x7F80, dtype=np.uint32).astype(np.uint16)
    keep = pats[oracle.f32(pats) <= amax]
    both = np.concatenate([keep, keep | 0x8000]).astype(np.uint16)
    nb = (len(both) + 14) // 15
    blocks = np.zeros((nb, 16), dtype=np.uint16)
    flat = np.zeros(nb * 15, dtype=np.uint16)
    flat[:len(both)] = both
    blocks[:, 1:] = flat.reshape(nb, 15)
    blocks[:, 0] = amax_bits
    rows = 8
    per_row = (nb + rows - 1) // rows + 1                # + a zero block in every row
    per_row = (per_row + 3) // 4 * 4                      # whole 64-column blocks
    w = np.zeros((rows * per_row, 16), dtype=np.uint16)
    idx = np.arange(nb)
    w[(idx // (per_row - 1)) * per_row + idx % (per_row - 1)] = blocks
    w = np.ascontiguousarray(w.reshape(rows, per_row * 16))
    q, sc = _quantize_on_gpu(1, from_u16(w).cuda())
    q_ref, sc_ref, g = oracle.nvfp4_quantize(1, w)
    assert np.array_equal(sc, nv_scales_as_stored(sc_ref, g, _amax_bits(w)))
    assert np.array_equal(q, q_ref)


SHAPES = [             # N, M, K, H
    (2, 1, 1024, 512),      # one token: K split, folded in the kernel
    (4, 3, 2048, 640),      # three tokens: K split, fp32 parts, split ring kernel
    (2, 1, 17408, 5120),    # the down-projection of the decode example, full size
    (8, 64, 1024, 4096),    # 256 units: bf16 partials and the ring kernel
    (8, 300, 1024, 4224),   # 256-token tiles: bf16 partials and the ring kernel
]
CASES = [("auto", s) for s in SHAPES] + [("cluster", (8, 64, 1024, 4096)),
                                          ("cluster", (3, 40, 768, 6504)),
                                          ("cluster", (2, 1, 5120, 5120))]
IDS = [f"{v}-N{n}M{m}K{k}H{h}" for v, (n, m, k, h) in CASES]


@pytest.mark.parametrize("variant,shape", CASES, ids=IDS)
def test_nv_reconcile_against_oracle(variant, shape):
    import tensor_layer_reconciliation_b200 as tlr
    n, m, k, h = shape
    dev = torch.device("cuda")
    x, w, r = inputs(n, m, k, h, 950 + sum(shape), dev)
    plan = tlr.Plan(n, m, k, h, variant=variant)
    q, sc = plan.pack_weights_nvfp4(w)
    out = plan.reconcile_nvfp4(x, q, sc, r)
    torch.cuda.synchronize()
    assert plan.device_error_flags() == 0
    q_ref, sc_ref, g = oracle.nvfp4_quantize(n, u16(w))
    assert np.array_equal(q.cpu().numpy().reshape(q_ref.shape), q_ref)
    w_deq = oracle.nvfp4_dequant_bf16(n, q_ref, sc_ref, g)
    ref = oracle.reconcile(n, h, u16(x), w_deq, u16(r), threads=8)
    ref["res"] = u16(r)
    fp, fo, mx, rl2 = check_against_oracle(u16(out), ref["partials"], ref, n, outputs_only=True)
    print(f"{shape}: fragile partials {fp}, outputs touched {fo}, max abs {mx:.3g}, rel L2 {rl2:.3g}")


def test_nv_one_hot_and_limits():
    import tensor_layer_reconciliation_b200 as tlr
    dev = torch.device("cuda")
    n, m, k, h = 2, 1, 2048, 512
    _, w, r = inputs(n, m, k, h, 57, dev)
    plan = tlr.Plan(n, m, k, h)
    q, sc = plan.pack_weights_nvfp4(w)
    x1 = torch.zeros(m, k, dtype=torch.bfloat16, device=dev)
    x1[0, k - 5] = 1.0                                   # selects one dequantised weight per row
    out = plan.reconcile_nvfp4(x1, q, sc, r)
    torch.cuda.synchronize()
    q_ref, sc_ref, g = oracle.nvfp4_quantize(n, u16(w))
    w_deq = oracle.nvfp4_dequant_bf16(n, q_ref, sc_ref, g)
    ref = oracle.reconcile(n, h, u16(x1), w_deq, u16(r))
    assert np.array_equal(u16(out), ref["out"])
    bad = tlr.Plan(1, 1, 96, 256)                        # K/N = 96: not whole 64-column blocks
    assert tlr.tp_plan_nvfp4_bytes(bad.handle)[0] == tlr.TP_ERR_UNSUPPORTED
