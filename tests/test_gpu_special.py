"""Special cases of the method on every kernel path, against what they must
give exactly:

* x = 0: every partial is a zero, so the output is the residual, bit for bit;
* a one-hot x (a single 1.0): every partial is one weight or a zero, so the
  tensor-core and MXFP8 paths, whose summation order otherwise differs from
  the oracle's, must also match the oracle bit for bit;
* W = 0 on the tensor-core paths: the output is the residual;
* rotating which rank owns which K slice (N = 4, exact path): bit-identical
  to the oracle run on the rotated inputs, and within the rounding of the
  re-associated ring adds of the unrotated output.
Paths: the in-kernel fold (one token), the k-split ring kernel (three
tokens), the one-CTA kernel with the ring kernel (32 tokens), the CTA-pair
kernel (300 tokens), the MXFP8 kernel (one token).
"""

import numpy as np
import pytest
import torch

import oracle
from gpu_util import inputs, oracle_point
from helpers import u16

pytestmark = pytest.mark.gpu

TENSOR_SHAPES = [      # N, M, K, H, variant
    (2, 1, 2048, 512, "auto"),        # one token, 2 ranks x 8 parts: the counter fold
    (4, 3, 2048, 640, "auto"),        # three tokens: k-split parts and the split ring kernel
    (4, 32, 1024, 512, "auto"),       # 32 tokens, 16 units: k-split parts and the split ring kernel
    (8, 300, 1024, 4224, "auto"),     # 300 tokens: CTA pairs and the ring kernel
    (8, 64, 1024, 4096, "auto"),      # 64 tokens, 256 units: bf16 partials and the ring kernel
    (8, 64, 1024, 4096, "cluster"),   # the same folded on chip in clusters of 8
    (3, 40, 768, 6504, "cluster"),    # clusters of 3, ragged last H tile and token tile
    (2, 1, 5120, 5120, "cluster"),    # clusters of 2 ranks x 3 K parts (fp32 parts on chip)
]
TIDS = [f"{v}-N{n}M{m}K{k}H{h}" for n, m, k, h, v in TENSOR_SHAPES]


def _plan(n, m, k, h, variant="auto"):
    import tensor_layer_reconciliation_b200 as tlr
    return tlr.Plan(n, m, k, h, variant=variant)


def _run(plan, x, w, r):
    out = plan.reconcile(x, plan.pack_weights(w), r)
    torch.cuda.synchronize()
    assert plan.device_error_flags() == 0
    return u16(out)


def _one_hot(m, k, cols, dev):
    x = torch.zeros(m, k, dtype=torch.bfloat16, device=dev)
    for i in range(m):
        x[i, cols[i % len(cols)]] = 1.0
    return x


@pytest.mark.parametrize("shape", TENSOR_SHAPES, ids=TIDS)
def test_tensor_zero_x_gives_residual(shape):
    n, m, k, h, variant = shape
    dev = torch.device("cuda")
    _, w, r = inputs(n, m, k, h, 41 + n + m + k + h, dev)
    x = torch.zeros(m, k, dtype=torch.bfloat16, device=dev)
    assert np.array_equal(_run(_plan(n, m, k, h, variant), x, w, r), u16(r))


@pytest.mark.parametrize("shape", TENSOR_SHAPES, ids=TIDS)
def test_tensor_zero_w_gives_residual(shape):
    n, m, k, h, variant = shape
    dev = torch.device("cuda")
    x, _, r = inputs(n, m, k, h, 43 + n + m + k + h, dev)
    w = torch.zeros(h, k, dtype=torch.bfloat16, device=dev)
    assert np.array_equal(_run(_plan(n, m, k, h, variant), x, w, r), u16(r))


@pytest.mark.parametrize("shape", TENSOR_SHAPES, ids=TIDS)
def test_tensor_one_hot_x_bit_exact(shape):
    n, m, k, h, variant = shape
    dev = torch.device("cuda")
    _, w, r = inputs(n, m, k, h, 47 + n + m + k + h, dev)
    x = _one_hot(m, k, [3, k - 1, k // 2 + 5], dev)      # columns in the first, last, middle rank
    got = _run(_plan(n, m, k, h, variant), x, w, r)
    ref = oracle_point(n, h, x.cpu(), w.cpu(), r.cpu())
    assert np.array_equal(got, ref["out"])


def test_mx_zero_x_and_one_hot():
    n, m, k, h = 2, 1, 2048, 512
    dev = torch.device("cuda")
    _, w, r = inputs(n, m, k, h, 53, dev)
    plan = _plan(n, m, k, h)
    q, sc = plan.pack_weights_mxfp8(w)
    x0 = torch.zeros(m, k, dtype=torch.bfloat16, device=dev)
    out0 = plan.reconcile_mxfp8(x0, q, sc, r)
    x1 = _one_hot(m, k, [k - 7], dev)
    out1 = plan.reconcile_mxfp8(x1, q, sc, r)
    torch.cuda.synchronize()
    assert np.array_equal(u16(out0), u16(r))
    q_ref, sc_ref = oracle.mx_quantize(n, u16(w))
    w_deq = oracle.mx_dequant_bf16(n, q_ref, sc_ref)
    ref = oracle.reconcile(n, h, u16(x1), w_deq, u16(r))
    assert np.array_equal(u16(out1), ref["out"])


def test_rotated_shards_exact_n4():
    n, m, k, h = 4, 2, 1024, 512
    dev = torch.device("cuda")
    x, w, r = inputs(n, m, k, h, 59, dev)
    ks = k // n
    t = 1                                          # rank i now holds slice i + t
    perm = torch.cat([torch.arange(((i + t) % n) * ks, ((i + t) % n + 1) * ks) for i in range(n)])
    xr = x[:, perm].contiguous()
    wr = w[:, perm].contiguous()
    plan = _plan(n, m, k, h, variant="exact")
    got_rot = _run(plan, xr, wr, r)
    got = _run(plan, x, w, r)
    ref_rot = oracle_point(n, h, xr.cpu(), wr.cpu(), r.cpu())
    assert np.array_equal(got_rot, ref_rot["out"])
    # the same partials summed from other starting ranks: the rounding of the
    # N-1 ring adds and the residual add apart
    a = oracle.f32(got_rot).astype(np.float64)
    b = oracle.f32(got).astype(np.float64)
    pabs = np.abs(oracle.f32(ref_rot["partials"]).astype(np.float64)).sum(axis=0)
    res = np.abs(oracle.f32(u16(r)).astype(np.float64))

    def ulp(v):
        v = np.maximum(v, 2.0 ** -126)
        return 2.0 ** (np.floor(np.log2(v)) - 7)

    bound = (n - 1) * ulp(pabs) + 2 * ulp(res + pabs)
    assert np.all(np.abs(a - b) <= bound)
