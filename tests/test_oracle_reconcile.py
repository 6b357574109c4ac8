"""Pins of the oracle's partials and of the whole reconciliation point.

* integer-valued x, W in {-1, 0, 1} and small integer residuals: every
  rounding is exact, so the output must equal the int64 product x.W + res;
* a crafted order-sensitive dot product: fp32 accumulation with k ascending
  gives 0 where the exact sum is 1 (the accumulator reading);
* a crafted dot product with a subnormal product: each product is added to
  the running fp32 sum with one rounding (fused multiply-add), which gives a
  different bf16 partial than rounding the product first and then adding;
* each partial lies within the textbook error bound of recursive fp32
  summation (Higham, "Accuracy and Stability of Numerical Algorithms", 4.2:
  |error| <= gamma_(n-1) * sum |x_k w_k|) of the exact rational dot product,
  before its one bf16 rounding;
* Gaussian tiny inputs: the whole output lies within the propagated rounding
  bound of the fp64 result x.W + res;
* special cases: W = 0 gives the residual; N = 1 has no ring; a one-hot x
  selects weight entries; the result does not depend on the thread count.
"""

from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from helpers import bf16_value, round_bf16_exact, round_f32_exact, u16
from workloads import KIND_RESIDUAL, KIND_W, KIND_X, get_config, point_tensor

U = 2.0 ** -8          # bf16 unit roundoff
U32 = 2.0 ** -24       # fp32 unit roundoff


def gamma(n, u=U32):
    return n * u / (1 - n * u)


def _bits(a):
    return oracle.bf16_rne(np.asarray(a, dtype=np.float32))


@pytest.mark.parametrize("n,m,k,h", [(1, 1, 16, 8), (2, 3, 64, 16), (4, 2, 256, 32),
                                     (8, 5, 512, 64), (3, 1, 96, 24)])
def test_integer_exact(n, m, k, h):
    rng = np.random.default_rng(n * 100 + k)
    x = rng.integers(-1, 2, size=(m, k))
    w = rng.integers(-1, 2, size=(h, k))
    res = rng.integers(-8, 9, size=(m, h))
    got = oracle.reconcile(n, h, _bits(x), _bits(w), _bits(res))
    want = x @ w.T + res                                 # int64, exact
    assert np.all(np.abs(want) <= 256)                   # every value fits bf16 exactly
    assert np.array_equal(oracle.f32(got["out"]).astype(np.int64), want)


def test_partial_order_fp32_ascending():
    # products 2^24, 1, -2^24, 0: fp32 k-ascending gives 2^24 (the tie of
    # 2^24 + 1 goes to even), then 0; the exact sum (or the reverse order) is 1
    x = _bits([[4096.0, 1.0, -4096.0, 0.0]])
    w = _bits([[4096.0, 1.0, 4096.0, 0.0]])
    p, p64, _ = oracle.partials(1, x, w)
    assert oracle.f32(p)[0, 0, 0] == 0.0
    assert p64[0, 0, 0] == 1.0


# Four products, k ascending (hand-derived): p0 = (1 + 2^-7) 2^-124 = b, a bf16
# value with an odd last bit; p1 = 2^-132, half a bf16 unit of b, so the sum
# is the bf16 midpoint m = b + 2^-132; p2 = -2^-147, one fp32 unit in this
# binade, so the sum is m - 2^-147; p3 = 1.75 * 2^-149, a product below the
# fp32 normal range. Fused: m - 2^-147 + 0.4375 units rounds back to
# m - 2^-147, below the midpoint, and the partial is b (0x0181). Product
# rounded first: 1.75 * 2^-149 becomes 2^-148 (subnormal quantum 2^-149),
# the sum m - 2^-148 is an fp32 tie that goes to the even m, and m is a bf16
# tie that goes to the even b + 2^-131 (0x0182).
FMA_PIN_X = [0x3F81, 0x1E80, 0xB880, 0x37E0]     # 1+2^-7, 2^-66, -2^-14, 1.75*2^-16
FMA_PIN_W = [0x0180, 0x1E80, 0x0001, 0x0001]     # 2^-124, 2^-66, 2^-133, 2^-133


def _chain(xs, ws, fused):
    acc = Fraction(0)
    for xb, wb in zip(xs, ws):
        prod = bf16_value(xb) * bf16_value(wb)
        acc = round_f32_exact(acc + (prod if fused else round_f32_exact(prod)))
    return round_bf16_exact(acc)


def test_partial_adds_each_product_with_one_rounding():
    fused = _chain(FMA_PIN_X, FMA_PIN_W, True)
    rounded_first = _chain(FMA_PIN_X, FMA_PIN_W, False)
    assert (fused, rounded_first) == (0x0181, 0x0182)    # the two readings differ here
    x = np.array([FMA_PIN_X], dtype=np.uint16)
    w = np.array([FMA_PIN_W], dtype=np.uint16)
    p, _, _ = oracle.partials(1, x, w)
    assert int(p[0, 0, 0]) == fused


def test_partials_within_recursive_summation_bound():
    rng = np.random.default_rng(9)
    n, m, k, rows = 2, 2, 256, 12
    x = _bits(rng.standard_normal((m, k)))
    w = _bits(rng.standard_normal((rows, k)) * 0.02)
    p, _, _ = oracle.partials(n, x, w)
    ks = k // n
    for r in range(n):
        for t in range(m):
            for i in range(rows):
                terms = [bf16_value(x[t, r * ks + j]) * bf16_value(w[i, r * ks + j])
                         for j in range(ks)]
                exact = sum(terms, Fraction(0))
                bound = Fraction(gamma(ks - 1)) * sum(abs(v) for v in terms)
                lo = round_bf16_exact(exact - bound)
                hi = round_bf16_exact(exact + bound)
                got = bf16_value(p[r, t, i])
                assert bf16_value(lo) <= got <= bf16_value(hi)


def test_tiny_dense_within_propagated_bound():
    cfg = get_config("tiny")
    for pt in cfg.points:
        x = point_tensor(cfg, pt, KIND_X)
        w = point_tensor(cfg, pt, KIND_W)
        res = point_tensor(cfg, pt, KIND_RESIDUAL)
        got = oracle.reconcile(cfg.n_ranks, cfg.hidden, u16(x), u16(w), u16(res))
        xd, wd, rd = x.double(), w.double(), res.double()
        n, ks = cfg.n_ranks, pt.k // cfg.n_ranks
        e = torch.stack([xd[:, r * ks:(r + 1) * ks] @ wd[:, r * ks:(r + 1) * ks].T
                         for r in range(n)])                        # exact partials [N, M, H]
        a = torch.stack([xd[:, r * ks:(r + 1) * ks].abs() @ wd[:, r * ks:(r + 1) * ks].abs().T
                         for r in range(n)])
        ref = rd + e.sum(0)
        # partial: recursive fp32 sum, then one bf16 rounding
        perr = gamma(ks - 1) * a + U * (e.abs() + gamma(ks - 1) * a)
        pmag = e.abs() + perr
        # ring: N-1 bf16 adds, each within U of a value bounded by sum |P|
        ring_err = (n - 1) * U * (1 + U) ** n * pmag.sum(0)
        # residual add: one more rounding
        out_err = U * (rd.abs() + pmag.sum(0) + ring_err)
        bound = perr.sum(0) + ring_err + out_err + 2 ** -120
        err = (torch.from_numpy(oracle.f32(got["out"])).double() - ref).abs()
        assert torch.all(err <= bound), float((err - bound).max())
        # the bound is tight enough that dropping one rank's partial breaks it
        assert torch.all(e.abs().max(0).values > 0)
        dropped = (torch.from_numpy(oracle.f32(got["out"])).double() - (ref - e[0])).abs()
        assert (dropped > bound).float().mean() > 0.5


def test_weight_zero_gives_residual():
    rng = np.random.default_rng(1)
    n, m, k, h = 4, 3, 64, 32
    x = _bits(rng.standard_normal((m, k)))
    w = np.zeros((h, k), np.uint16)
    res = _bits(rng.standard_normal((m, h)))
    got = oracle.reconcile(n, h, x, w, res)
    assert np.array_equal(got["out"], res)


def test_n1_has_no_ring():
    rng = np.random.default_rng(2)
    m, k, h = 2, 48, 16
    x = _bits(rng.standard_normal((m, k)))
    w = _bits(rng.standard_normal((h, k)) * 0.02)
    res = _bits(rng.standard_normal((m, h)))
    got = oracle.reconcile(1, h, x, w, res)
    p, _, _ = oracle.partials(1, x, w)
    assert np.array_equal(got["out"], oracle.residual(res, p[0]))
    assert int(got["bytes_sent"][0]) == 0


def test_one_hot_x_selects_weights():
    rng = np.random.default_rng(3)
    n, k, h = 4, 64, 16
    w = _bits(rng.standard_normal((h, k)) * 0.02)
    j = 37                                         # in rank 37 // 16 = 2's slice
    x = np.zeros((1, k), np.uint16)
    x[0, j] = 0x3F80                               # 1.0
    p, _, _ = oracle.partials(n, x, w)
    for r in range(n):
        want = w[:, j] if r == j // (k // n) else np.zeros(h, np.uint16)
        assert np.array_equal(p[r, 0], want)


def test_thread_count_does_not_change_bits():
    rng = np.random.default_rng(4)
    n, m, k, h = 2, 3, 128, 40
    x = _bits(rng.standard_normal((m, k)))
    w = _bits(rng.standard_normal((h, k)) * 0.02)
    res = _bits(rng.standard_normal((m, h)))
    a = oracle.reconcile(n, h, x, w, res, threads=1)
    b = oracle.reconcile(n, h, x, w, res, threads=7)
    assert np.array_equal(a["out"], b["out"])
    assert np.array_equal(a["partials"], b["partials"])


def test_column_subset_matches_full():
    cfg = get_config("tiny")
    pt = cfg.points[1]
    x, w, res = (u16(point_tensor(cfg, pt, kd)) for kd in (KIND_X, KIND_W, KIND_RESIDUAL))
    full = oracle.reconcile(cfg.n_ranks, cfg.hidden, x, w, res)
    cols = np.array([0, 1, 127, 128, 200, 255])
    sub = oracle.reconcile(cfg.n_ranks, cfg.hidden, x, np.ascontiguousarray(w[cols]),
                           np.ascontiguousarray(res[:, cols]), cols=cols)
    assert np.array_equal(sub["out"], full["out"][:, cols])


def test_rejects_indivisible_k():
    with pytest.raises(oracle.OracleError):
        oracle.partials(3, np.zeros((1, 10), np.uint16), np.zeros((2, 10), np.uint16))
