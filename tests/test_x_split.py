"""The activation split of the block-scaled MXFP8 form, against its stated
error bound.

For at most 8 tokens the MXFP8 codes go to the tensor cores as stored, and
each 32-value run of a bf16 activation row is written as two E4M3 terms with
E8M0 scales of their own: e1 = floor(log2 max|x|) - 7 (at least -127), q1 the
E4M3 value nearest x / 2^e1 (ties to even), r = x - 2^e1 q1, e2 the same rule
on max|r|, q2 the E4M3 value nearest r / 2^e2. The claim the parity margin
rests on (helpers.x_split_error_bound):

    |x - (2^e1 q1 + 2^e2 q2)| <= (2^(e1 - 14) if |x| < 2^(e1 - 6) else 0) + 2^-137

and no term saturates (|x| / 2^e1 < 256 < 448). This test models those steps
in exact arithmetic (every step is exact in f32 as well: products by powers
of two and differences of nearby values with few significant bits) and checks
the claim for every finite bf16 magnitude, both signs, under run maxima from
the smallest subnormal to the largest finite value. E4M3 rounding uses the
oracle's code table (pinned in test_oracle_mx.py).
"""

import numpy as np
import pytest

import oracle
from helpers import x_split_exponent


def _e4m3_table():
    return np.array([oracle.e4m3_value(c) for c in range(0x7F)], dtype=np.float64)   # 0 .. 448


E4M3 = _e4m3_table()


def e4m3_rne(v):
    """Nearest E4M3 value to each v (|v| <= 448 here), ties to the even code."""
    a = np.abs(v)
    hi = np.clip(np.searchsorted(E4M3, a), 0, len(E4M3) - 1)
    lo = np.clip(hi - 1, 0, len(E4M3) - 1)
    dlo, dhi = a - E4M3[lo], E4M3[hi] - a
    pick = np.where(dlo < dhi, lo, np.where(dhi < dlo, hi, np.where(lo % 2 == 0, lo, hi)))
    return np.sign(v) * E4M3[pick]


def split(runs):
    """runs [R, 32] exact values -> (2^e1 q1 + 2^e2 q2, e1, the largest |x| / 2^e1)."""
    e1 = x_split_exponent(np.abs(runs).max(axis=1))[:, None]
    y = np.ldexp(runs, -e1)
    t1 = np.ldexp(e4m3_rne(y), e1)
    r = runs - t1
    e2 = x_split_exponent(np.abs(r).max(axis=1))[:, None]
    t2 = np.ldexp(e4m3_rne(np.ldexp(r, -e2)), e2)
    return t1 + t2, e1, np.abs(y).max()


@pytest.mark.parametrize("amax_bits", [0x3F80, 0x3FFF, 0x3E40, 0x0780, 0x7F7F, 0x0001, 0x3B00, 0x0080])
def test_split_within_bound(amax_bits):
    amax = float(oracle.f32(np.array([amax_bits], dtype=np.uint16))[0])
    pats = np.arange(0, 0x7F80, dtype=np.uint32).astype(np.uint16)            # finite magnitudes
    vals = oracle.f32(pats).astype(np.float64)
    keep = vals[vals <= amax]
    both = np.concatenate([keep, -keep])
    nr = (len(both) + 30) // 31
    runs = np.zeros((nr, 32))
    runs[:, 0] = amax                                    # every run has the same maximum
    runs[:, 1:].flat[:len(both)] = both
    got, e1, ymax = split(runs)
    assert ymax < 256                                    # q1 never saturates
    bound = np.where(np.abs(runs) < np.ldexp(1.0, e1 - 6), np.ldexp(1.0, e1 - 14), 0.0) + 2.0 ** -137
    assert np.all(np.abs(runs - got) <= bound)
    if amax >= 2.0 ** -100:                              # ordinary magnitudes
        big = np.abs(runs) >= np.ldexp(1.0, e1 - 6)
        assert np.array_equal(got[big], runs[big])        # exact where the bound says 0


def test_split_exact_for_gaussian_runs():
    """N(0,1) activations: every value at least 2^-13 of its run's maximum
    splits exactly; the rest stay inside the bound."""
    rng = np.random.default_rng(7)
    x = oracle.f32(oracle.bf16_rne(rng.standard_normal(32 * 4096).astype(np.float32))).astype(np.float64)
    runs = x.reshape(-1, 32)
    got, e1, _ = split(runs)
    small = np.abs(runs) < np.ldexp(1.0, e1 - 6)
    assert np.array_equal(got[~small], runs[~small])
    bound = np.broadcast_to(np.ldexp(1.0, e1 - 14), runs.shape)
    assert np.all(np.abs(runs - got)[small] <= bound[small] + 2.0 ** -137)


def test_margin_bounds_the_split_partials():
    """helpers.x_split_error_bound against the exact effect of the split on
    each partial (sum over k of (x - split(x)) * w, one rank slice), on inputs
    that put small values into runs with large maxima."""
    from helpers import x_split_error_bound
    rng = np.random.default_rng(11)
    n, m, k, h = 2, 3, 256, 8
    x = rng.standard_normal((m, k)).astype(np.float32)
    x[:, ::7] *= 1e-5                                    # values far below their run's maximum
    w = (0.02 * rng.standard_normal((h, k))).astype(np.float32)
    xb, wb = oracle.bf16_rne(x), oracle.bf16_rne(w)
    xv = oracle.f32(xb).astype(np.float64)
    wv = oracle.f32(wb).astype(np.float64)
    got, _, _ = split(xv.reshape(-1, 32))
    err = (xv - got.reshape(m, k))
    ks = k // n
    exact = np.stack([np.abs(err[:, r * ks:(r + 1) * ks] @ wv[:, r * ks:(r + 1) * ks].T) for r in range(n)])
    bound = x_split_error_bound(n, xb, wb)
    assert exact.shape == bound.shape
    assert np.all(exact <= bound)
    assert exact.max() > 0                               # the case exercises inexact splits
