"""Pins of the oracle's bf16 arithmetic against definitions outside the oracle.

* rounding float32 -> bf16 against exact rational rounding (IEEE 754 definition)
  and against torch's float32 -> bfloat16 conversion (a library routine);
* the oracle's bf16 add (fp32 add, then one rounding, as the ring does) against
  the correctly rounded sum of the exact rationals; Figueroa ("When is double
  rounding innocuous?", 1995) shows the two agree for any intermediate of at
  least 2p+2 = 18 bits, and these tests check it on the oracle's code.
"""

import random
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from helpers import bf16_finite_patterns, bf16_value, round_bf16_exact, round_bf16_float

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _f32_exact(f: np.float32) -> Fraction:
    return Fraction(float(f))


def _edge_floats():
    vals = [0.0, -0.0, 1.0, -1.0, 256.0, 257.0, 258.0, 259.0, 1.00390625, 1.005859375,
            3.3895313892515355e38, 3.3961775292304e38, 3.4e38, 1e-38, 1e-40, 1e-45,
            9.18354961579912e-41, 9.183549615799121e-41 * 1.5, 2.0 ** -133, 2.0 ** -134,
            3 * 2.0 ** -135, 2.0 ** -149, 65504.0, 0.1, -0.1, 1.0 / 3]
    out = [np.float32(v) for v in vals]
    # every exponent, with the fraction patterns around the rounding boundary
    for e in range(0, 255):
        for frac in (0x0000, 0x7FFF, 0x8000, 0x8001, 0x17FFF, 0x18000, 0x18001, 0x7FFFFF,
                     0x7F8000, 0x7F7FFF, 0x10000):
            for s in (0, 1):
                u = (s << 31) | (e << 23) | (frac & 0x7FFFFF)
                out.append(np.array([u], dtype=np.uint32).view(np.float32)[0])
    return np.array(out, dtype=np.float32)


def test_bf16_rne_matches_exact_rounding_on_edges():
    f = _edge_floats()
    got = oracle.bf16_rne(f)
    for v, g in zip(f, got):
        want = round_bf16_float(v)
        assert int(g) == want, (float(v), hex(int(g)), hex(want))


def test_bf16_rne_matches_exact_rounding_random():
    rng = np.random.default_rng(7)
    bits = rng.integers(0, 2 ** 32, size=20000, dtype=np.uint64).astype(np.uint32)
    f = bits.view(np.float32)
    f = f[np.isfinite(f)]
    got = oracle.bf16_rne(f)
    for v, g in zip(f, got):
        assert int(g) == round_bf16_float(v)


def test_bf16_rne_matches_torch_conversion():
    rng = np.random.default_rng(11)
    bits = rng.integers(0, 2 ** 32, size=1 << 22, dtype=np.uint64).astype(np.uint32)
    f = np.concatenate([bits.view(np.float32), _edge_floats()])
    f = f[~np.isnan(f)]
    got = oracle.bf16_rne(f)
    want = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, want)


def test_bf16_rne_nan_stays_nan():
    f = np.array([np.nan, -np.nan], dtype=np.float32)
    got = oracle.bf16_rne(f)
    assert all((int(g) & 0x7F80) == 0x7F80 and (int(g) & 0x7F) != 0 for g in got)


def test_bf16_rne_f64_matches_exact_rounding():
    rng = np.random.default_rng(3)
    vals = list(rng.standard_normal(3000) * 10.0 ** rng.integers(-45, 39, 3000))
    vals += [2.0 ** -134, 2.0 ** -134 * 1.0000001, 3 * 2.0 ** -135, 2.0 ** -140,
             257.0, 257.0000001, 258.0, 259.0, (2 - 2 ** -8) * 2.0 ** 127,
             (2 - 2 ** -8) * 2.0 ** 127 * (1 - 1e-12), 1e300, -1e300, 0.0, -0.0]
    for v in vals:
        got = int(oracle.bf16_rne_f64(np.array([v]))[0])
        assert got == round_bf16_float(v), v


def _stratified_b():
    # every exponent and sign with a spread of fractions
    out = []
    for s in (0, 1):
        for e in range(0, 255):
            for m in (0, 1, 0x3F, 0x40, 0x41, 0x7E, 0x7F):
                out.append((s << 15) | (e << 7) | m)
    return np.array(out, dtype=np.uint16)


def test_bf16_add_fp32_route_equals_fp64_route_all_a():
    """Every finite a against a stratified set of b: the ring's add (fp32 add,
    one rounding) equals the correctly rounded double sum (exact for two bf16
    values unless one is far below the other's half-ulp)."""
    a_all = bf16_finite_patterns()
    b_all = _stratified_b()
    fa = oracle.f32(a_all).astype(np.float32)
    fb = oracle.f32(b_all).astype(np.float32)
    for i in range(0, b_all.size, 256):
        b = fb[i:i + 256]
        s32 = (fa[:, None] + b[None, :]).astype(np.float32)
        s64 = fa[:, None].astype(np.float64) + b[None, :].astype(np.float64)
        r32 = oracle.bf16_rne(s32)
        r64 = oracle.bf16_rne_f64(s64)
        finite = np.isfinite(s64)
        assert np.array_equal(r32[finite], r64[finite])
        nan64 = np.isnan(s64)
        assert np.all((r32[nan64] & 0x7F80) == 0x7F80)


def test_bf16_add_matches_exact_rational_sum():
    """The ring's add, through the oracle's ring with N=2 and a residual of -0
    (which leaves every sum unchanged), against exact rational rounding."""
    rng = random.Random(5)
    pats = [int(p) for p in bf16_finite_patterns()]
    special = [0x0000, 0x8000, 0x0001, 0x8001, 0x007F, 0x0080, 0x4380, 0x3F80, 0x3F81,
               0x7F7F, 0xFF7F, 0x4381, 0x3B80, 0x3B00]
    pairs = [(a, b) for a in special for b in special]
    pairs += [(rng.choice(pats), rng.choice(pats)) for _ in range(4000)]
    # near-cancellation and tie-producing pairs
    for _ in range(2000):
        a = rng.choice(pats)
        pairs.append((a, a ^ 0x8000 ^ rng.randrange(0, 4)))
        pairs.append((a, (a & 0xFF80) - (7 << 7) if (a & 0x7F80) > (8 << 7) else a))
    a = np.array([p[0] for p in pairs], dtype=np.uint16)
    b = np.array([p[1] & 0xFFFF for p in pairs], dtype=np.uint16)
    n = a.size
    parts = np.stack([a, b])[:, None, :]                         # [2, 1, n]
    red, _ = oracle.ring(2, 2 * n, np.concatenate([parts, parts], axis=2)[:, :, :],
                         cols=np.arange(2 * n))
    res = np.full((1, 2 * n), 0x8000, dtype=np.uint16)          # -0
    out = oracle.residual(res, red)[0]
    for i, (x, y) in enumerate(zip(a, b)):
        if int(x) == 0x8000 and int(y) == 0x8000:
            want = 0x8000                        # -0 + -0 = -0; any other exact zero is +0
        else:
            want = round_bf16_exact(bf16_value(x) + bf16_value(y))
        # both chunks (rank 0 first and rank 1 first) give the same: + commutes
        assert int(out[i]) == want, (hex(int(x)), hex(int(y)))
        assert int(out[n + i]) == want
