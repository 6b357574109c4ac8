"""Pins of the oracle's NVFP4 weight shards against the format's definition.

* the E2M1 grid: the eight magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6 and the sign
  bit 3; every code round-trips; every midpoint between neighbours goes to
  the even magnitude index; values at or beyond 6 saturate;
* the second-level exponent g: amax / 2^g <= 6 * 448 < amax / 2^(g-1) (the
  smallest such g), 0 for an all-zero tensor;
* the block scale: the E4M3 value nearest to the block maximum / (6 * 2^g);
* every element is within half a grid step of its exact scaled value (or
  saturated), and weights already on the grid come back unchanged;
* two codes per byte, the earlier k in the low nibble; blocks of 16 inside a
  rank slice; dequantisation is exact in bf16.
"""

import numpy as np
import pytest

import oracle
from helpers import round_bf16_float

MAGS = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e2m1_grid_and_round_trip():
    for c in range(16):
        v = oracle.e2m1_value(c)
        assert abs(v) == MAGS[c & 7] and (v < 0) == bool(c & 8 and c != 8)
        assert oracle.e2m1_rne(v if c != 8 else -0.0) == c


@pytest.mark.parametrize("v,code", [
    (0.25, 0), (0.75, 2), (1.25, 2), (1.75, 4), (2.5, 4), (3.5, 6), (5.0, 6),   # ties to even index
    (0.2499, 0), (0.2501, 1), (5.0001, 7), (4.9999, 6),                       # either side of a tie
    (6.0, 7), (6.5, 7), (1e9, 7), (-1e9, 15), (-0.75, 10),                     # saturation, sign
])
def test_e2m1_midpoints_and_saturation(v, code):
    assert oracle.e2m1_rne(v) == code


@pytest.mark.parametrize("amax", [0.1, 0.02 * 4.3, 1.0, 2688.0, 2688.0001, 3e-30, 7.5e20])
def test_global_exponent_rule(amax):
    g = oracle.nvfp4_global_exp(amax)
    assert amax / 2.0 ** g <= 6 * 448
    assert amax / 2.0 ** (g - 1) > 6 * 448
    assert oracle.nvfp4_global_exp(0.0) == 0


def _bf16(vals):
    return np.array([round_bf16_float(v) for v in vals], dtype=np.uint16)


def test_block_scale_and_element_rule():
    rng = np.random.default_rng(7)
    n, h, k = 2, 6, 128
    w = _bf16(rng.normal(0, 0.02, size=h * k)).reshape(h, k)
    q, sc, g = oracle.nvfp4_quantize(n, w)
    wf = oracle.f32(w).astype(np.float64)
    amax = np.abs(wf).max()
    assert g == oracle.nvfp4_global_exp(amax)
    ks = k // n
    for r in range(n):
        for row in range(h):
            for b in range(ks // 16):
                blk = wf[row, r * ks + 16 * b: r * ks + 16 * b + 16]
                bs = oracle.e4m3_value(int(sc[r, row, b]))
                assert sc[r, row, b] == oracle.e4m3_rne(np.abs(blk).max() / (6 * 2.0 ** g))
                for i, wv in enumerate(blk):
                    j = 16 * b + i
                    byte = int(q[r, row, j // 2])
                    c = byte & 0xF if j % 2 == 0 else byte >> 4
                    got = oracle.e2m1_value(c)
                    exact = wv / (bs * 2.0 ** g)
                    if abs(exact) < 6:
                        # half the larger neighbouring step of the E2M1 grid
                        step = 0.5 if abs(exact) <= 2 else (1.0 if abs(exact) <= 4 else 2.0)
                        assert abs(got - exact) <= step / 2 + 1e-12, (r, row, j, exact, got)
                    else:
                        assert abs(got) == 6.0


def test_grid_weights_come_back_unchanged_and_nibble_order():
    # one rank, one row, 32 weights (two blocks of 16) already on the grid
    # times 2^-8: amax = 6 * 2^-8 gives g = -16, each block's scale is the
    # E4M3 value 256, and every weight divided by 256 * 2^-16 is a grid value
    vals = [m * s for s in (1, -1) for m in MAGS] * 2            # 32 values
    w64 = np.array(vals, dtype=np.float64) * 2.0 ** -8
    w = _bf16(w64).reshape(1, 32)
    q, sc, g = oracle.nvfp4_quantize(1, w)
    back = oracle.nvfp4_dequant_bf16(1, q, sc, g)
    assert np.array_equal(back, w)
    # earlier k in the low nibble: weights 0 and 1 of the row are +0 and +0.5 (codes 0, 1)
    assert q[0, 0, 0] == 0x10
    assert q[0, 0, 1] == (3 << 4) | 2                            # +1.5 over +1.0


def test_dequant_exact_in_bf16_and_zero_tensor():
    rng = np.random.default_rng(11)
    w = _bf16(rng.normal(0, 0.02, size=4 * 256)).reshape(4, 256)
    q, sc, g = oracle.nvfp4_quantize(4, w)
    back = oracle.nvfp4_dequant_bf16(4, q, sc, g)            # raises if not exact
    assert back.shape == w.shape
    z = np.zeros((3, 64), dtype=np.uint16)
    q, sc, g = oracle.nvfp4_quantize(2, z)
    assert g == 0 and not q.any() and not sc.any()


def test_rejects_slices_not_in_blocks_of_16():
    with pytest.raises(oracle.OracleError):
        oracle.nvfp4_quantize(2, np.zeros((2, 48), dtype=np.uint16))
