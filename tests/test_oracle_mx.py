"""Pins of the oracle's MXFP8 weight shards (OCP Microscaling v1.0, MXFP8
E4M3: 32-element blocks along K sharing an E8M0 power-of-two scale).

What the format fixes and these tests check:
* the E4M3 grid: bias 7, 3 fraction bits, largest finite 448 (0x7E), smallest
  normal 2^-6 (0x08), smallest subnormal 2^-9 (0x01), 0x7F is NaN and is
  never produced; every code's value against that closed form;
* the element conversion: every representable value encodes to its own code,
  every midpoint between neighbouring codes goes to the even code and anything
  off the midpoint to the nearer code, values at or above 448 saturate;
* the scale: X = 2^(floor(log2 amax) - 8), so a block's largest magnitude
  lands in [256, 512) before rounding; an all-zero block has X = 2^-127;
* blocks follow each rank's slice of K and never straddle two ranks;
* dequantised weights are within half a unit of the E4M3 grid of the
  original (or equal 448 X when saturated), and weights already on the grid
  come back unchanged.
"""

import math

import numpy as np
import pytest

import torch

import oracle


def round_bf16_exact(a):
    """float32 array -> bf16 bit patterns (round to nearest even)."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bf16_value(b):
    """bf16 bit patterns -> float64 values (exact)."""
    return oracle.f32(np.ascontiguousarray(b, dtype=np.uint16)).astype(np.float64)


def _code_value(c):
    e, m = (c >> 3) & 0xF, c & 7
    mag = m * 2.0 ** -9 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7)
    return -mag if c & 0x80 else mag


def _finite_codes():
    return [c for c in range(256) if (c & 0x7F) != 0x7F]


def test_e4m3_grid_landmarks():
    assert oracle.e4m3_value(0x7E) == 448.0
    assert oracle.e4m3_value(0x08) == 2.0 ** -6
    assert oracle.e4m3_value(0x01) == 2.0 ** -9
    assert oracle.e4m3_value(0x38) == 1.0
    for c in _finite_codes():
        assert oracle.e4m3_value(c) == _code_value(c)


def test_e4m3_every_code_round_trips():
    for c in _finite_codes():
        assert oracle.e4m3_rne(_code_value(c)) == c, hex(c)


def test_e4m3_midpoints_go_to_even_and_saturation():
    pos = sorted((_code_value(c), c) for c in range(0x7F) if c != 0x7F)
    for (a, ca), (b, cb) in zip(pos, pos[1:]):
        mid = (a + b) / 2
        even = ca if ca % 2 == 0 else cb
        assert oracle.e4m3_rne(mid) == even, (a, b)
        assert oracle.e4m3_rne(-mid) == even | 0x80
        step = (b - a) / 8
        assert oracle.e4m3_rne(mid - step) == ca
        assert oracle.e4m3_rne(mid + step) == cb
    for v in (448.0, 449.0, 464.0, 480.0, 511.9, 1e6):
        assert oracle.e4m3_rne(v) == 0x7E
        assert oracle.e4m3_rne(-v) == 0xFE
    assert oracle.e4m3_rne(0.0) == 0x00 and oracle.e4m3_rne(-0.0) == 0x80


def _block_weights(rng, h, k, scale=0.02):
    w = rng.normal(0.0, scale, size=(h, k)).astype(np.float32)
    return round_bf16_exact(w)


def test_scale_rule_and_block_max():
    rng = np.random.default_rng(7)
    n, h, k = 2, 6, 256
    w = _block_weights(rng, h, k)
    q, sc = oracle.mx_quantize(n, w)
    wf = bf16_value(w)
    ks = k // n
    for r in range(n):
        for i in range(h):
            for b in range(ks // 32):
                blk = wf[i, r * ks + 32 * b: r * ks + 32 * b + 32]
                amax = float(np.max(np.abs(blk)))
                s = math.floor(math.log2(amax)) - 8
                assert sc[r, i, b] == s + 127
                assert 256.0 <= amax / 2.0 ** s < 512.0
                j = int(np.argmax(np.abs(blk)))
                code = int(q[r, i, 32 * b + j])
                assert abs(_code_value(code)) == min(448.0, abs(_code_value(oracle.e4m3_rne(amax / 2.0 ** s))))


def test_zero_block_and_rank_boundaries():
    n, h, k = 2, 1, 64
    w = np.zeros((h, k), dtype=np.float32)
    w[0, 32:] = 3.0                              # rank 0's second block: a distinct scale
    w[0, 0] = 0.0
    wb = round_bf16_exact(w)
    q, sc = oracle.mx_quantize(n, wb)
    assert sc[0, 0, 0] == 0 and not q[0, 0, :32].any()        # all-zero block
    assert sc[0, 0, 0 + 0] == 0
    assert sc[1, 0, 0] == math.floor(math.log2(3.0)) - 8 + 127  # rank 1's block holds 3.0
    w2 = np.zeros((1, 64), dtype=np.float32)
    w2[0, :32] = 1.0                              # rank 0 only
    w2[0, 32:] = 2.0 ** -20                       # rank 1 only
    q2, sc2 = oracle.mx_quantize(2, round_bf16_exact(w2))
    assert sc2[0, 0, 0] == 0 - 8 + 127 and sc2[1, 0, 0] == -20 - 8 + 127


def test_dequant_error_bound_and_grid_fixed_points():
    rng = np.random.default_rng(11)
    n, h, k = 4, 8, 512
    w = _block_weights(rng, h, k)
    q, sc = oracle.mx_quantize(n, w)
    d = bf16_value(oracle.mx_dequant_bf16(n, q, sc))
    wf = bf16_value(w)
    ks = k // n
    for r in range(n):
        for i in range(h):
            for b in range(ks // 32):
                sl = slice(r * ks + 32 * b, r * ks + 32 * b + 32)
                s = int(sc[r, i, b]) - 127
                x = 2.0 ** s
                for wv, dv in zip(wf[i, sl], d[i, sl]):
                    v = abs(wv) / x
                    if v >= 448:
                        assert abs(dv) == 448 * x
                    elif v < 2.0 ** -6:
                        assert abs(dv - wv) <= 2.0 ** -10 * x
                    else:
                        assert abs(dv - wv) <= 2.0 ** (math.floor(math.log2(v)) - 4) * x
    # weights already on the grid of their block come back unchanged
    q2, sc2 = oracle.mx_quantize(n, oracle.mx_dequant_bf16(n, q, sc))
    assert np.array_equal(q2, q) and np.array_equal(sc2, sc)


def test_mx_rejects_bad_shapes():
    w = np.zeros((2, 96), dtype=np.uint16)
    with pytest.raises(oracle.OracleError):
        oracle.mx_quantize(2, w)                 # K/N = 48 is not a multiple of 32
