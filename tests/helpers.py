"""Shared test helpers: bf16 bit views, exact rational rounding, golden files."""

from __future__ import annotations

import math
import os
from fractions import Fraction

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def golden_rows(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


def u16(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> numpy uint16 bit patterns (CPU copy)."""
    assert t.dtype == torch.bfloat16
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def from_u16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)


def bf16_value(b: int) -> Fraction:
    """Exact rational value of a finite bf16 bit pattern."""
    b = int(b) & 0xFFFF
    sign = -1 if b & 0x8000 else 1
    e = (b >> 7) & 0xFF
    m = b & 0x7F
    assert e != 0xFF, "not finite"
    if e == 0:
        return sign * Fraction(m, 1 << 7) * Fraction(1, 1 << 126)
    return sign * (1 + Fraction(m, 1 << 7)) * Fraction(2) ** (e - 127)


def round_bf16_exact(v: Fraction) -> int:
    """Correct round-to-nearest-even of an exact rational to a bf16 pattern.

    Written from the IEEE 754 definition: pick the representable value nearest
    to v (8 significant bits, exponent -126..127, subnormal quantum 2^-133),
    ties to the even significand, overflow to infinity when |v| reaches
    (2 - 2^-8) * 2^127, the midpoint above the largest finite bf16.
    """
    sign = 0x8000 if v < 0 else 0
    a = -v if v < 0 else v
    if a == 0:
        return sign
    if a >= (2 - Fraction(1, 256)) * Fraction(2) ** 127:
        return sign | 0x7F80
    # exponent e with 2^e <= a < 2^(e+1)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    q = max(e - 7, -133)                     # quantum of the binade (or subnormal)
    scaled = a / Fraction(2) ** q
    n = math.floor(scaled)
    rem = scaled - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    val = n * Fraction(2) ** q
    if val >= Fraction(2) ** 128:
        return sign | 0x7F80
    # encode
    if val < Fraction(2) ** -126:
        mant = int(val / Fraction(2) ** -133)
        return sign | mant
    e2 = val.numerator.bit_length() - val.denominator.bit_length()
    if Fraction(2) ** e2 > val:
        e2 -= 1
    mant = int((val / Fraction(2) ** e2 - 1) * 128)
    return sign | ((e2 + 127) << 7) | mant


def bf16_finite_patterns():
    """All finite bf16 patterns as numpy uint16."""
    a = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    return a[(a & 0x7F80) != 0x7F80]


def round_bf16_float(v) -> int:
    """Correct rounding of a finite float (float32 or float64) to bf16, with the
    sign of zero kept (an exact rational has no signed zero)."""
    v = float(v)
    if v == 0.0:
        return 0x8000 if math.copysign(1.0, v) < 0 else 0
    return round_bf16_exact(Fraction(v))


def round_f32_exact(v: Fraction) -> Fraction:
    """Correct round-to-nearest-even of an exact rational to an IEEE binary32
    value (returned as an exact rational), from the format's definition: 24
    significant bits, exponent down to -126, subnormal quantum 2^-149;
    |v| at or above the largest finite value's upper midpoint is refused."""
    if v == 0:
        return Fraction(0)
    a = -v if v < 0 else v
    assert a < (2 - Fraction(1, 1 << 24)) * Fraction(2) ** 127, "overflow"
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    q = max(e - 23, -149)
    scaled = a / Fraction(2) ** q
    n = math.floor(scaled)
    rem = scaled - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    r = n * Fraction(2) ** q
    return -r if v < 0 else r


def mx_scales_as_stored(sc):
    """The oracle's MXFP8 scales [N][H][K/N/32] in the library's storage order,
    flattened: [N][ceil(H/128)][ceil(K/N/128)] chunks of 512 bytes, row t of a
    128-row tile and run j (of the chunk's four 32-column runs) at byte
    16 (t % 32) + 4 (t // 32) + j; zeros where rows pass H or runs pass K/N.
    A permutation plus padding only."""
    sc = np.asarray(sc, dtype=np.uint8)
    n, h, nb = sc.shape
    ht, kg = (h + 127) // 128, (nb + 3) // 4
    pad = np.zeros((n, ht * 128, kg * 4), dtype=np.uint8)
    pad[:, :h, :nb] = sc
    # (rank, tile, t // 32, t % 32, chunk, j) -> (rank, tile, chunk, t % 32, t // 32, j)
    return np.ascontiguousarray(pad.reshape(n, ht, 4, 32, kg, 4).transpose(0, 1, 4, 3, 2, 5)).reshape(-1)


def x_split_exponent(amax):
    """E8M0 exponent e1 of the block-scaled form's first activation term for
    32-value runs with largest magnitude amax: floor(log2 amax) - 7, at
    least -127."""
    a = np.asarray(amax, dtype=np.float64)
    _, e = np.frexp(np.where(a > 0, a, 1.0))
    return np.where(a > 0, np.maximum(e - 1 - 7, -127), -127).astype(np.int64)


def x_split_error_bound(n, x_u16, w_u16):
    """Bound on how far the block-scaled MXFP8 form's partials [N][M][H] can
    move from the exact products by splitting each activation into two E4M3
    terms (x = 2^e1 q1 + 2^e2 q2 per 32-value run of a rank slice): an x below
    2^(e1 - 6) may be off by 2^(e1 - 14), any x by at most 2^-137 (runs so
    small that the second term's exponent stops at -127); each error is
    weighted by |w|. x [M][K], w [H][K] as bf16 bit patterns."""
    from oracle import f32
    x = f32(np.asarray(x_u16, dtype=np.uint16)).astype(np.float64)
    w = np.abs(f32(np.asarray(w_u16, dtype=np.uint16)).astype(np.float64))
    m, k = x.shape
    ks = k // n
    runs = np.abs(x).reshape(m, n, ks // 32, 32)
    e1 = x_split_exponent(runs.max(axis=3))[..., None]
    err = np.where(runs < np.ldexp(1.0, e1 - 6), np.ldexp(1.0, e1 - 14), 0.0) + 2.0 ** -137
    err = err.reshape(m, n, ks)
    return np.stack([err[:, r, :] @ w[:, r * ks:(r + 1) * ks].T for r in range(n)])


def nv_scales_as_stored(sc, g, amax_bits):
    """The oracle's NVFP4 block scales [N][H][K/N/16] and exponent g in the
    library's storage order: [N][K/N/64][H][4], flattened, then 16 bytes
    (g as int32, the weight's largest magnitude as bf16 bits in an int32,
    8 zero bytes). A permutation and a packing only."""
    sc = np.asarray(sc)
    n, h, nb = sc.shape
    assert nb % 4 == 0
    body = np.ascontiguousarray(sc.reshape(n, h, nb // 4, 4).transpose(0, 2, 1, 3)).reshape(-1)
    trailer = np.array([g, amax_bits, 0, 0], dtype=np.int32).view(np.uint8)
    return np.concatenate([body, trailer])
