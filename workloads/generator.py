"""Counter-based seeded bf16 generator, bit-identical on CPU and CUDA.

Uniform bits: Philox4x32-10 as defined by Salmon, Moraes, Dror and Shaw
("Parallel random numbers: as easy as 1, 2, 3", SC'11): a 4x32-bit counter and
a 2x32-bit key, ten rounds, each round multiplying words 0 and 2 by the two
Philox constants, swapping and xoring the high halves with the other words and
the round key, with the key bumped by the two Weyl constants between rounds.

Gaussian values: each Philox block gives eight 16-bit uniforms u. A value is
``table[u]`` where ``table[i]`` is the bf16 rounding of sigma * Phi^-1((i+1/2)/2^16),
the standard normal quantile at the midpoint of the i-th of 2^16 equal
probability bins (inverse-transform sampling on a 2^16-point grid, whose tail
is cut at 4.32 sigma). The table is built once on the host in float64
(``statistics.NormalDist``) and the lookup is a gather, so the CPU and the
CUDA device produce the same bits with no transcendental function on either.

All arithmetic is on int64 torch tensors holding 32-bit words, so the same
code runs on any torch device. The 32x32->64-bit products are split into
16-bit halves so that no intermediate leaves the int64 range.

Element j of a tensor uses Philox block j // 8 (counter = (block lo, block hi,
0, 0), key = (seed, tensor id)) and its 16-bit half j % 8 (word (j % 8) // 2,
low half first).
"""

from __future__ import annotations

import functools
from statistics import NormalDist
from typing import Iterable, Sequence

import torch

MASK32 = 0xFFFFFFFF
PHILOX_M0 = 0xD2511F53
PHILOX_M1 = 0xCD9E8D57
PHILOX_W0 = 0x9E3779B9
PHILOX_W1 = 0xBB67AE85

KIND_X = 0
KIND_W = 1
KIND_RESIDUAL = 2


def tensor_id(point_index: int, kind: int) -> int:
    """Substream id of one tensor of one reconciliation point."""
    return point_index * 4 + kind


def _mulhilo(a: torch.Tensor, m: int):
    """(hi, lo) 32-bit words of the 64-bit product a*m, a in [0, 2^32)."""
    m_hi, m_lo = m >> 16, m & 0xFFFF
    t = a * m_hi                      # < 2^48
    s = ((t & 0xFFFF) << 16) + a * m_lo   # < 2^49
    lo = s & MASK32
    hi = (t >> 16) + (s >> 32)
    return hi & MASK32, lo


def philox4x32_10(c0, c1, c2, c3, k0: int, k1: int):
    """Philox4x32-10 on int64 tensors (or ints) holding 32-bit words."""
    c = [torch.as_tensor(v, dtype=torch.int64) for v in (c0, c1, c2, c3)]
    k0 &= MASK32
    k1 &= MASK32
    for rnd in range(10):
        if rnd:
            k0 = (k0 + PHILOX_W0) & MASK32
            k1 = (k1 + PHILOX_W1) & MASK32
        hi0, lo0 = _mulhilo(c[0], PHILOX_M0)
        hi1, lo1 = _mulhilo(c[2], PHILOX_M1)
        c = [hi1 ^ c[1] ^ k0, lo1, hi0 ^ c[3] ^ k1, lo0]
    return c


@functools.lru_cache(maxsize=None)
def _table_cpu(sigma: float) -> torch.Tensor:
    nd = NormalDist()
    q = [sigma * nd.inv_cdf((i + 0.5) / 65536.0) for i in range(65536)]
    return torch.tensor(q, dtype=torch.float64).to(torch.float32).to(torch.bfloat16)


_table_dev_cache = {}


def gaussian_table(sigma: float, device="cpu") -> torch.Tensor:
    """The 2^16-entry bf16 quantile table for standard deviation sigma."""
    dev = torch.device(device)
    if dev.type == "cpu":
        return _table_cpu(float(sigma))
    key = (float(sigma), str(dev))
    t = _table_dev_cache.get(key)
    if t is None:
        t = _table_cpu(float(sigma)).to(dev)
        _table_dev_cache[key] = t
    return t


def _uniform16(seed: int, tid: int, start: int, count: int, device) -> torch.Tensor:
    """16-bit uniforms for elements [start, start+count) of substream (seed, tid)."""
    if count == 0:
        return torch.empty(0, dtype=torch.int64, device=device)
    b0 = start // 8
    b1 = (start + count - 1) // 8 + 1
    blocks = torch.arange(b0, b1, dtype=torch.int64, device=device)
    w = philox4x32_10(blocks & MASK32, blocks >> 32, torch.zeros_like(blocks),
                      torch.zeros_like(blocks), seed, tid)
    words = torch.stack(w, dim=1)                          # [nblk, 4]
    halves = torch.stack([words & 0xFFFF, words >> 16], dim=2)  # [nblk, 4, 2]
    u = halves.reshape(-1)
    off = start - b0 * 8
    return u[off:off + count]


def gaussian_bf16(seed: int, tid: int, start: int, count: int, sigma: float,
                  device="cpu", chunk: int = 1 << 24) -> torch.Tensor:
    """bf16 N(0, sigma^2) draws for elements [start, start+count) of a substream."""
    dev = torch.device(device)
    out = torch.empty(count, dtype=torch.bfloat16, device=dev)
    table = gaussian_table(sigma, dev)
    pos = 0
    while pos < count:
        n = min(chunk, count - pos)
        u = _uniform16(seed, tid, start + pos, n, dev)
        out[pos:pos + n] = table[u]
        pos += n
    return out


def point_tensor(cfg, point, kind: int, device="cpu") -> torch.Tensor:
    """Whole tensor of one point: x [M, K], W [H, K] or residual [M, H]."""
    m, h, k = cfg.tokens, cfg.hidden, point.k
    shape, sigma = {
        KIND_X: ((m, k), cfg.sigma_x),
        KIND_W: ((h, k), cfg.sigma_w),
        KIND_RESIDUAL: ((m, h), cfg.sigma_res),
    }[kind]
    n = shape[0] * shape[1]
    v = gaussian_bf16(cfg.seed, tensor_id(point.index, kind), 0, n, sigma, device)
    return v.view(*shape)


def point_tensor_rows(cfg, point, kind: int, rows: Sequence[int], device="cpu") -> torch.Tensor:
    """Selected rows of one point's tensor (same bits as the whole tensor's rows).

    For W the rows are output features h (rows of the [H, K] Linear weight);
    for x and the residual they are tokens m.
    """
    m, h, k = cfg.tokens, cfg.hidden, point.k
    width, sigma = {
        KIND_X: (k, cfg.sigma_x),
        KIND_W: (k, cfg.sigma_w),
        KIND_RESIDUAL: (h, cfg.sigma_res),
    }[kind]
    tid = tensor_id(point.index, kind)
    parts = [gaussian_bf16(cfg.seed, tid, int(r) * width, width, sigma, device) for r in rows]
    if not parts:
        return torch.empty(0, width, dtype=torch.bfloat16, device=device)
    return torch.stack(parts, 0)


def point_columns(cfg, point, kind: int, cols: Iterable[int], device="cpu") -> torch.Tensor:
    """Selected columns of the residual [M, H] (all tokens), as [M, len(cols)]."""
    res = point_tensor(cfg, point, kind, device)
    idx = torch.as_tensor(list(cols), dtype=torch.int64, device=res.device)
    return res[:, idx].contiguous()
