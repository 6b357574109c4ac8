"""Helpers for the GPU parity tests: seeded inputs on both sides, one point
through the C ABI, and the oracle on the same inputs."""

from __future__ import annotations

import numpy as np
import torch

import oracle
from helpers import u16
from workloads import gaussian_bf16


def draw(shape, sigma, seed, tid, device):
    n = int(np.prod(shape))
    return gaussian_bf16(seed, tid, 0, n, sigma, device).view(*shape)


def inputs(n, m, k, h, seed, device, sigma_w=0.02):
    """x [M,K], W [H,K], residual [M,H] on `device` (same bits on any device)."""
    x = draw((m, k), 1.0, seed, 0, device)
    w = draw((h, k), sigma_w, seed, 1, device)
    r = draw((m, h), 1.0, seed, 2, device)
    return x, w, r


def gpu_point(plan, x, w, res, staged=False, variant="exact"):
    """Run one point on the GPU; returns (out, partials) as CPU uint16 arrays."""
    plan.set_variant(variant, staged)
    wp = plan.pack_weights(w)
    out = plan.reconcile(x, wp, res)
    parts = plan.partials(x, wp)
    torch.cuda.synchronize()
    assert plan.device_error_flags() == 0
    return u16(out), u16(parts), wp


def oracle_point(n, h, x, w, res, cols=None, threads=8):
    xs, ws, rs = u16(x), u16(w), u16(res)
    if cols is not None:
        cols = np.asarray(cols, dtype=np.int64)
        ws = np.ascontiguousarray(ws[cols])
        rs = np.ascontiguousarray(rs[:, cols])
    return oracle.reconcile(n, h, xs, ws, rs, cols=cols, threads=threads)


def sample_cols(h, n, count=40, seed=0):
    """Output columns to check at full size: both ends of every chunk plus a spread."""
    hc = h // n
    cols = {0, 1, h - 1, h - 2}
    for c in range(n):
        cols |= {c * hc, c * hc + 1, c * hc + hc - 1}
    rng = np.random.default_rng(seed)
    cols |= set(int(v) for v in rng.integers(0, h, count))
    return np.array(sorted(c for c in cols if 0 <= c < h), dtype=np.int64)
