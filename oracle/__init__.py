"""ORACLE for the tensor-parallel reconciliation point -- TEST INFRASTRUCTURE.

A thin ctypes wrapper around ``oracle.c`` (plain C, built with gcc by
``oracle/build.py``). Only the test suite, the package smoke check and the
benchmark's CPU-baseline leg import this module. It imports nothing from the
CUDA package and the CUDA package imports nothing from it.

Arrays are numpy ``uint16`` bf16 bit patterns (the top half of an IEEE
float32), C-contiguous.

Functions and the passages they follow:

* ``partials``  -- each rank's partial x_r . W_r over its K/N slice
  ("Interconnects e clusters", 01 Conceito: each weight matrix is split between
  ranks and each rank computes a partial result over its slice; bf16 on the
  wire). fp32 accumulation by fused multiply-add, k ascending, one rounding
  to bf16 (reading of an unstated step).
* ``ring``      -- ring all-reduce simulated message by message: reduce-scatter
  of H/N chunks then all-gather ("Interconnects e clusters", 01 Conceito: a ring
  all-reduce puts 2(N-1)/N times the payload on each rank's wire; NVL72 hosting
  post, All-reduce section: each peer reduces one slice of the input, then
  broadcasts it to the rest).
* ``residual``  -- the residual add after reconciliation (01 Conceito: the
  slices are summed before the residual stream continues).
* ``ring_bytes`` -- 2(N-1)/N x payload per rank (01 Conceito, worked example).
* ``allreduce_bytes`` -- per-rank bytes of the ring, naive and switch-reduction
  all-reduce schemes (NVL72 hosting post, All-reduce section).
* ``moe_combine_bytes`` -- per-rank bytes of an MoE combine: local weighted
  accumulation, then one all-reduce (NVL72 hosting post, MoE dispatch/combine).
* ``mx_quantize`` / ``mx_dequant_bf16`` -- MXFP8 shards (OCP MX E4M3, E8M0 per
  32 weights of a rank slice) for the NVL72 hosting post's MXFP8 weights.
* ``nvfp4_quantize`` / ``nvfp4_dequant_bf16`` -- NVFP4 shards (E2M1, E4M3 per 16
  weights, power-of-two second-level scale) for the TP=4-vs-TP=8 post's NVFP4
  weights.

Pins that tie each function to the pages or to mathematics (not to itself)
live in ``tests/test_oracle_*.py``. Parity unpinned: the exact fp32 rounding of
a Gaussian partial whose fp64 value lies next to a bf16 rounding boundary
(only its neighbourhood is pinned, by the rounding-error bound of recursive
summation).
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import numpy as np

from . import build as _build

_lib = None
_U16P = ctypes.POINTER(ctypes.c_uint16)
_F64P = ctypes.POINTER(ctypes.c_double)
_F32P = ctypes.POINTER(ctypes.c_float)
_I64P = ctypes.POINTER(ctypes.c_int64)
_U64P = ctypes.POINTER(ctypes.c_uint64)
_U8P = ctypes.POINTER(ctypes.c_uint8)

ORC_OK, ORC_ERR_ARGS, ORC_ERR_ALLOC, ORC_ERR_RING = 0, 1, 2, 3


class OracleError(RuntimeError):
    pass


def lib():
    """Load (building first if needed) the oracle's shared library."""
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        L.orc_bf16_rne.argtypes = [ctypes.c_float]
        L.orc_bf16_rne.restype = ctypes.c_uint16
        L.orc_bf16_rne_f64.argtypes = [ctypes.c_double]
        L.orc_bf16_rne_f64.restype = ctypes.c_uint16
        L.orc_f32.argtypes = [ctypes.c_uint16]
        L.orc_f32.restype = ctypes.c_float
        L.orc_bf16_rne_array.argtypes = [ctypes.c_int64, _F32P, _U16P]
        L.orc_bf16_rne_array.restype = None
        L.orc_bf16_rne_f64_array.argtypes = [ctypes.c_int64, _F64P, _U16P]
        L.orc_bf16_rne_f64_array.restype = None
        L.orc_partials.argtypes = [ctypes.c_int, ctypes.c_int64, ctypes.c_int64, _U16P,
                                   ctypes.c_int64, _U16P, _U16P, _F64P, _F64P, ctypes.c_int]
        L.orc_partials.restype = ctypes.c_int
        L.orc_ring.argtypes = [ctypes.c_int, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                               _I64P, _U16P, _U16P, _U64P]
        L.orc_ring.restype = ctypes.c_int
        L.orc_residual.argtypes = [ctypes.c_int64, _U16P, _U16P, _U16P]
        L.orc_residual.restype = None
        L.orc_reconcile.argtypes = [ctypes.c_int, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                    _U16P, ctypes.c_int64, _I64P, _U16P, _U16P, _U16P, _U16P,
                                    _F64P, _F64P, _U64P, ctypes.c_int]
        L.orc_reconcile.restype = ctypes.c_int
        L.orc_ring_bytes.argtypes = [ctypes.c_int, ctypes.c_int64, ctypes.c_int64, ctypes.c_int,
                                     ctypes.c_int64]
        L.orc_ring_bytes.restype = ctypes.c_uint64
        L.orc_allreduce_bytes.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int64, ctypes.c_int64,
                                          ctypes.c_int, ctypes.c_int64]
        L.orc_allreduce_bytes.restype = ctypes.c_uint64
        L.orc_moe_combine_bytes.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int64,
                                            ctypes.c_int64, ctypes.c_int, ctypes.c_int64,
                                            ctypes.c_int]
        L.orc_moe_combine_bytes.restype = ctypes.c_uint64
        L.orc_e2m1_rne.argtypes = [ctypes.c_double]
        L.orc_e2m1_rne.restype = ctypes.c_uint8
        L.orc_e2m1_value.argtypes = [ctypes.c_uint8]
        L.orc_e2m1_value.restype = ctypes.c_double
        L.orc_nvfp4_global_exp.argtypes = [ctypes.c_double]
        L.orc_nvfp4_global_exp.restype = ctypes.c_int
        L.orc_nvfp4_quantize.argtypes = [ctypes.c_int, ctypes.c_int64, ctypes.c_int64, _U16P, _U8P, _U8P,
                                         ctypes.POINTER(ctypes.c_int)]
        L.orc_nvfp4_quantize.restype = ctypes.c_int
        L.orc_nvfp4_dequant_bf16.argtypes = [ctypes.c_int, ctypes.c_int64, ctypes.c_int64, _U8P, _U8P,
                                             ctypes.c_int, _U16P]
        L.orc_nvfp4_dequant_bf16.restype = ctypes.c_int
        L.orc_e4m3_rne.argtypes = [ctypes.c_double]
        L.orc_e4m3_rne.restype = ctypes.c_uint8
        L.orc_e4m3_value.argtypes = [ctypes.c_uint8]
        L.orc_e4m3_value.restype = ctypes.c_double
        L.orc_mx_quantize.argtypes = [ctypes.c_int, ctypes.c_int64, ctypes.c_int64, _U16P, _U8P, _U8P]
        L.orc_mx_quantize.restype = ctypes.c_int
        L.orc_mx_dequant_bf16.argtypes = [ctypes.c_int, ctypes.c_int64, ctypes.c_int64, _U8P, _U8P,
                                          _U16P]
        L.orc_mx_dequant_bf16.restype = ctypes.c_int
        _lib = L
    return _lib


def _ptr(a: Optional[np.ndarray], typ):
    if a is None:
        return ctypes.cast(None, typ)
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(typ)


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError(f"expected uint16 bf16 bit patterns, got {a.dtype}")
    return a


# ----------------------------------------------------------------- bf16 --

def f32(b) -> np.ndarray:
    """bf16 bit patterns -> float32 values (exact)."""
    b = np.asarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def bf16_rne(f) -> np.ndarray:
    """float32 values -> bf16 bit patterns, round to nearest even."""
    f = np.ascontiguousarray(np.asarray(f, dtype=np.float32))
    out = np.empty(f.shape, dtype=np.uint16)
    lib().orc_bf16_rne_array(f.size, _ptr(f, _F32P), _ptr(out, _U16P))
    return out


def bf16_rne_f64(d) -> np.ndarray:
    """float64 values -> bf16 bit patterns, correctly rounded from the double."""
    d = np.ascontiguousarray(np.asarray(d, dtype=np.float64))
    out = np.empty(d.shape, dtype=np.uint16)
    lib().orc_bf16_rne_f64_array(d.size, _ptr(d, _F64P), _ptr(out, _U16P))
    return out


# -------------------------------------------------------------- partials --

def partials(n_ranks: int, x: np.ndarray, w_rows: np.ndarray, threads: int = 1):
    """Partials [N, M, R] of rows w_rows [R, K] against x [M, K].

    Returns (p, p64, pabs): bf16 partials, the fp64 sums of the same products
    and the fp64 sums of their absolute values.
    """
    x = _u16(x)
    w_rows = _u16(w_rows)
    m, k = x.shape
    r, k2 = w_rows.shape
    if k2 != k:
        raise ValueError("x and w_rows disagree on K")
    p = np.empty((n_ranks, m, r), dtype=np.uint16)
    p64 = np.empty((n_ranks, m, r), dtype=np.float64)
    pabs = np.empty((n_ranks, m, r), dtype=np.float64)
    rc = lib().orc_partials(n_ranks, m, k, _ptr(x, _U16P), r, _ptr(w_rows, _U16P),
                            _ptr(p, _U16P), _ptr(p64, _F64P), _ptr(pabs, _F64P), threads)
    if rc != ORC_OK:
        raise OracleError(f"orc_partials failed with {rc}")
    return p, p64, pabs


# ------------------------------------------------------------------ ring --

def ring(n_ranks: int, hidden: int, p: np.ndarray, cols: Optional[Sequence[int]] = None):
    """Ring all-reduce of partials p [N, M, C] on columns cols (default all H).

    Returns (reduced [M, C], bytes_sent [N]).
    """
    p = _u16(p)
    n, m, c = p.shape
    if n != n_ranks:
        raise ValueError("p's first dimension must be N")
    if cols is None:
        cols = np.arange(c, dtype=np.int64)
        if c != hidden:
            raise ValueError("cols must be given when p does not hold all H columns")
    cols = np.ascontiguousarray(np.asarray(cols, dtype=np.int64))
    red = np.empty((m, c), dtype=np.uint16)
    sent = np.zeros(n_ranks, dtype=np.uint64)
    rc = lib().orc_ring(n_ranks, m, hidden, c, _ptr(cols, _I64P), _ptr(p, _U16P),
                        _ptr(red, _U16P), _ptr(sent, _U64P))
    if rc != ORC_OK:
        raise OracleError(f"orc_ring failed with {rc}")
    return red, sent


def residual(res: np.ndarray, reduced: np.ndarray) -> np.ndarray:
    res = _u16(res)
    reduced = _u16(reduced)
    if res.shape != reduced.shape:
        raise ValueError("shape mismatch")
    out = np.empty(res.shape, dtype=np.uint16)
    lib().orc_residual(res.size, _ptr(res, _U16P), _ptr(reduced, _U16P), _ptr(out, _U16P))
    return out


# ---------------------------------------------------------- whole point --

def reconcile(n_ranks: int, hidden: int, x: np.ndarray, w_rows: np.ndarray,
              res_cols: np.ndarray, cols: Optional[Sequence[int]] = None, threads: int = 1):
    """One reconciliation point on output columns cols.

    x [M, K]; w_rows [C, K] = rows cols of W [H, K]; res_cols [M, C].
    Returns a dict with out [M, C], partials [N, M, C], p64, pabs, bytes_sent [N].
    """
    x = _u16(x)
    w_rows = _u16(w_rows)
    res_cols = _u16(res_cols)
    m, k = x.shape
    c = w_rows.shape[0]
    if cols is None:
        if c != hidden:
            raise ValueError("cols must be given when w_rows does not hold all H rows")
        cols = np.arange(c, dtype=np.int64)
    cols = np.ascontiguousarray(np.asarray(cols, dtype=np.int64))
    if res_cols.shape != (m, c) or cols.shape != (c,):
        raise ValueError("shape mismatch")
    out = np.empty((m, c), dtype=np.uint16)
    p = np.empty((n_ranks, m, c), dtype=np.uint16)
    p64 = np.empty((n_ranks, m, c), dtype=np.float64)
    pabs = np.empty((n_ranks, m, c), dtype=np.float64)
    sent = np.zeros(n_ranks, dtype=np.uint64)
    rc = lib().orc_reconcile(n_ranks, m, k, hidden, _ptr(x, _U16P), c, _ptr(cols, _I64P),
                             _ptr(w_rows, _U16P), _ptr(res_cols, _U16P), _ptr(out, _U16P),
                             _ptr(p, _U16P), _ptr(p64, _F64P), _ptr(pabs, _F64P),
                             _ptr(sent, _U64P), threads)
    if rc != ORC_OK:
        raise OracleError(f"orc_reconcile failed with {rc}")
    return {"out": out, "partials": p, "p64": p64, "pabs": pabs, "bytes_sent": sent}


def ring_bytes(n_ranks: int, tokens: int, hidden: int, elem_bytes: int, points: int) -> int:
    return int(lib().orc_ring_bytes(n_ranks, tokens, hidden, elem_bytes, points))


def e4m3_rne(v: float) -> int:
    """E4M3 code of the exact value v, nearest even, saturating at 448."""
    return int(lib().orc_e4m3_rne(float(v)))


def e4m3_value(code: int) -> float:
    return float(lib().orc_e4m3_value(int(code)))


def mx_quantize(n_ranks: int, w_hk: np.ndarray):
    """Linear weight [H, K] bf16 -> (q [N, H, K/N] uint8 E4M3 codes,
    scales [N, H, K/N/32] uint8 E8M0 bytes)."""
    w = _u16(w_hk)
    h, k = w.shape
    ks = k // n_ranks
    q = np.empty((n_ranks, h, ks), dtype=np.uint8)
    sc = np.empty((n_ranks, h, ks // 32), dtype=np.uint8)
    rc = lib().orc_mx_quantize(n_ranks, h, k, _ptr(w, _U16P), _ptr(q, _U8P), _ptr(sc, _U8P))
    if rc != ORC_OK:
        raise OracleError(f"orc_mx_quantize failed with {rc}")
    return q, sc


def mx_dequant_bf16(n_ranks: int, q: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """MXFP8 shards -> the dequantised Linear weight [H, K] as bf16 bit patterns."""
    q = np.ascontiguousarray(q, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    n, h, ks = q.shape
    w = np.empty((h, n * ks), dtype=np.uint16)
    rc = lib().orc_mx_dequant_bf16(n_ranks, h, n * ks, _ptr(q, _U8P), _ptr(scales, _U8P),
                                   _ptr(w, _U16P))
    if rc != ORC_OK:
        raise OracleError(f"orc_mx_dequant_bf16 failed with {rc}")
    return w


ALLREDUCE_SCHEMES = {"ring": 0, "naive": 1, "sharp": 2}


def allreduce_bytes(scheme: str, n_ranks: int, tokens: int, hidden: int, elem_bytes: int,
                    points: int) -> int:
    """Per-rank NVLink bytes of one all-reduce scheme (see orc_allreduce_bytes)."""
    return int(lib().orc_allreduce_bytes(ALLREDUCE_SCHEMES[scheme], n_ranks, tokens, hidden,
                                         elem_bytes, points))


def moe_combine_bytes(scheme: str, n_ranks: int, tokens: int, hidden: int, elem_bytes: int,
                      top_k: int, local_accumulate: bool = True) -> int:
    """Per-rank NVLink bytes of an MoE combine: the weighted contributions of
    each rank's experts accumulated locally, then one all-reduce of the
    [tokens][hidden] buffer (NVL72 hosting post, MoE dispatch/combine);
    local_accumulate=False all-reduces each of the top_k expert slots apart."""
    return int(lib().orc_moe_combine_bytes(ALLREDUCE_SCHEMES[scheme], n_ranks, tokens, hidden,
                                           elem_bytes, top_k, int(bool(local_accumulate))))


def e2m1_rne(v: float) -> int:
    """E2M1 code (sign in bit 3) of the exact value v, nearest even, saturating at 6."""
    return int(lib().orc_e2m1_rne(float(v)))


def e2m1_value(code: int) -> float:
    return float(lib().orc_e2m1_value(int(code)))


def nvfp4_global_exp(amax: float) -> int:
    return int(lib().orc_nvfp4_global_exp(float(amax)))


def nvfp4_quantize(n_ranks: int, w_hk: np.ndarray):
    """Linear weight [H, K] bf16 -> (q [N, H, K/N/2] uint8, two E2M1 codes per
    byte (earlier k in the low nibble); scales [N, H, K/N/16] E4M3; g, the
    second-level exponent)."""
    w_hk = _u16(w_hk)
    h, k = w_hk.shape
    ks = k // n_ranks
    q = np.zeros((n_ranks, h, ks // 2), dtype=np.uint8)
    sc = np.zeros((n_ranks, h, ks // 16), dtype=np.uint8)
    g = ctypes.c_int(0)
    rc = lib().orc_nvfp4_quantize(n_ranks, h, k, _ptr(w_hk, _U16P), _ptr(q, _U8P), _ptr(sc, _U8P),
                                  ctypes.byref(g))
    if rc != ORC_OK:
        raise OracleError(f"orc_nvfp4_quantize failed with {rc}")
    return q, sc, g.value


def nvfp4_dequant_bf16(n_ranks: int, q: np.ndarray, scales: np.ndarray, g: int) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    n, h, half = q.shape
    k = 2 * half * n
    w = np.empty((h, k), dtype=np.uint16)
    rc = lib().orc_nvfp4_dequant_bf16(n_ranks, h, k, _ptr(q, _U8P), _ptr(scales, _U8P), int(g),
                                      _ptr(w, _U16P))
    if rc != ORC_OK:
        raise OracleError(f"orc_nvfp4_dequant_bf16 failed with {rc}")
    return w


def cores() -> int:
    return len(os.sched_getaffinity(0))
