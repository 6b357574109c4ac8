"""Pins of the oracle's all-reduce byte model for three schemes (ring, naive,
switch reduction), against what the pages fix:

* the first page's ring bytes per rank for its worked example (golden file);
* the NVL72 hosting post's All-reduce section: the naive scheme reads
  N(N-1)B in total; reducing slices and broadcasting them moves (N-1)B/N per
  peer each way, 2(N-1)B in total; the switch reduction moves the fraction
  N/(2(N-1)) of the ring's transfers (a 33% saving at four peers);
* one rank communicates nothing;
* the MoE combine (same post, dispatch/combine section) accumulates each
  rank's expert contributions locally and then all-reduces one buffer, so its
  cost is one all-reduce whatever top_k is (golden file, invariants).
"""

from fractions import Fraction

import pytest

import oracle
from helpers import golden_rows


def test_allreduce_bytes_golden():
    rows = golden_rows("allreduce_bytes.txt")
    assert len(rows) == 5
    for scheme, n, m, h, e, pts, want in rows:
        assert oracle.allreduce_bytes(scheme, int(n), int(m), int(h), int(e), int(pts)) == int(want)


@pytest.mark.parametrize("n", range(2, 9))
def test_allreduce_closed_forms(n):
    tokens, hidden, elem, points = 3, 840, 2, 5          # 840 = lcm(1..8): whole slices
    b = tokens * hidden * elem * points
    ring = oracle.allreduce_bytes("ring", n, tokens, hidden, elem, points)
    naive = oracle.allreduce_bytes("naive", n, tokens, hidden, elem, points)
    sharp = oracle.allreduce_bytes("sharp", n, tokens, hidden, elem, points)
    assert ring == oracle.ring_bytes(n, tokens, hidden, elem, points)   # the first page's model
    assert n * ring == 2 * (n - 1) * b                  # 2(N-1)B reads and writes in total
    assert n * naive == n * (n - 1) * b                 # N(N-1)B reads in total
    assert Fraction(sharp, ring) == Fraction(n, 2 * (n - 1))
    if n == 4:
        assert 1 - Fraction(sharp, ring) == Fraction(1, 3)   # "33% with four peers"


def test_allreduce_single_rank_and_bad_args():
    for s in ("ring", "naive", "sharp"):
        assert oracle.allreduce_bytes(s, 1, 4, 5120, 2, 128) == 0
        assert oracle.allreduce_bytes(s, 0, 4, 5120, 2, 128) == 0
        assert oracle.allreduce_bytes(s, 4, -1, 5120, 2, 128) == 0
    assert int(oracle.lib().orc_allreduce_bytes(7, 4, 1, 5120, 2, 128)) == 0


def test_moe_combine_bytes_golden():
    rows = golden_rows("moe_combine_bytes.txt")
    assert len(rows) == 4
    for scheme, n, m, h, e, k, local, want in rows:
        got = oracle.moe_combine_bytes(scheme, int(n), int(m), int(h), int(e), int(k), local == "1")
        assert got == int(want), (scheme, n, m, h, e, k, local)


@pytest.mark.parametrize("scheme", ["ring", "naive", "sharp"])
def test_moe_combine_invariants(scheme):
    for n in range(1, 9):
        one = oracle.allreduce_bytes(scheme, n, 7, 840, 2, 1)
        for top_k in (1, 2, 8):
            # local accumulation: one all-reduce of the [tokens][hidden] buffer
            assert oracle.moe_combine_bytes(scheme, n, 7, 840, 2, top_k, True) == one
            # slots reduced apart: top_k all-reduces
            assert oracle.moe_combine_bytes(scheme, n, 7, 840, 2, top_k, False) == top_k * one
    assert oracle.moe_combine_bytes(scheme, 4, 7, 840, 2, 0, True) == 0
    assert int(oracle.lib().orc_moe_combine_bytes(0, 4, 7, 840, 2, 2, 2)) == 0
