"""Pins of the oracle's ring all-reduce and byte model.

* bytes per rank: the pages' printed worked example (1.25 MiB at N=2,
  about 1.875 MiB at N=4), and the message-by-message counter of the
  simulated ring equal to the closed form 2(N-1)/N x payload for N = 1..8;
* the per-peer and total traffic of a reduce-then-broadcast all-reduce
  (NVL72 hosting post, All-reduce section: (N-1)*B/N read per peer, 2(N-1)*B
  reads and writes in total);
* the fold order: a hand-derived three-rank example (tests/golden);
* integer-valued partials: every order gives the exact integer sum;
* rotating the rank -> shard map: N=2 bit-identical (bf16 addition commutes),
  N>2 equal up to the rounding of the re-associated adds.
"""

import numpy as np
import pytest

import oracle
from helpers import golden_rows


def test_ring_bytes_pages_worked_example():
    rows = golden_rows("ring_bytes.txt")
    assert rows, "golden file is empty"
    for n, m, h, e, pts, want in rows:
        assert oracle.ring_bytes(int(n), int(m), int(h), int(e), int(pts)) == int(want)
    # the printed values, in MiB
    assert oracle.ring_bytes(2, 1, 5120, 2, 128) / 2 ** 20 == 1.25
    assert oracle.ring_bytes(4, 1, 5120, 2, 128) / 2 ** 20 == 1.875


@pytest.mark.parametrize("n", range(1, 9))
def test_ring_counter_equals_closed_form(n):
    hidden, tokens = 840, 3                          # 840 = lcm(1..8)
    rng = np.random.default_rng(n)
    p = rng.integers(0, 0x3F80, size=(n, tokens, hidden), dtype=np.uint16)
    red, sent = oracle.ring(n, hidden, p)
    payload = tokens * hidden * 2
    closed = oracle.ring_bytes(n, tokens, hidden, 2, 1)
    assert all(int(s) == closed for s in sent)
    assert closed == 2 * (n - 1) * payload // n
    # reduce-scatter half: each peer receives (N-1) * B/N; total traffic of
    # the reduce-then-broadcast scheme is 2(N-1)B summed over the N ranks
    assert closed // 2 == (n - 1) * payload // n
    assert sum(int(s) for s in sent) == 2 * (n - 1) * payload


def test_ring_fold_order_golden():
    (row,) = golden_rows("ring_order_n3.txt")
    p0, p1, p2, e0, e1, e2 = (float(v) for v in row)
    vals = np.array([p0, p1, p2], dtype=np.float32)
    bits = oracle.bf16_rne(vals)
    p = np.repeat(bits[:, None, None], 3, axis=2)          # [3 ranks, 1 token, 3 cols]
    red, _ = oracle.ring(3, 3, p)
    out = oracle.residual(np.zeros((1, 3), np.uint16), red)
    assert list(oracle.f32(out[0])) == [e0, e1, e2]


def test_ring_integer_partials_exact_any_n():
    rng = np.random.default_rng(0)
    for n in range(1, 9):
        h = 8 * n
        ints = rng.integers(-30, 31, size=(n, 2, h))
        p = oracle.bf16_rne(ints.astype(np.float32))
        red, _ = oracle.ring(n, h, p)
        assert np.array_equal(oracle.f32(red), ints.sum(axis=0).astype(np.float32))


def _rotate(p, t):
    n = p.shape[0]
    return np.stack([p[(r + t) % n] for r in range(n)])


def test_ring_rotation_n2_bit_identical():
    rng = np.random.default_rng(1)
    p = oracle.bf16_rne(rng.standard_normal((2, 4, 64)).astype(np.float32))
    red0, _ = oracle.ring(2, 64, p)
    red1, _ = oracle.ring(2, 64, _rotate(p, 1))
    assert np.array_equal(red0, red1)


@pytest.mark.parametrize("n", [3, 4, 8])
def test_ring_rotation_equal_up_to_association(n):
    rng = np.random.default_rng(n)
    h = 16 * n
    pf = rng.standard_normal((n, 3, h)).astype(np.float32)
    p = oracle.bf16_rne(pf)
    exact = oracle.f32(p).astype(np.float64).sum(axis=0)
    absum = np.abs(oracle.f32(p).astype(np.float64)).sum(axis=0)
    u = 2.0 ** -8
    # each of the N-1 adds rounds once, to within u of its result, and every
    # intermediate is at most the sum of absolute values (times (1+u)^N)
    bound = (n - 1) * u * absum * (1 + u) ** n
    for t in range(n):
        red, _ = oracle.ring(n, h, _rotate(p, t))
        err = np.abs(oracle.f32(red).astype(np.float64) - exact)
        assert np.all(err <= bound)
    # and the rotations do differ somewhere for N > 2 (the order matters)
    outs = {oracle.ring(n, h, _rotate(p, t))[0].tobytes() for t in range(n)}
    assert len(outs) > 1


def test_ring_n1_is_identity_and_sends_nothing():
    rng = np.random.default_rng(2)
    p = rng.integers(0, 0x7F00, size=(1, 3, 10), dtype=np.uint16)
    red, sent = oracle.ring(1, 10, p)
    assert np.array_equal(red, p[0])
    assert int(sent[0]) == 0


def test_ring_column_subset_matches_full():
    rng = np.random.default_rng(4)
    n, h = 4, 64
    p = oracle.bf16_rne(rng.standard_normal((n, 2, h)).astype(np.float32))
    full, _ = oracle.ring(n, h, p)
    cols = np.array([0, 5, 16, 17, 40, 63])
    sub, _ = oracle.ring(n, h, np.ascontiguousarray(p[:, :, cols]), cols=cols)
    assert np.array_equal(sub, full[:, cols])


def test_ring_rejects_bad_args():
    with pytest.raises(oracle.OracleError):
        oracle.ring(3, 10, np.zeros((3, 1, 10), np.uint16))   # H % N != 0
