"""The library's MXFP8 scale order, as the tests and smoke() build it from the
oracle's [N][H][K/N/32] scales, against the layout the header states, written
out element by element: chunks of 512 bytes [N][ceil(H/128)][ceil(K/N/128)],
row t of a 128-row tile and run j of the chunk's four 32-weight runs at byte
16 (t % 32) + 4 (t // 32) + j; rows past H and runs past K/N hold 0."""

import numpy as np
import pytest

from helpers import mx_scales_as_stored


def stored_by_formula(sc):
    n, h, nb = sc.shape
    ht, kg = (h + 127) // 128, (nb + 3) // 4
    out = np.zeros(n * ht * kg * 512, dtype=np.uint8)
    for r in range(n):
        for row in range(h):
            for b in range(nb):
                t = row % 128
                chunk = (r * ht + row // 128) * kg + b // 4
                out[chunk * 512 + 16 * (t % 32) + 4 * (t // 32) + b % 4] = sc[r, row, b]
    return out


@pytest.mark.parametrize("n,h,nb", [(1, 128, 4), (2, 96, 2), (2, 256, 6), (3, 200, 8)])
def test_scale_order_matches_the_stated_layout(n, h, nb):
    rng = np.random.default_rng(n * 1000 + h + nb)
    sc = rng.integers(1, 255, size=(n, h, nb), dtype=np.uint8)   # 0 only in the padding
    got = mx_scales_as_stored(sc)
    assert got.shape == stored_by_formula(sc).shape
    assert np.array_equal(got, stored_by_formula(sc))
    # every scale lands exactly once; the rest is padding
    assert np.count_nonzero(got) == sc.size


def test_smoke_builds_the_same_order():
    """smoke() writes the permutation inline (H a multiple of 128, K/N of 128)."""
    n, h, nb = 2, 256, 16
    rng = np.random.default_rng(3)
    sc = rng.integers(0, 255, size=(n, h, nb), dtype=np.uint8)
    inline = sc.reshape(n, h // 128, 4, 32, nb // 4, 4).transpose(0, 1, 4, 3, 2, 5).reshape(-1)
    assert np.array_equal(inline, stored_by_formula(sc))
