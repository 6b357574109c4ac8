"""The seeded input generator: Philox4x32-10 known answers, the Gaussian
quantile table, and random access (any element range draws the same bits)."""

import numpy as np
import torch

from helpers import golden_rows
from workloads import (CONFIGS, KIND_RESIDUAL, KIND_W, KIND_X, gaussian_bf16, gaussian_table,
                       get_config, philox4x32_10, point_tensor, point_tensor_rows)


def test_philox_known_answers():
    rows = golden_rows("philox4x32_10_kat.txt")
    assert len(rows) == 3
    for row in rows:
        v = [int(s, 16) for s in row]
        out = philox4x32_10(v[0], v[1], v[2], v[3], v[4], v[5])
        assert [int(o) for o in out] == v[6:10]


def test_gaussian_table_shape():
    for sigma in (1.0, 0.02):
        t = gaussian_table(sigma).double()
        assert t.numel() == 65536
        assert torch.all(t[1:] >= t[:-1])                       # monotone
        assert torch.equal(t, -t.flip(0))                       # symmetric
        assert abs(t.std().item() / sigma - 1) < 2e-3
        assert 4.2 < t.max().item() / sigma < 4.4


def test_random_access_matches_whole():
    whole = gaussian_bf16(3, 9, 0, 5000, 1.0)
    for start, count in [(0, 7), (1, 16), (13, 100), (4093, 907)]:
        assert torch.equal(gaussian_bf16(3, 9, start, count, 1.0), whole[start:start + count])
    # chunked generation equals one-shot generation
    assert torch.equal(gaussian_bf16(3, 9, 0, 5000, 1.0, chunk=999), whole)


def test_point_rows_match_whole_tensor():
    cfg = get_config("tiny")
    pt = cfg.points[2]
    w = point_tensor(cfg, pt, KIND_W)
    rows = [0, 5, 255]
    assert torch.equal(point_tensor_rows(cfg, pt, KIND_W, rows), w[rows])


def test_substreams_differ_and_moments():
    cfg = get_config("tiny")
    pt = cfg.points[0]
    x = point_tensor(cfg, pt, KIND_X).double()
    w = point_tensor(cfg, pt, KIND_W).double()
    r = point_tensor(cfg, pt, KIND_RESIDUAL).double()
    assert x.shape == (1, 1024) and w.shape == (256, 1024) and r.shape == (1, 256)
    assert abs(w.std().item() / 0.02 - 1) < 0.02
    assert abs(w.mean().item()) < 1e-3
    assert not torch.equal(point_tensor(cfg, cfg.points[1], KIND_X), point_tensor(cfg, pt, KIND_X))


def test_config_shapes_divide():
    for cfg in CONFIGS.values():
        assert cfg.hidden % cfg.n_ranks == 0
        for p in cfg.points:
            assert p.k % cfg.n_ranks == 0 and (p.k // cfg.n_ranks) % 8 == 0
        assert (cfg.hidden // cfg.n_ranks) % 8 == 0
    assert get_config("decode_n2").n_points == 128
    assert get_config("decode_n8_m64").n_points == 96
