"""Every workload at its full size, in the launch configuration bench.py times
(all points of the step captured in one CUDA graph with programmatic
dependent launch), checked against the oracle on sampled output columns (all
tokens of each sampled column): bit-exact for the exact variant."""

import gc

import numpy as np
import pytest
import torch

import oracle
from gpu_util import sample_cols
from helpers import u16
from workloads import KIND_RESIDUAL, KIND_W, KIND_X, get_config, point_tensor, point_tensor_rows

pytestmark = pytest.mark.gpu


def _check_points(wl, cfg, idx, cols):
    for i in idx:
        p = cfg.points[i]
        x = u16(point_tensor(cfg, p, KIND_X))
        w = u16(point_tensor_rows(cfg, p, KIND_W, cols))
        r = u16(point_tensor(cfg, p, KIND_RESIDUAL))[:, cols]
        ref = oracle.reconcile(cfg.n_ranks, cfg.hidden, x, w, np.ascontiguousarray(r),
                               cols=cols, threads=oracle.cores())
        got = u16(wl.out(i))[:, cols]
        assert np.array_equal(got, ref["out"]), (cfg.name, i, int(np.sum(got != ref["out"])))


@pytest.mark.parametrize("name", ["tiny", "decode_n2", "decode_n4_m32", "decode_n8_m64",
                                  "prefill_n4"])
def test_config_graph_step_exact(name):
    import bench
    cfg = get_config(name)
    dev = torch.device("cuda", 0)
    wl = bench.Workload(cfg, dev, variant="exact", staged=False)
    g = wl.capture()
    wl.out_all.fill_(0)
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    assert next(iter(wl.plans.values())).device_error_flags() == 0
    kinds = {}
    for p in cfg.points:
        kinds.setdefault(p.kind, []).append(p.index)
    idx = sorted({v for lst in kinds.values() for v in (lst[0], lst[-1])})
    ncols = 24 if cfg.tokens >= 1024 else 48
    cols = np.arange(cfg.hidden) if cfg.hidden <= 256 else sample_cols(cfg.hidden, cfg.n_ranks,
                                                                       ncols, seed=len(name))
    _check_points(wl, cfg, idx, cols)
    del g, wl
    gc.collect()
    torch.cuda.empty_cache()


@pytest.mark.parametrize("name", ["tiny", "decode_n2", "decode_n4_m32", "decode_n8_m64",
                                  "prefill_n4"])
def test_config_graph_step_tensor(name):
    """The default (AUTO) variant runs the tensor cores; outputs
    follow the fragile-partial rule of test_gpu_tensor on sampled columns."""
    import bench
    from test_gpu_tensor import bf16_ulp, fragile_mask
    cfg = get_config(name)
    dev = torch.device("cuda", 0)
    wl = bench.Workload(cfg, dev, variant="auto", staged=False)
    g = wl.capture()
    wl.out_all.fill_(0)
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    assert next(iter(wl.plans.values())).device_error_flags() == 0
    kinds = {}
    for p in cfg.points:
        kinds.setdefault(p.kind, []).append(p.index)
    idx = sorted({v for lst in kinds.values() for v in (lst[0], lst[-1])})
    cols = np.arange(cfg.hidden) if cfg.hidden <= 256 else \
        sample_cols(cfg.hidden, cfg.n_ranks, 16 if cfg.tokens >= 1024 else 40, seed=len(name))
    n = cfg.n_ranks
    for i in idx:
        p = cfg.points[i]
        x = u16(point_tensor(cfg, p, KIND_X))
        w = u16(point_tensor_rows(cfg, p, KIND_W, cols))
        r = np.ascontiguousarray(u16(point_tensor(cfg, p, KIND_RESIDUAL))[:, cols])
        ref = oracle.reconcile(n, cfg.hidden, x, w, r, cols=cols, threads=oracle.cores())
        got = u16(wl.out(i))[:, cols]
        frag = fragile_mask(ref["p64"], ref["pabs"])
        out_frag = frag.any(axis=0)
        assert np.array_equal(got[~out_frag], ref["out"][~out_frag]), (name, i)
        go = oracle.f32(got).astype(np.float64)
        ro = oracle.f32(ref["out"]).astype(np.float64)
        pf = np.abs(oracle.f32(ref["partials"]).astype(np.float64))
        res = np.abs(oracle.f32(r).astype(np.float64))
        bound = (2 * bf16_ulp(pf) * frag).sum(axis=0) + (n - 1) * bf16_ulp(pf.sum(axis=0)) \
            + bf16_ulp(res + pf.sum(axis=0))
        assert np.all(np.abs(go - ro)[out_frag] <= bound[out_frag]), (name, i)
        diff = np.abs(go - ro)
        assert np.linalg.norm(go - ro) / np.linalg.norm(ro) <= 5e-3
        assert np.all(diff[~out_frag] <= 2e-2)
        print(f"{name} point {i}: fragile outputs {int(out_frag.sum())} of {out_frag.size}, "
              f"max abs {diff.max():.4g}")
    del g, wl
    gc.collect()
    torch.cuda.empty_cache()
