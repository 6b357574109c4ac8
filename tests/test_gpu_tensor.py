"""Parity of the tensor-core variant (tcgen05, fp32 accumulation in TMEM)
against the oracle.

The tensor cores accumulate in their own order, so a partial can differ from
the oracle's k-ascending fp32 sum where that sum lies next to a bf16 rounding
boundary. The checks:

* integer-valued x, W in {-1, 0, 1}: every sum is an exactly representable
  integer, so partials and outputs must be bit-identical to the oracle (this
  pins the operand layouts, descriptors and tile indexing);
* Gaussian inputs: a partial is "fragile" when the bf16 rounding of its fp64
  value d is not the same at d - e and d + e, with e = 2^-19 * sum|x*w|, far
  above any fp32 accumulation error at these sizes (about 2^-24 * sqrt(K/N)
  relative). Every non-fragile partial must equal bf16(d) and the oracle's
  partial; a fragile one must be one of the two bf16 values around d. An
  output whose N partials are all non-fragile must equal the oracle's bit
  for bit; for the rest, a flipped partial moves its addend by one bf16
  unit of that partial, and each of the N-1 ring adds and the residual add
  may then round the other way, so
      |out - out_oracle| <= sum over fragile r of 2 ulp(P_r)
                            + (N-1) ulp(sum_r |P_r|) + ulp(|res| + sum_r |P_r|);
* the acceptance tolerance: relative L2 error <= 5e-3 over the whole
  output, and max abs error <= 2e-2 over every output with no fragile
  partial (there it is 0: bit-exact). On a fragile output the bound above
  applies instead: one unit of a partial of magnitude >= 2 is already
  2^-6 = 0.016, so no accumulation order other than the oracle's own can
  keep such an output within 2e-2 everywhere. The largest error over all
  outputs is reported.
"""

import numpy as np
import pytest
import torch

import oracle
from gpu_util import inputs, oracle_point
from helpers import from_u16, u16

pytestmark = pytest.mark.gpu

SHAPES = [             # N, M, K, H
    (4, 32, 512, 512),      # decode batch, token tile 32
    (8, 64, 1024, 256),     # decode batch, token tile 64, N = 8
    (2, 16, 128, 128),      # 16 tokens in a 32-token tile
    (2, 1, 8192, 512),      # one token: K split 8 ways across CTAs, folded in the kernel
    (8, 1, 2048, 1024),     # one token, N = 8: K split 4 ways, folded in the kernel
    (2, 2, 4096, 384),      # two tokens (the most folded in the kernel), H % 128 != 0
    (4, 3, 2048, 640),      # three tokens, K split, H % 128 != 0
    (4, 100, 640, 384),     # token tile 128 with a ragged tail; 3 weight tiles
    (4, 300, 512, 256),     # token tile 256, two tiles, second ragged
    (1, 48, 400, 200),      # N = 1; K/N = 400 ends in a partial 64-column block; H % 128 != 0
    (8, 512, 1024, 4096),   # prefill-sized: CTA pairs (2-SM MMA), 16 H-tile pairs, 2 token tiles
    (8, 300, 1024, 4224),   # CTA pairs, odd H-tile count (last pair half out of range), ragged tokens
    (1, 260, 512, 768),     # CTA pairs for the partials, N = 1, ragged second token tile
    (8, 64, 1024, 4096),    # 256 units, no split: bf16 partials and the ring kernel
    (4, 32, 1024, 5120),
    (8, 1, 1024, 4096),     # one token without a k-split: the counter fold over whole partials
    (2, 1, 5120, 5120),     # the decode example's out-projection: 2 ranks x 3 parts, counter fold
]
# The CLUSTER variant: the N ranks (x K parts) of a tile fold on chip in one cluster.
CLUSTER_SHAPES = [
    (8, 64, 1024, 4096),    # clusters of 8, one tile each
    (4, 32, 1024, 5120),    # clusters of 4
    (3, 40, 768, 6504),     # clusters of 3, ragged H tile and tokens
    (2, 100, 512, 10240),   # 128-token tile, one CTA per SM: some clusters fold two tiles
    (8, 64, 512, 8192),     # 64 tiles on 37 clusters: the shared partial tile is reused
    (1, 16, 256, 19200),    # N = 1: a cluster of one CTA
    (8, 1, 1024, 4096),     # one token, no split
    (2, 1, 5120, 5120),     # 2 ranks x 3 K parts: fp32 parts folded on chip
    (4, 1, 4096, 4096),     # 4 ranks x 2 parts
    (2, 3, 2048, 4096),     # 2 ranks x 4 parts, three tokens
    (1, 1, 512, 10240),     # N = 1: 3 parts
    (2, 1, 8192, 512),      # 8 parts: too many for a cluster, staged as TENSOR would
]
CIDS = [f"N{n}M{m}K{k}H{h}" for n, m, k, h in CLUSTER_SHAPES]
IDS = [f"N{n}M{m}K{k}H{h}" for n, m, k, h in SHAPES]


def _run(n, m, k, h, x, w, r, variant="tensor"):
    import tensor_layer_reconciliation_b200 as tlr
    plan = tlr.Plan(n, m, k, h, variant=variant)
    wp = plan.pack_weights(w)
    out = plan.reconcile(x, wp, r)
    parts = plan.partials(x, wp)
    torch.cuda.synchronize()
    assert plan.device_error_flags() == 0
    return u16(out), u16(parts)


@pytest.mark.parametrize("variant,shape", [("tensor", sh) for sh in SHAPES] +
                         [("cluster", sh) for sh in CLUSTER_SHAPES],
                         ids=[f"tensor-{i}" for i in IDS] + [f"cluster-{i}" for i in CIDS])
def test_tensor_integer_exact(variant, shape):
    n, m, k, h = shape
    dev = torch.device("cuda")
    g = torch.Generator().manual_seed(sum(shape))
    xi = torch.randint(-1, 2, (m, k), generator=g)
    wi = torch.randint(-1, 2, (h, k), generator=g)
    ri = torch.randint(-8, 9, (m, h), generator=g)
    out, parts = _run(n, m, k, h, xi.to(dev, torch.bfloat16), wi.to(dev, torch.bfloat16),
                      ri.to(dev, torch.bfloat16), variant)
    ref = oracle_point(n, h, xi.to(torch.bfloat16), wi.to(torch.bfloat16), ri.to(torch.bfloat16))
    assert np.array_equal(parts, ref["partials"])
    assert np.array_equal(out, ref["out"])
    assert torch.equal(from_u16(out).long(), xi @ wi.T + ri)


def bf16_ulp(a):
    """Spacing of bf16 values at magnitude a (subnormal spacing below 2^-126)."""
    a = np.maximum(np.asarray(a, dtype=np.float64), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(a)) - 7)


def fragile_mask(p64, pabs):
    e = pabs * 2.0 ** -19
    lo = oracle.bf16_rne_f64(p64 - e)
    hi = oracle.bf16_rne_f64(p64 + e)
    return lo != hi


def check_against_oracle(out, parts, ref, n, outputs_only=False):
    p64, pabs = ref["p64"], ref["pabs"]
    frag = fragile_mask(p64, pabs)
    exact_p = oracle.bf16_rne_f64(p64)
    # partials: bit-exact where not fragile, a neighbour of d where fragile
    # (outputs_only: the kernel keeps its partials on chip; only the oracle's are checked)
    assert np.array_equal(ref["partials"][~frag], exact_p[~frag])
    if not outputs_only:
        assert np.array_equal(parts[~frag], exact_p[~frag])
    if frag.any() and not outputs_only:
        lo = oracle.bf16_rne_f64(np.nextafter(p64[frag], -np.inf) - pabs[frag] * 2.0 ** -19)
        hi = oracle.bf16_rne_f64(p64[frag] + pabs[frag] * 2.0 ** -19)
        g = oracle.f32(parts[frag])
        assert np.all((g >= oracle.f32(lo)) & (g <= oracle.f32(hi)))
    # outputs
    out_frag = frag.any(axis=0)
    assert np.array_equal(out[~out_frag], ref["out"][~out_frag])
    go, ro = oracle.f32(out).astype(np.float64), oracle.f32(ref["out"]).astype(np.float64)
    pf = np.abs(oracle.f32(ref["partials"]).astype(np.float64))
    res = np.abs(oracle.f32(ref["res"]).astype(np.float64))
    bound = (2 * bf16_ulp(pf) * frag).sum(axis=0) + (n - 1) * bf16_ulp(pf.sum(axis=0)) \
        + bf16_ulp(res + pf.sum(axis=0))
    assert np.all(np.abs(go - ro)[out_frag] <= bound[out_frag])
    # acceptance tolerance
    diff = np.abs(go - ro)
    rel_l2 = np.linalg.norm(go - ro) / max(np.linalg.norm(ro), 1e-30)
    assert rel_l2 <= 5e-3
    assert np.all(diff[~out_frag] <= 2e-2)
    return int(frag.sum()), int(out_frag.sum()), float(diff.max()), float(rel_l2)


@pytest.mark.parametrize("variant,shape", [("tensor", sh) for sh in SHAPES] +
                         [("cluster", sh) for sh in CLUSTER_SHAPES],
                         ids=[f"tensor-{i}" for i in IDS] + [f"cluster-{i}" for i in CIDS])
def test_tensor_gaussian_fragile_rule(variant, shape):
    n, m, k, h = shape
    dev = torch.device("cuda")
    x, w, r = inputs(n, m, k, h, 500 + sum(shape), dev)
    out, parts = _run(n, m, k, h, x, w, r, variant)
    ref = oracle_point(n, h, x.cpu(), w.cpu(), r.cpu())
    ref["res"] = u16(r)
    fp, fo, mx, rl2 = check_against_oracle(out, parts, ref, n)
    print(f"{shape}: fragile partials {fp}, outputs touched {fo}, max abs {mx:.3g}, rel L2 {rl2:.3g}")


def test_auto_uses_tensor_cores():
    import tensor_layer_reconciliation_b200 as tlr
    plan = tlr.Plan(2, 64, 4096, 1024)                 # AUTO
    assert plan.effective_variant(1) == "tensor"
    assert plan.effective_variant(64) == "tensor"
    assert plan.workspace_bytes(1) > 0                 # tensor, 2 ranks x 8 K parts: counter fold
    plan.set_variant("exact")
    assert plan.effective_variant(1) == "exact"
    assert plan.workspace_bytes(1) == 0                # exact, fused: no workspace
    assert tlr.tp_plan_kernel_variant(plan.handle, 0) == -1


def test_fold_counters_return_to_zero():
    """One zeroed workspace serves many calls: the in-kernel fold (one or two
    tokens) hands out tickets per tile in the workspace's first words (the
    folding CTA sets them back to zero) and counts each tile's folds in the
    next ones (the tag its parts carry the next call)."""
    import tensor_layer_reconciliation_b200 as tlr
    dev = torch.device("cuda")
    n, k, h = 4, 4096, 640
    plan = tlr.Plan(n, 2, k, h)                        # AUTO
    for m in (1, 2):
        assert plan.launches(m) == 1                   # partials and fold in one kernel
        need = plan.workspace_bytes(m)
        ws = torch.zeros(need, dtype=torch.uint8, device=dev)
        h_tiles = (h + 127) // 128                     # tickets, then folds done, per tile
        for call, seed in enumerate((31, 32, 33)):
            x, w, r = inputs(n, m, k, h, seed + 10 * m, dev)
            wp = plan.pack_weights(w)
            out = plan.reconcile(x, wp, r, workspace=ws)
            fresh = plan.reconcile(x, wp, r)           # its own zeroed workspace
            torch.cuda.synchronize()
            assert plan.device_error_flags() == 0
            assert torch.equal(out.view(torch.int16), fresh.view(torch.int16))
            words = ws[:8 * h_tiles].view(torch.int32).cpu()
            assert int(torch.count_nonzero(words[:h_tiles])) == 0          # tickets
            assert torch.equal(words[h_tiles:2 * h_tiles], torch.full((h_tiles,), call + 1, dtype=torch.int32))
    assert plan.launches(3) == 2                       # from three tokens: a ring kernel follows


def test_pair_fold_counters_return_to_zero():
    """Prefill-sized calls on CTA pairs fold in their epilogue: one kernel a
    call; the CTA storing a half tile's last rank folds it and sets its count
    back to zero, so one zeroed workspace serves many calls."""
    import tensor_layer_reconciliation_b200 as tlr
    dev = torch.device("cuda")
    n, m, k, h = 8, 300, 1024, 4224
    plan = tlr.Plan(n, m, k, h)                        # AUTO
    assert plan.launches(m) == 1
    need = plan.workspace_bytes(m)
    ws = torch.zeros(need, dtype=torch.uint8, device=dev)
    pair_words = 2 * ((h + 255) // 256) * ((m + 255) // 256)
    counter_bytes = ((2 * ((h + 127) // 128) + pair_words) * 4 + 255) // 256 * 256
    for seed in (41, 42):
        x, w, r = inputs(n, m, k, h, seed, dev)
        wp = plan.pack_weights(w)
        out = plan.reconcile(x, wp, r, workspace=ws)
        fresh = plan.reconcile(x, wp, r)               # its own zeroed workspace
        torch.cuda.synchronize()
        assert plan.device_error_flags() == 0
        assert torch.equal(out.view(torch.int16), fresh.view(torch.int16))
        assert int(torch.count_nonzero(ws[:counter_bytes])) == 0


def test_cluster_fold_needs_no_workspace():
    """The CLUSTER variant: when the N ranks x K parts of a tile make at most 8
    CTAs they fold on chip in one cluster: one kernel per call, nothing
    staged, no workspace."""
    import tensor_layer_reconciliation_b200 as tlr
    for n, m, k, h in [(8, 64, 1024, 4096), (4, 32, 1024, 5120), (8, 1, 1024, 4096),
                       (2, 1, 5120, 5120), (2, 3, 2048, 4096)]:
        plan = tlr.Plan(n, m, k, h, variant="cluster")
        assert plan.launches(m) == 1 and plan.workspace_bytes(m) == 0, (n, m, k, h)
        assert plan.effective_variant(m) == "tensor"
        auto = tlr.Plan(n, m, k, h)                      # AUTO stages its partials
        assert auto.workspace_bytes(m) > 0 and auto.launches(m) == (1 if m <= 2 else 2)
        x, w, r = inputs(n, m, k, h, 5, torch.device("cuda"))
        out = plan.reconcile(x, plan.pack_weights(w), r)
        torch.cuda.synchronize()
        assert out.shape == (m, h) and plan.device_error_flags() == 0
