"""Benchmark of the reconciliation point on B200: one step = every point of a
workload (all partials, ring folds and residual adds) over one batch.

Usage:
  python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME|all]
                  [--variant auto|exact|tensor] [--staged] [--weights bf16|mxfp8]
                  [--impl ours|reference]

With the default --config all, the four benchmarked workloads run one after
another (decode_n2, decode_n4_m32, decode_n8_m64, prefill_n4), each on its
own freshly allocated buffers; the headline numbers are decode_n2's (the
pages' worked decode example) and every workload's numbers are under
"per_config". Prints ONE JSON line on rank 0. With --gpus N > 1 it runs under
torch.distributed.run, one process per GPU; every rank runs an independent
replica of the step (the N tensor-parallel ranks of the method are emulated
inside each GPU), so there is no data-path collective and the scaling is weak.
"""

from __future__ import annotations

import argparse
import dataclasses
import datetime
import gc
import json
import os
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from workloads import (KIND_RESIDUAL, KIND_W, KIND_X, get_config, point_tensor,  # noqa: E402
                       point_tensor_rows)
from workloads.configs import CONFIG_ORDER  # noqa: E402

METRIC = "reconciliations/s & tokens/s on 1 B200; achieved HBM GB/s (TC util) vs peak"
HEADLINE_CONFIG = "decode_n2"
BENCH_CONFIGS = ["decode_n2", "decode_n4_m32", "decode_n8_m64", "prefill_n4"]
TOL_MAX_ABS, TOL_REL_L2 = 2e-2, 5e-3      # acceptance tolerance against the oracle


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


# DRAM bytes (read + write) per reconciliation call, averaged over the points
# of a workload, from ncu captures of the kernels as they are built from the
# sources whose digest is recorded; a digest that no longer matches the
# sources means the kernels changed since, and the traffic is reported null.
PROFILED_TRAFFIC = {
    # (workload, path): (bytes per call, kernel-source digest, the ncu capture)
    ("decode_n2", "tensor"): (116298944, "6deafc10c0aa3bd1",
        "ncu dram__bytes of tc_partial_kernel<32> (counter fold) on decode_n2, one call per point kind"),
    ("decode_n4_m32", "tensor"): (119870080, "0a546cf619614267",
        "ncu dram__bytes of tc_partial_kernel<32> + ring_reduce_kernel on decode_n4_m32, one call per point kind"),
    ("decode_n8_m64", "tensor"): (81532160, "6deafc10c0aa3bd1",
        "ncu dram__bytes of tc_partial_kernel<64> + ring_reduce_kernel on decode_n8_m64, one call per point kind"),
    ("prefill_n4", "tensor"): (886932608, "6deafc10c0aa3bd1",
        "ncu dram__bytes of tc2_partial_kernel (fold in the epilogue) on prefill_n4, one call per point kind"),
    ("decode_n2", "exact-fused"): (117532032, "0a546cf619614267",
        "ncu dram__bytes of exact_partial_kernel<1> on decode_n2, one call per point kind"),
    ("decode_n2", "mxfp8"): (60123584, "6deafc10c0aa3bd1",
        "ncu dram__bytes of tc_partial_kernel<32> block-scaled MXFP8 form on decode_n2, one call per point kind"),
    ("decode_n2", "nvfp4"): (32578176, "0a546cf619614267",
        "ncu dram__bytes of tc_partial_kernel<32> NVFP4 form on decode_n2, one call per point kind"),
    ("decode_n2", "tensor-cluster"): (118056320, "0a546cf619614267",
        "ncu dram__bytes of tc_partial_kernel<32> cluster fold on decode_n2, one call per point kind"),
}

def _kernel_source_digest():
    """Digest of the kernel sources with comments and blank space removed, so
    that only a change of code makes the recorded traffic stale."""
    import hashlib
    import re
    d = hashlib.sha256()
    src = os.path.join(ROOT, "tensor_layer_reconciliation_b200", "csrc")
    for name in sorted(os.listdir(src)):
        with open(os.path.join(src, name), encoding="utf-8") as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        text = " ".join(text.split())
        d.update(name.encode() + b"\0" + text.encode())
    return d.hexdigest()[:16]


def _profiled_traffic(workload, path):
    rec = PROFILED_TRAFFIC.get((workload, path))
    if rec is None or rec[1] != _kernel_source_digest():
        return None
    return rec[0]


# ------------------------------------------------------------------ workload --

class Workload:
    """All points of one config resident on one GPU: packed weights, inputs, outputs.

    x and the residual of all points live in two flat buffers (one host->device
    copy each per end-to-end step); the outputs likewise (one copy back).
    """

    def __init__(self, cfg, device, variant="auto", staged=False, weights="bf16"):
        import tensor_layer_reconciliation_b200 as tlr
        self.cfg = cfg
        self.device = device
        self.weights = weights
        m, h, n = cfg.tokens, cfg.hidden, cfg.n_ranks
        self.plans = {}
        for p in cfg.points:
            if p.k not in self.plans:
                self.plans[p.k] = tlr.Plan(n, m, p.k, h, variant=variant, staged=staged)
        x_sizes = [m * p.k for p in cfg.points]
        self.x_off = np.concatenate([[0], np.cumsum(x_sizes)]).astype(np.int64)
        self.x_all = torch.empty(int(self.x_off[-1]), dtype=torch.bfloat16, device=device)
        self.res_all = torch.empty(cfg.n_points * m * h, dtype=torch.bfloat16, device=device)
        self.out_all = torch.empty(cfg.n_points * m * h, dtype=torch.bfloat16, device=device)
        self.w_packed = []
        ws_fn = {"mxfp8": "mxfp8_workspace_bytes", "nvfp4": "nvfp4_workspace_bytes"}.get(
            weights, "workspace_bytes")
        ws_need = max(getattr(pl, ws_fn)(m) for pl in self.plans.values())
        self.workspace = (torch.zeros(ws_need, dtype=torch.uint8, device=device)
                          if ws_need else None)   # counter head zero on first use
        for i, p in enumerate(cfg.points):
            self.x(i).copy_(point_tensor(cfg, p, KIND_X, device))
            self.res(i).copy_(point_tensor(cfg, p, KIND_RESIDUAL, device))
            w = point_tensor(cfg, p, KIND_W, device)
            if weights == "mxfp8":        # (E4M3 codes, E8M0 scales) per point
                self.w_packed.append(self.plans[p.k].pack_weights_mxfp8(w))
            elif weights == "nvfp4":      # (E2M1 code pairs, E4M3 block scales + g) per point
                self.w_packed.append(self.plans[p.k].pack_weights_nvfp4(w))
            else:
                self.w_packed.append(self.plans[p.k].pack_weights(w))
            del w
        torch.cuda.synchronize(device)

    def x(self, i):
        p = self.cfg.points[i]
        return self.x_all[int(self.x_off[i]):int(self.x_off[i + 1])].view(self.cfg.tokens, p.k)

    def res(self, i):
        m, h = self.cfg.tokens, self.cfg.hidden
        return self.res_all[i * m * h:(i + 1) * m * h].view(m, h)

    def out(self, i):
        m, h = self.cfg.tokens, self.cfg.hidden
        return self.out_all[i * m * h:(i + 1) * m * h].view(m, h)

    def call(self, i, stream=None):
        """The reconciliation of point i through the public API."""
        plan = self.plans[self.cfg.points[i].k]
        if self.weights in ("mxfp8", "nvfp4"):
            q, sc = self.w_packed[i]
            fn = plan.reconcile_mxfp8 if self.weights == "mxfp8" else plan.reconcile_nvfp4
            fn(self.x(i), q, sc, self.res(i), out=self.out(i), workspace=self.workspace, stream=stream)
        else:
            plan.reconcile(self.x(i), self.w_packed[i], self.res(i), out=self.out(i),
                           workspace=self.workspace, stream=stream)

    def step(self):
        """One pass of the hot path over every point, on the current stream."""
        for i in range(self.cfg.n_points):
            self.call(i)

    def weight_bytes_read(self):
        """Bytes of packed weights one step reads."""
        if self.weights in ("mxfp8", "nvfp4"):
            return sum(q.numel() + sc.numel() for q, sc in self.w_packed)
        return self.cfg.weight_bytes()

    def path_name(self):
        """Which kernels one call runs: 'tensor' (tensor-core partials),
        'tensor-cluster' (the CLUSTER variant), 'exact-staged', 'exact-fused',
        'mxfp8' or 'nvfp4' (quantised shards)."""
        if self.weights in ("mxfp8", "nvfp4"):
            return self.weights
        pl = next(iter(self.plans.values()))
        if pl.effective_variant(self.cfg.tokens) == "tensor":
            return "tensor-cluster" if pl.variant == "cluster" else "tensor"
        return "exact-staged" if pl.staged else "exact-fused"

    def launches_per_step(self):
        """Kernels one step launches (MXFP8 calls take the tensor-core path's
        kernels: one where it folds on chip, two where a ring kernel follows)."""
        m = self.cfg.tokens
        if self.weights in ("mxfp8", "nvfp4"):
            return sum(1 if self.workspace is None or m <= 2 else 2 for p in self.cfg.points)
        return sum(self.plans[p.k].launches(m) for p in self.cfg.points)

    def capture(self):
        g = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream(self.device)
        s.wait_stream(torch.cuda.current_stream(self.device))
        with torch.cuda.stream(s):
            self.step()                      # warm the plans outside capture
        torch.cuda.current_stream(self.device).wait_stream(s)
        torch.cuda.synchronize(self.device)
        with torch.cuda.graph(g):
            self.step()
        return g


# --------------------------------------------------------------------- clocks --

class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu_index = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        import tempfile
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu_index}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = []
        try:
            with open(self.path) as f:
                for line in f:
                    parts = [s.strip() for s in line.split(",")]
                    if len(parts) >= 9:
                        rows.append(parts)
        except OSError:
            pass
        finally:
            if self.path:
                try:
                    os.unlink(self.path)
                except OSError:
                    pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[j] for r in rows for j in range(4) if r[5 + j] == "Active"})
        return {"sm_mhz": float(np.median(sm)) if sm else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": reasons,
                "samples": len(rows)}


# ------------------------------------------------------------------- oracle --

def _cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def cpu_baseline(cfg, threads=None, target_s=12.0):
    """The oracle as it stands on this host's cores, on a bounded sample.

    Sample: the first point of each projection kind (all M tokens; all H
    output columns, or a leading block of them for the large workloads), run
    repeatedly for about target_s seconds of oracle work in total; the step
    time is extrapolated by the number of points of each kind.
    """
    import oracle
    threads = threads or len(os.sched_getaffinity(0))
    kinds = {}
    for p in cfg.points:
        kinds.setdefault(p.kind, []).append(p)
    per_kind, desc, measured = {}, [], 0.0
    budget = target_s / len(kinds)
    for kind, pts in kinds.items():
        p = pts[0]
        x = point_tensor(cfg, p, KIND_X).view(torch.int16).numpy().view(np.uint16)
        w = point_tensor(cfg, p, KIND_W).view(torch.int16).numpy().view(np.uint16)
        r = point_tensor(cfg, p, KIND_RESIDUAL).view(torch.int16).numpy().view(np.uint16)
        # columns per call: all of them unless one call would exceed the budget
        t0 = time.perf_counter()
        oracle.reconcile(cfg.n_ranks, cfg.hidden, x, np.ascontiguousarray(w[:16]),
                         np.ascontiguousarray(r[:, :16]), cols=np.arange(16), threads=threads)
        per_col = (time.perf_counter() - t0) / 16
        cols = int(max(16, min(cfg.hidden, budget / max(per_col, 1e-9))))
        wc, rc, cc = (np.ascontiguousarray(w[:cols]), np.ascontiguousarray(r[:, :cols]),
                      np.arange(cols))
        reps, spent = 0, 0.0
        while spent < budget or reps == 0:
            t0 = time.perf_counter()
            oracle.reconcile(cfg.n_ranks, cfg.hidden, x, wc, rc, cols=cc, threads=threads)
            spent += time.perf_counter() - t0
            reps += 1
        per_kind[kind] = spent / reps * cfg.hidden / cols
        measured += spent
        desc.append(f"{kind} point {p.index} (K={p.k}): {cols} of {cfg.hidden} output columns "
                    f"x {reps} runs")
    step_s = sum(per_kind[p.kind] for p in cfg.points)
    return {"step_s": step_s, "cores": threads, "cpu_model": _cpu_model(),
            "sample": "; ".join(desc) +
            f"; step time extrapolated over {cfg.n_points} points ({measured:.1f} s measured)"}


def _sample_cols(hidden, n_ranks, count, seed):
    """Output columns checked at full size: both ends of every H/N chunk and a
    seeded spread."""
    hc = hidden // n_ranks
    cols = {0, 1, hidden - 1, hidden - 2}
    for c in range(n_ranks):
        cols |= {c * hc, c * hc + 1, c * hc + hc - 1}
    rng = np.random.default_rng(seed)
    cols |= set(int(v) for v in rng.integers(0, hidden, count))
    return np.array(sorted(c for c in cols if 0 <= c < hidden), dtype=np.int64)


def oracle_parity(wl, threads=None):
    """Parity of the outputs the timed graph wrote against the oracle, on
    sampled columns of sampled points (the first and last point of each
    projection kind; every token of each sampled column). Part of the CPU
    leg, outside every timed region.

    A partial is fragile when its fp64 value lies within 2^-19 * sum|x*w| of
    a bf16 rounding boundary, where a summation order other than the
    oracle's k-ascending fp32 chain may round it the other way; an output is
    fragile when one of its N partials is. Reported: the largest absolute
    error, the relative L2 error, the fragile partial and output counts, the
    outputs that differ from the oracle (and how many of those are not
    fragile: 0 is required), and the outputs beyond the 2e-2 absolute
    tolerance (and how many of those are not fragile).
    """
    import oracle
    cfg = wl.cfg
    threads = threads or len(os.sched_getaffinity(0))
    kinds = {}
    for p in cfg.points:
        kinds.setdefault(p.kind, []).append(p.index)
    idx = sorted({v for lst in kinds.values() for v in (lst[0], lst[-1])})
    cols = _sample_cols(cfg.hidden, cfg.n_ranks, 16 if cfg.tokens >= 1024 else 40,
                        seed=len(cfg.name))
    sq_err = sq_ref = 0.0
    st = dict(max_abs=0.0, fragile_partials=0, fragile_outputs=0, outputs_differing=0,
              differing_not_fragile=0, over_max_abs=0, over_max_abs_not_fragile=0,
              sampled_outputs=0, sampled_partials=0)
    t0 = time.perf_counter()
    for i in idx:
        p = cfg.points[i]
        x = point_tensor(cfg, p, KIND_X).view(torch.int16).numpy().view(np.uint16)
        w = point_tensor_rows(cfg, p, KIND_W, cols).view(torch.int16).numpy().view(np.uint16)
        r = point_tensor(cfg, p, KIND_RESIDUAL).view(torch.int16).numpy().view(np.uint16)
        r = np.ascontiguousarray(r[:, cols])
        if wl.weights == "mxfp8":     # over the dequantised shards (a row quantises alone)
            q, sc = oracle.mx_quantize(cfg.n_ranks, np.ascontiguousarray(w))
            w = oracle.mx_dequant_bf16(cfg.n_ranks, q, sc)
        elif wl.weights == "nvfp4":   # the tensor scale needs the whole weight's maximum
            wfull = point_tensor(cfg, p, KIND_W).view(torch.int16).numpy().view(np.uint16)
            q, sc, g = oracle.nvfp4_quantize(cfg.n_ranks, wfull)
            w = np.ascontiguousarray(oracle.nvfp4_dequant_bf16(cfg.n_ranks, q, sc, g)[cols])
        ref = oracle.reconcile(cfg.n_ranks, cfg.hidden, x, np.ascontiguousarray(w), r, cols=cols,
                               threads=threads)
        got = wl.out(i)[:, torch.from_numpy(cols).to(wl.device)].cpu().view(torch.int16).numpy().view(np.uint16)
        e = ref["pabs"] * 2.0 ** -19
        frag = oracle.bf16_rne_f64(ref["p64"] - e) != oracle.bf16_rne_f64(ref["p64"] + e)
        out_frag = frag.any(axis=0)
        g64 = oracle.f32(got).astype(np.float64)
        r64 = oracle.f32(ref["out"]).astype(np.float64)
        diff = np.abs(g64 - r64)
        differ = got != ref["out"]
        over = diff > TOL_MAX_ABS
        sq_err += float(np.sum((g64 - r64) ** 2))
        sq_ref += float(np.sum(r64 ** 2))
        st["max_abs"] = max(st["max_abs"], float(diff.max()))
        st["fragile_partials"] += int(frag.sum())
        st["fragile_outputs"] += int(out_frag.sum())
        st["outputs_differing"] += int(differ.sum())
        st["differing_not_fragile"] += int((differ & ~out_frag).sum())
        st["over_max_abs"] += int(over.sum())
        st["over_max_abs_not_fragile"] += int((over & ~out_frag).sum())
        st["sampled_outputs"] += int(got.size)
        st["sampled_partials"] += int(frag.size)
    st["rel_l2"] = float(np.sqrt(sq_err / sq_ref)) if sq_ref > 0 else 0.0
    st["within_tolerance"] = bool(st["rel_l2"] <= TOL_REL_L2 and st["max_abs"] <= TOL_MAX_ABS)
    st["within_tolerance_except_fragile"] = bool(st["rel_l2"] <= TOL_REL_L2 and
                                                 st["over_max_abs_not_fragile"] == 0 and
                                                 st["differing_not_fragile"] == 0)
    st["tolerance"] = {"max_abs": TOL_MAX_ABS, "rel_l2": TOL_REL_L2}
    st["sample"] = (f"points {idx} x {len(cols)} output columns x {cfg.tokens} tokens; "
                    f"oracle {time.perf_counter() - t0:.1f} s on {threads} threads")
    return st


# --------------------------------------------------------------------- main --

class HostPipeline:
    """A step from pinned host buffers through the public API.

    The points are cut into chunks. Chunk c's x and residual go host->device
    on one stream, its points are reconciled (one C-ABI call each) on the
    compute stream once they have arrived, and its outputs go device->host on
    a third stream; events order each chunk's buffers against the previous
    step's use of them, so consecutive steps may overlap safely.
    """

    def __init__(self, wl, chunks=8):
        self.wl = wl
        n = wl.cfg.n_points
        self.bounds = [(n * c // chunks, n * (c + 1) // chunks) for c in range(chunks)
                       if n * c // chunks < n * (c + 1) // chunks]
        self.x_host = torch.empty(wl.x_all.shape, dtype=torch.bfloat16, pin_memory=True)
        self.r_host = torch.empty(wl.res_all.shape, dtype=torch.bfloat16, pin_memory=True)
        self.o_host = torch.empty(wl.out_all.shape, dtype=torch.bfloat16, pin_memory=True)
        self.x_host.copy_(wl.x_all.cpu())
        self.r_host.copy_(wl.res_all.cpu())
        dev = wl.device
        self.s_in, self.s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        k = len(self.bounds)
        self.ev_in = [torch.cuda.Event() for _ in range(k)]
        self.ev_done = [torch.cuda.Event() for _ in range(k)]
        self.ev_out = [torch.cuda.Event() for _ in range(k)]
        self.used = False

    def start(self, compute):
        """Copies of the next step begin after what `compute` has queued."""
        self.s_in.wait_stream(compute)

    def step(self, compute):
        wl, mh = self.wl, self.wl.cfg.tokens * self.wl.cfg.hidden
        for c, (a, b) in enumerate(self.bounds):
            xa, xb = int(wl.x_off[a]), int(wl.x_off[b])
            ra, rb = a * mh, b * mh
            if self.used:   # chunk c's inputs were last read by these kernels
                self.s_in.wait_event(self.ev_done[c])
            with torch.cuda.stream(self.s_in):
                wl.x_all[xa:xb].copy_(self.x_host[xa:xb], non_blocking=True)
                wl.res_all[ra:rb].copy_(self.r_host[ra:rb], non_blocking=True)
            self.ev_in[c].record(self.s_in)
            compute.wait_event(self.ev_in[c])
            if self.used:   # chunk c's outputs were last read by this copy
                compute.wait_event(self.ev_out[c])
            with torch.cuda.stream(compute):
                for i in range(a, b):
                    wl.call(i, stream=compute)
            self.ev_done[c].record(compute)
            self.s_out.wait_event(self.ev_done[c])
            with torch.cuda.stream(self.s_out):
                self.o_host[ra:rb].copy_(wl.out_all[ra:rb], non_blocking=True)
            self.ev_out[c].record(self.s_out)
        self.used = True

    def finish(self, compute):
        """`compute` waits for every copy of the steps queued so far."""
        compute.wait_stream(self.s_out)
        compute.wait_stream(self.s_in)


def _dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def _max_over_ranks(v, world, device):
    if world == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _job_rate(units_per_rank, ms_per_step_max, world):
    """Whole-job rate: every rank's units of one step over the slowest rank's
    step time (weak scaling, one replica per rank)."""
    return units_per_rank * world / (ms_per_step_max * 1e-3)


def _barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def _config_keys(cfg, world, args):
    """The `config` object of a bench line: the same keys and values on both
    arms (what the library's own path does goes under `path` instead)."""
    return {"workload": cfg.name, "n_ranks": cfg.n_ranks, "tokens": cfg.tokens,
            "hidden": cfg.hidden, "points": cfg.n_points,
            "weights": args.weights, "variant": args.variant,
            "l2": "no flush: every step streams all points' distinct weights "
                  f"({cfg.weight_bytes() / 1e9:.2f} GB), larger than the 126 MB L2",
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU"}


def _configs_to_run(args):
    return BENCH_CONFIGS if args.config == "all" else [args.config]


def run_reference(args, world, rank):
    """The reference arm: the oracle timed on the host cores, on the headline
    workload (the first of the workloads the GPU arm runs)."""
    if rank != 0:
        return 0
    cfg = get_config(_configs_to_run(args)[0])
    for _ in range(args.warmup):
        cpu_baseline(cfg, target_s=1.0)
    times = []
    last = None
    for _ in range(args.steps):
        last = cpu_baseline(cfg, target_s=args.ref_seconds)
        times.append(last["step_s"])
    step_s = float(np.mean(times))
    tok = cfg.tokens / step_s
    line = {
        "impl": "reference", "metric": METRIC, "value": tok, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": step_s * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32-accumulate bf16", "data": "synthetic (seeded Philox)",
        "reconciliations_per_s": cfg.n_points / step_s,
        "config": _config_keys(cfg, world, args),
        "cpu_baseline": {"value": tok, "unit": "tokens/s", "cores": last["cores"],
                         "cpu_model": last["cpu_model"], "kind": "oracle",
                         "sample": last["sample"]},
        "e2e": {"value": tok, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_config(name, args, device, world, rank, local, peaks):
    """Times one workload (graph replays, eager calls, the end-to-end host
    pipeline) and, on rank 0 of a single-GPU run, the CPU leg (oracle
    baseline and parity). Returns its bench line (without the top-level
    per_config object). Every buffer is released before it returns."""
    cfg = get_config(name)
    if args.points:
        cfg = dataclasses.replace(cfg, layers=1, layer_points=cfg.layer_points)
        cfg.points[:] = cfg.points[:args.points]
    wl = Workload(cfg, device, variant=args.variant, staged=args.staged, weights=args.weights)

    graph = wl.capture()
    stream = torch.cuda.current_stream(device)
    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize(device)

    # ---- timed region: K graph replays, device-timed, max over ranks ------
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        _barrier(world)
        torch.cuda.synchronize(device)
        ev0.record(stream)
        marks = []
        for _ in range(args.steps):
            graph.replay()
            marks.append(torch.cuda.Event(enable_timing=True))
            marks[-1].record(stream)
        ev1.record(stream)
        torch.cuda.synchronize(device)
        _barrier(world)
    step_ms = ev0.elapsed_time(ev1) / args.steps
    step_ms = _max_over_ranks(step_ms, world, device)
    per_step = np.diff([0.0] + [ev0.elapsed_time(e) for e in marks])
    step_stats = {"min": float(per_step.min()), "median": float(np.median(per_step)),
                  "max": float(per_step.max())}
    clocks = clk.summary()

    # ---- per-call durations outside a graph (for reference only) ---------
    # the calls stage partials (bf16 partials or fp32 k-parts) exactly when
    # they need a workspace; the cluster fold and the exact fused kernel do not
    staged_path = wl.workspace is not None
    per_launch = []
    for _ in range(2):
        evs = []
        for i, p in enumerate(cfg.points):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            wl.call(i)
            b.record(stream)
            evs.append((a, b))
        torch.cuda.synchronize(device)
        per_launch.append([a.elapsed_time(b) for a, b in evs])
    call_ms_eager = np.mean(np.array(per_launch), axis=0)      # per point, ms

    # ---- end to end through the public API with host buffers -------------
    pipe = HostPipeline(wl, chunks=8)
    e2e_steps = max(3, min(args.steps, 10))
    for _ in range(2):
        pipe.step(stream)
    pipe.finish(stream)
    torch.cuda.synchronize(device)
    _barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    pipe.start(stream)
    for _ in range(e2e_steps):
        pipe.step(stream)
    pipe.finish(stream)
    e1.record(stream)
    torch.cuda.synchronize(device)
    e2e_ms = _max_over_ranks(e0.elapsed_time(e1) / e2e_steps, world, device)
    if not torch.equal(pipe.o_host, wl.out_all.cpu()):
        raise RuntimeError("end-to-end outputs differ from the graph's")
    h2d = (wl.x_all.numel() + wl.res_all.numel()) * 2
    d2h = wl.out_all.numel() * 2

    # ---- numbers ---------------------------------------------------------
    value = _job_rate(cfg.tokens, step_ms, world)
    recon = _job_rate(cfg.n_points, step_ms, world)
    step_bytes = cfg.algorithmic_bytes(staged_partials=staged_path)
    if args.weights in ("mxfp8", "nvfp4"):   # codes + scales in place of bf16 weights
        step_bytes = (cfg.algorithmic_bytes(staged_partials=staged_path) - cfg.weight_bytes()
                      + wl.weight_bytes_read())
    flops = cfg.flops()
    tensor_bound = cfg.tokens >= 1024
    # The hot path of one point is one reconciliation call: the partial kernel
    # and, on staged paths, the ring fold kernel, chained by programmatic
    # dependent launch inside the graph. Its average duration is the graph's
    # device time over the timed region divided by the points per step.
    call_ms = step_ms / cfg.n_points
    path = wl.path_name()
    one_kernel = wl.launches_per_step() == cfg.n_points
    fold_where = ("the N ranks of a tile in one cluster, ring fold through distributed shared memory"
                  if wl.workspace is None else
                  "k-split parts, ring fold by the CTA completing a tile")
    kern_name = {
        "mxfp8": (f"reconciliation call: tc_partial_kernel, MXFP8 form ("
                  + ("codes and scales to the block-scaled MMA, activations split into two E4M3 terms on chip"
                     if cfg.tokens <= 8 else "codes widened to bf16 tiles on chip")
                  + f"; {fold_where})" if one_kernel else
                  "reconciliation call: tc_partial_kernel, MXFP8 form, then a ring fold kernel"),
        "nvfp4": (f"reconciliation call: tc_partial_kernel, NVFP4 form (codes widened to bf16 "
                  f"tiles on chip; {fold_where})" if one_kernel else
                  "reconciliation call: tc_partial_kernel, NVFP4 form, then a ring fold kernel"),
        "exact-fused": "reconciliation call: exact_partial_kernel (partials, ring fold, residual)",
        "exact-staged": "reconciliation call: exact_partial_kernel then ring_reduce_kernel",
        "tensor": ("reconciliation call: tc2_partial_kernel on CTA pairs (partials staged; the CTA "
                   "storing a half tile's last rank folds it: ring order, residual)"
                   if one_kernel and cfg.tokens > 128 else
                   f"reconciliation call: tc_partial_kernel ({fold_where}; residual)"
                   if one_kernel else
                   "reconciliation call: tc_partial_kernel then a ring fold kernel"),
        "tensor-cluster": ("reconciliation call: tc_partial_kernel, CLUSTER variant (the N ranks x K parts "
                           "of a tile in one cluster, ring fold through distributed shared memory; residual)"),
    }[path]
    if tensor_bound:
        achieved = flops / (step_ms * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"]}
    else:
        achieved = step_bytes / (step_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"]}
    roof["traffic"] = _profiled_traffic(cfg.name, path)
    roof["traffic_unit"] = "bytes per call (DRAM read + write, ncu), averaged over the points"
    rec = PROFILED_TRAFFIC.get((cfg.name, path))
    roof["traffic_source"] = rec[2] if roof["traffic"] is not None else None
    roof["peak_source"] = peaks["source"] + " (burst: the step is timed alone)"
    roof["kernel"] = kern_name
    roof["call_ms_mean"] = call_ms
    roof["call_ms_mean_eager"] = float(np.mean(call_ms_eager))
    roof["algorithmic_bytes_per_call"] = step_bytes / cfg.n_points
    roof["algorithmic_flops_per_call"] = flops / cfg.n_points

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded Philox4x32-10, Gaussian by 2^16-point inverse CDF)",
        "reconciliations_per_s": recon,
        "step_ms_stats": step_stats,
        "hbm_gbs_step": step_bytes / (step_ms * 1e-3) / 1e9,
        "tflops_step": flops / (step_ms * 1e-3) / 1e12,
        "config": _config_keys(cfg, world, args),
        "path": {"weights_gb_per_step": wl.weight_bytes_read() / 1e9, "staged_partials": staged_path},
        "roofline": roof,
        "e2e": {"value": _job_rate(cfg.tokens, e2e_ms, world), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "mode": "pinned host copies + one C-ABI reconcile call per point, no graph; "
                        "8 chunks of points, copies on two streams overlapping the kernels"},
        "gpu_launches": wl.launches_per_step() * args.steps,
        "clocks": clocks,
    }
    # ---- the CPU leg: oracle baseline and parity (rank 0, one GPU) -------
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["parity"] = oracle_parity(wl)
        cb = cpu_baseline(cfg, target_s=args.cpu_seconds)
        line["cpu_baseline"] = {"value": cfg.tokens / cb["step_s"], "unit": "tokens/s",
                                "cores": cb["cores"], "cpu_model": cb["cpu_model"],
                                "kind": "oracle", "sample": cb["sample"]}
    del graph, pipe, wl
    gc.collect()
    torch.cuda.empty_cache()
    return line


def _per_config_entry(line):
    """The compact per-workload record under per_config."""
    keep = ("value", "unit", "ms_per_step", "reconciliations_per_s", "step_ms_stats", "roofline",
            "e2e", "gpu_launches", "clocks", "parity", "cpu_baseline", "config", "path")
    return {k: line[k] for k in keep if k in line}


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--config", default="all", choices=["all"] + CONFIG_ORDER,
                    help="one workload, or all four benchmarked ones (headline: decode_n2)")
    ap.add_argument("--variant", default="auto", choices=["auto", "exact", "tensor", "cluster"])
    ap.add_argument("--staged", action="store_true")
    ap.add_argument("--weights", default="bf16", choices=["bf16", "mxfp8", "nvfp4"],
                    help="mxfp8: E4M3 codes, E8M0 scales per 32 weights; nvfp4: E2M1 codes, "
                         "E4M3 scales per 16 weights, power-of-two tensor scale")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true",
                    help="skip the CPU leg (oracle baseline and parity)")
    ap.add_argument("--cpu-seconds", type=float, default=8.0,
                    help="oracle seconds of the CPU baseline per workload")
    ap.add_argument("--ref-seconds", type=float, default=8.0)
    ap.add_argument("--points", type=int, default=0,
                    help="run only the first P points of each workload (small profiling cases)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    names = _configs_to_run(args)

    world, rank, local = _dist_env()
    if world != args.gpus:
        ap.error(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    if args.impl == "reference":
        return run_reference(args, world, rank)

    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)
    peaks = _peaks()
    lines = {name: run_config(name, args, device, world, rank, local, peaks) for name in names}
    line = dict(lines[names[0]])
    if len(names) > 1:
        line["per_config"] = {name: _per_config_entry(lines[name]) for name in names}
        line["headline"] = f"{names[0]} (the pages' worked decode example); every workload " \
                           f"under per_config"
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
