"""Host logic of bench.py's multi-rank path, run as two gloo ranks on the CPU.

With --gpus N every rank runs an independent replica of the step (the method's
tensor-parallel ranks are emulated inside each GPU), so the only cross-rank
steps are the barriers around the timed region and the max over ranks of the
step time; the job rate is every rank's units over the slowest rank's time.
The reference arm runs on rank 0 alone and the other ranks exit without work.
"""

import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
                      RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w, r, lr = bench._dist_env()
        assert (w, r, lr) == (world, rank, rank)
        bench._barrier(w)
        step_ms = 2.0 + rank                    # rank 1 is the slower one
        mx = bench._max_over_ranks(step_ms, w, torch.device("cpu"))
        rate = bench._job_rate(1, mx, w)
        # reference arm: rank 0 alone does work; the others return at once
        args = type("A", (), {"config": "tiny", "warmup": 3, "steps": 1, "ref_seconds": 0.1,
                              "weights": "bf16", "variant": "auto", "gpus": world})()
        ret = bench.run_reference(args, w, r) if r != 0 else None
        bench._barrier(w)
        q.put((rank, mx, rate, ret))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_and_job_rate():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(q.get(timeout=5) for _ in range(world))
    for rank, mx, rate, ret in got:
        assert mx == 3.0                         # both ranks see the slowest rank's time
        assert rate == pytest.approx(2 / 3e-3)   # 2 replicas x 1 unit over 3 ms
        if rank != 0:
            assert ret == 0


def test_job_rate_single_rank():
    sys.path.insert(0, ROOT)
    import bench
    assert bench._job_rate(128, 2.0, 1) == pytest.approx(64000.0)
    assert bench._max_over_ranks(1.5, 1, None) == 1.5
