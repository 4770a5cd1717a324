"""CPU (gloo, world size 2): the host side of `bench.py --gpus N`.

The pass does not shard (one weight pass per GPU; N GPUs run N independent replicas),
so the only cross-rank logic is the timing: every rank times its own replica, the
slowest rank's time is the job's step time, and the job throughput counts every
replica's bytes. The reference arm runs on rank 0 only.
"""

import contextlib
import importlib.util
import io
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        b = _bench()
        local = [3.25, 4.5][rank]                       # each rank's own device time
        slowest = b.max_over_ranks(dist, torch, local, torch.device("cpu"))
        q.put((rank, slowest, b.job_gbs(world, 12_228_526_080, slowest)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_gloo():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs)
    got = sorted(q.get(timeout=10) for _ in range(world))
    for rank, slowest, gbs in got:
        assert slowest == 4.5                              # every rank sees the slowest replica's time
        assert gbs == pytest.approx(2 * 12_228_526_080 / 4.5e-3 / 1e9)


def test_one_rank_max_is_identity():
    b = _bench()
    assert b.max_over_ranks(None, torch, 2.5, torch.device("cpu")) == 2.5
    assert b.job_gbs(1, 10**9, 1.0) == pytest.approx(1000.0)


def test_reference_arm_prints_on_rank_zero_only():
    b = _bench()

    class Args:
        steps, warmup = 1, 3

    out = io.StringIO()
    with contextlib.redirect_stdout(out):
        b.run_reference(Args(), rank=1, world=2)
    assert out.getvalue() == ""


def test_fp8_cpu_baseline_runs_the_oracle():
    b = _bench()
    r = b.cpu_baseline_fp8(seconds=0.01, rows=256)
    assert r["kind"] == "oracle" and r["unit"] == "GB/s" and r["value"] > 0 and r["cores"] >= 1
    assert "FP8 head slice" in r["sample"]
