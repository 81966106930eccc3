"""The N > 1 host path of bench.py on CPU: two gloo ranks.

Heads are independent, so the multi-GPU path has no data-path collective:
each rank runs the single-GPU prefill on its own GPU and the ranks meet only
in a barrier and in the max of their timings.  These tests run that host
logic with the gloo backend (world size 2, 127.0.0.1) — rank set-up, the
barrier, the max over ranks, the job-rate aggregation — and the reference
arm's rule that only rank 0 runs and prints."""
import io
import json
import multiprocessing as mp
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _env(rank, world, port):
    return {"RANK": str(rank), "LOCAL_RANK": str(rank), "WORLD_SIZE": str(world),
            "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)}


def _rank_timing(rank, world, port, out):
    os.environ.update(_env(rank, world, port))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    w, r, local = bench.dist_setup()
    bench.barrier(w)
    ms = 2.0 + 3.0 * r                       # rank 1 is the slow one
    slowest = bench.max_over_ranks(ms, w)
    rate = bench.job_rate(w, 131072, slowest)
    bench.barrier(w)
    dist.destroy_process_group()
    out.put((r, w, local, slowest, rate))


def _rank_reference(rank, world, port, out):
    os.environ.update(_env(rank, world, port))
    sys.path.insert(0, ROOT)
    import bench
    buf = io.StringIO()
    with redirect_stdout(buf):
        rc = bench.main(["--impl", "reference", "--gpus", str(world), "--steps", "1", "--warmup", "0",
                         "--ref-tokens", "8"])
    out.put((rank, rc, buf.getvalue()))


def _run(target, world=2, timeout=120):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=target, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=timeout) for _ in procs]
    for p in procs:
        p.join(timeout=timeout)
        assert p.exitcode == 0
    return sorted(res)


def test_two_rank_max_and_job_rate():
    res = _run(_rank_timing)
    assert [r[0] for r in res] == [0, 1]
    for r, w, local, slowest, rate in res:
        assert w == 2 and local == r
        assert slowest == 5.0                      # the max over ranks, seen by every rank
        assert rate == pytest.approx(2 * 131072 / 5e-3)


def test_reference_arm_prints_on_rank_zero_only():
    res = _run(_rank_reference, timeout=300)
    (r0, rc0, out0), (r1, rc1, out1) = res
    assert rc0 == 0 and rc1 == 0
    assert out1 == ""
    line = json.loads(out0.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["value"] > 0 and line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["cpu_baseline"]["kind"] == "oracle"


def test_job_rate_is_weak_scaling():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.job_rate(1, 100, 1.0) == pytest.approx(1e5)
    assert bench.job_rate(4, 100, 2.0) == pytest.approx(2e5)
