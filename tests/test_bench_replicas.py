"""The N > 1 path of bench.py on CPU: two gloo ranks stand in for two GPUs.

The forward has no exchange step (tokens are independent), so `bench.py --gpus N`
runs N replicas: one process group for the barriers, the slowest rank's time for
the whole job, whole-job tokens/s = N x tokens per rank / that time, and only
rank 0 prints (and, for the reference arm, works).
"""

import argparse
import contextlib
import io
import os
import socket

import torch
import torch.multiprocessing as mp

import bench

WORLD = 2
MS = [1.5, 2.5]  # per-rank step times (ms): rank 1 is the slow replica


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(WORLD), LOCAL_RANK=str(rank))
    pg = bench.init_replicas(WORLD, rank, backend="gloo")
    cpu = torch.device("cpu")
    torch.distributed.barrier()
    ms = bench.max_over_ranks(MS[rank], pg, cpu)
    e2e = bench.max_over_ranks(10.0 * MS[rank], pg, cpu)
    value = bench.replica_throughput(WORLD, 4096, ms)
    # the reference arm: ranks other than 0 return at once and print nothing
    out = io.StringIO()
    if rank != 0:
        with contextlib.redirect_stdout(out):
            bench.run_reference(argparse.Namespace(steps=1, warmup=3, gpus=WORLD),
                                dict(bench.WORKLOADS["tiny"]), rank)
    torch.distributed.barrier()
    torch.distributed.destroy_process_group()
    q.put((rank, pg, ms, e2e, value, out.getvalue()))


def test_two_replicas_report_the_slowest_rank_and_the_whole_job_throughput():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, port, q)) for r in range(WORLD)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(WORLD))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, pg, ms, e2e, value, printed in res:
        assert pg is True
        assert ms == max(MS) and e2e == 10.0 * max(MS)
        assert value == WORLD * 4096 / (max(MS) * 1e-3)
        assert printed == ""


def test_single_replica_needs_no_process_group():
    assert bench.init_replicas(1, 0) is False
    assert bench.max_over_ranks(3.25, False, torch.device("cpu")) == 3.25
    assert bench.replica_throughput(1, 4096, 2.0) == 4096 / 2e-3
