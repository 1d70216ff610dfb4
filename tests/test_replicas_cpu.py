"""The multi-process (replica) path of bench.py on CPU: two gloo ranks.

The layer does not shard across GPUs in this build (each rank runs full replicas of the step
on its own batches); what the ranks share is host logic: disjoint token ranges, the slowest
rank's time as the job's time, the whole-job rate, and rank 0 alone printing (and, for the
reference arm, alone running)."""
import io
import os
import socket
import sys
from contextlib import redirect_stdout
from datetime import timedelta

import pytest

from conftest import ROOT


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        import bench
        offs = [bench.replica_token_offset(rank, b, 16) for b in range(bench.N_BATCHES)]
        slowest = bench.max_over_ranks(1.5 + rank, "cpu", world)
        rate = bench.whole_job_rate(world, 16, 10, slowest)
        # the reference arm: ranks other than 0 return at once and print nothing
        out = io.StringIO()
        if rank != 0:
            class A:
                workload = "tiny"
                steps = 1
                warmup = 0
                ref_tokens = 2
            with redirect_stdout(out):
                bench.run_reference(A())
        dist.barrier()
        q.put((rank, offs, slowest, rate, out.getvalue()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_replicas():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, offs0, slow0, rate0, out0), (r1, offs1, slow1, rate1, out1) = res
    assert (r0, r1) == (0, 1)
    n = len(offs0)
    assert offs0 == [16 * b for b in range(n)]
    assert offs1 == [16 * (n + b) for b in range(n)]             # disjoint, contiguous after rank 0
    assert slow0 == slow1 == 2.5                                  # the slowest rank's time, everywhere
    assert rate0 == rate1 == pytest.approx(2 * 16 * 10 / 2.5e-3)  # tokens of both ranks / that time
    assert out1 == ""                                             # rank 1 of the reference arm: no work
