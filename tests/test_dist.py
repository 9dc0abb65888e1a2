"""The N > 1 path of bench.py on CPU: world_size-2 gloo ranks exercise the
host logic the multi-GPU bench uses (rank/world from the environment, per-rank
input shards, max-over-ranks timing, whole-job throughput, rank-0-only output of
the reference arm).  The data path itself has no collective: each rank owns its
own sequences."""
import multiprocessing as mp
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    try:
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                          WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
        sys.path.insert(0, ROOT)
        import datetime

        import torch
        import torch.distributed as dist
        dist.init_process_group("gloo", rank=rank, world_size=world,
                                timeout=datetime.timedelta(seconds=60))
        import bench
        w, r, l = bench._dist()
        ms = bench._max_over_ranks(10.0 + 5.0 * rank, w, torch.device("cpu"))
        dist.barrier()
        seeds = [bench.rank_seed(100, r, i) for i in range(3)]
        # the reference arm: only rank 0 runs it; the others return at once
        class A:  # noqa: E701 - minimal argument namespace
            workload, ref_tokens, ref_seconds, gpus = "t8k_h12", 64, 0.0, w
        rc = bench.run_reference(A, w, r) if r != 0 else 0
        q.put((r, w, l, ms, seeds, rc))
        dist.destroy_process_group()
    except Exception as e:  # report instead of hanging the parent
        q.put(("error", rank, repr(e)))


def test_two_gloo_ranks_host_logic():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
    errors = [x for x in res if x[0] == "error"]
    assert not errors, errors
    res = sorted(res)
    assert [x[0] for x in res] == [0, 1] and all(x[1] == 2 for x in res)
    assert all(x[3] == 15.0 for x in res)            # max over ranks, seen by every rank
    assert set(res[0][4]).isdisjoint(res[1][4])       # each rank draws its own shard
    assert res[1][5] == 0                             # non-zero ranks skip the reference arm


def test_whole_job_rate_is_weak_scaling():
    sys.path.insert(0, ROOT)
    import bench
    # 8192 tokens per rank per step, 4 ranks, 10 steps in 20 ms (slowest rank)
    assert bench.whole_job_rate(8192, 4, 10, 20.0) == pytest.approx(8192 * 4 * 10 / 0.02)
    assert bench.whole_job_rate(8192, 1, 10, 20.0) * 4 == bench.whole_job_rate(8192, 4, 10, 20.0)
