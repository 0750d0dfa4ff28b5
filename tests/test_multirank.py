"""The multi-GPU path is replicas only: every rank runs its own verify step
and the bench reports all ranks' nodes over the slowest rank's time.  The
cross-rank aggregation is checked here on CPU with world_size 2 over gloo."""
import os
import socket
import sys
import time
from datetime import timedelta
from pathlib import Path

import pytest
import torch.multiprocessing as mp

ROOT = Path(__file__).resolve().parents[1]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, queue):
    sys.path.insert(0, str(ROOT))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r took (r + 1) ms per step and (r + 2) ms end to end
        step_max, e2e_max = bench.reduce_max_over_ranks([1.0 + rank, 2.0 + rank], device="cpu")
        value = bench.whole_job_value(64, world, step_max)
        # the reference arm runs on rank 0 only; other ranks return at once
        ran = bench.run_reference(None, rank) if rank != 0 else None
        queue.put((rank, step_max, e2e_max, value, ran))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_value_gloo():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, queue)) for r in range(world)]
    for p in procs:
        p.start()
    results = [queue.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, step_max, e2e_max, value, ran in results:
        assert step_max == 2.0 and e2e_max == 3.0
        assert value == pytest.approx(2 * 64 / 2e-3)
        assert ran is None


def test_single_rank_aggregation_is_identity():
    sys.path.insert(0, str(ROOT))
    import bench
    assert bench.reduce_max_over_ranks([1.5, 2.5], device="cpu") == [1.5, 2.5]
    assert bench.whole_job_value(256, 1, 0.5) == pytest.approx(512_000.0)


def _dying_worker(rank, world, port, queue, how):
    """Rank 1 fails before the cross-rank reduction, between steps with
    nothing in flight: it exits ("exit") or stops answering without leaving
    ("stall").  Rank 0 must get an error from the reduction, at the latest
    when the process group's timeout runs out, instead of waiting forever."""
    sys.path.insert(0, str(ROOT))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=3))
    if rank == 1:
        queue.put((rank, "left"))
        queue.close()
        queue.join_thread()
        if how == "stall":
            time.sleep(10)
        os._exit(3)
    t0 = time.monotonic()
    try:
        bench.reduce_max_over_ranks([1.0], device="cpu")
        queue.put((rank, "no error"))
    except Exception as e:  # the backend's timeout or connection error
        queue.put((rank, f"error after {time.monotonic() - t0:.1f}s: {type(e).__name__}"))
    queue.close()
    queue.join_thread()
    os._exit(0)


@pytest.mark.parametrize("how", ["exit", "stall"])
def test_lost_rank_ends_the_reduction_with_an_error_gloo(how):
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    procs = [ctx.Process(target=_dying_worker, args=(r, world, port, queue, how)) for r in range(world)]
    for p in procs:
        p.start()
    results = dict(queue.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
    assert results[1] == "left"
    assert results[0].startswith("error after"), results[0]
    waited = float(results[0].split()[2].split("s")[0])
    assert waited < 60.0
    assert procs[0].exitcode == 0 and procs[1].exitcode == 3
