"""The benchmark's multi-rank logic on CPU: two gloo ranks.

Each rank decodes its own independent sequences (weak scaling, no data-path
collective); the job's time is the slowest rank's and its throughput counts
the tokens of every rank.  The oracle arm runs on rank 0 alone."""
import os
import socket

import pytest

torch = pytest.importorskip("torch")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, result_q):
    import datetime

    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms = [5.0, 8.25][rank]
        units = [4 * 64, 4 * 64 + 3][rank]
        t = bench.job_time_ms(ms, world, dist, "cpu")
        u = bench.job_units(units, world, dist, "cpu")
        # every rank takes the same collective steps; the reference arm does no work off rank 0
        ref_rc = bench.run_reference(_RefArgs()) if rank == 1 else None
        dist.barrier()
        result_q.put((rank, t, u, ref_rc))
    finally:
        dist.destroy_process_group()


class _RefArgs:
    seed, warmup, steps, gpus, workload = 0, 3, 2, 2, 2


def test_two_rank_time_is_max_and_units_sum():
    ctx = torch.multiprocessing.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    codes = [p.exitcode for p in procs]
    assert codes == [0, 0], codes
    res = sorted(q.get(timeout=5) for _ in range(2))
    for rank, t, u, _ in res:
        assert t == 8.25
        assert u == 4 * 64 * 2 + 3
    assert res[1][3] == 0


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.job_time_ms(3.5, 1) == 3.5
    assert bench.job_units(12, 1) == 12
