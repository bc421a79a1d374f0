"""The N-GPU path of the benchmark on CPU: two gloo ranks.

Decode shards by sequence batch with no exchange step (each rank owns its batch, block
pool and tables), so the only cross-rank operations are the timing reduction (max over
ranks) and the byte totals.  Each rank here builds its own batch (seed + rank), checks the
batches differ, and checks the max-over-ranks time and the whole-job GB/s.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import bench
    import synth
    from oracle.block_manager import BlockManager
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        w = synth.build_workload("tiny_fp32", bench.rank_seed(0, rank), BlockManager)
        mine = float(w.q.sum())
        t = torch.tensor([mine])
        gathered = [torch.zeros(1) for _ in range(world)]
        dist.all_gather(gathered, t)
        per_rank_time = 0.5 + rank            # rank 1 is the slow one
        slowest = bench.reduce_max(per_rank_time, dist)
        gbs = bench.whole_job_gbs([1e9] * world, 10, slowest)
        q.put((rank, [float(x) for x in gathered], slowest, gbs))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_time_as_the_slowest_and_sum_bytes():
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
    (_, g0, t0, b0), (_, g1, t1, b1) = res
    assert g0 == g1 and g0[0] != g0[1]      # each rank decodes its own batch
    assert t0 == t1 == 1.5                  # max over ranks
    assert b0 == b1 == pytest.approx(2 * 1e9 * 10 / 1.5 / 1e9)
