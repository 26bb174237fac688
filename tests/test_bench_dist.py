"""The bench's multi-rank plumbing on CPU (gloo, world size 2): ranks agree on
the max over ranks, and the whole-job value divides the slowest rank's time by
all layer-steps of all ranks. The data path has no collective; only timing is
reduced."""
import os
import socket

import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    w, r, lr = bench.dist_env()
    total_ms = [12.5, 20.0][rank]  # rank 1 is the slow one
    m = bench.reduce_max(total_ms, "cpu", w)
    per_rank, value = bench.aggregate_us(m, 100, w)
    dist.barrier()
    dist.destroy_process_group()
    q.put((r, lr, w, m, per_rank, value))


def test_two_rank_max_and_aggregate():
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
    for rank, (r, lr, w, m, per_rank, value) in enumerate(res):
        assert (r, lr, w) == (rank, rank, 2)
        assert m == 20.0  # both ranks see the slowest rank's time
        assert per_rank == 200.0  # µs per layer-step on the slowest rank
        assert value == 100.0  # 200 layer-steps completed in 20 ms


def test_single_rank_is_identity():
    assert bench.reduce_max(3.5, "cpu", 1) == 3.5
    assert bench.aggregate_us(10.0, 50, 1) == (200.0, 200.0)
