"""The N > 1 benchmark path on CPU: two gloo ranks, each with its own request batch (weak scaling,
no data-path collective); the whole-job value uses the slowest rank's time and the bytes of all
ranks."""
import os
import sys
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import torch.distributed as dist
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        # each rank: its own seeded batch, as bench.py builds it
        cases = bench._make_cases(rank, batch=4)
        local_bytes = sum(bench._kv_bytes(c) for c in cases)
        local_ms = 10.0 + 5.0 * rank
        ms, total = bench.aggregate_over_ranks(local_ms, local_bytes)
        q.put((rank, ms, total, local_bytes))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_aggregate_max_time_and_total_bytes():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    locals_ = [r[3] for r in res]
    assert locals_[0] != locals_[1]                      # the ranks really hold different batches
    for rank, ms, total, _ in res:
        assert ms == 15.0                                # slowest rank
        assert total == sum(locals_)                     # all ranks' bytes
