"""The N > 1 bench path on CPU: two gloo ranks check the max-over-ranks timing,
the whole-job rate and the per-rank seeds that make every rank's rollout
independent (no collective touches the data)."""
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
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench

    bench.init_dist(world, "gloo")
    r, w, _ = bench.dist_info()
    sec = 1.0 + r  # rank 1 is the slowest
    mx = bench.max_over_ranks(sec, w, torch.device("cpu"))
    rate = bench.aggregate_rate(120.0, w, mx)
    seeds = [None] * w
    dist.all_gather_object(seeds, bench.rank_seed(1001, r))
    q.put((r, mx, rate, seeds))
    dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_rank_timing_and_seeds():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=90) for _ in procs]
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    for r, mx, rate, seeds in res:
        assert mx == 2.0                      # the slowest rank's time
        assert rate == pytest.approx(120.0)   # 2 ranks x 120 frames / 2 s
        assert len(set(seeds)) == 2           # independent rollouts
