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


def _rollout_worker(rank, world, port, q):
    # each rank builds its inputs exactly as bench.py does (its own seed) and runs the
    # CPU oracle over a small rollout; the only collective is the gather of the results
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    from synthetic import CONFIGS
    from tests.test_multirank_cpu import _oracle_rollout

    bench.init_dist(world, "gloo")
    r, w, _ = bench.dist_info()
    cfg = CONFIGS["wan1.3b"].replace(H=2, P=48, F=2, chunks=4, S=24, nbits=6, capacity=1000)
    sizes, checksum = _oracle_rollout(cfg, bench.rank_seed(cfg.seed, r))
    out = [None] * w
    dist.all_gather_object(out, (r, sizes, checksum))
    q.put(out)
    dist.destroy_process_group()


def _oracle_rollout(cfg, seed):
    import numpy as np

    import bench
    from oracle import OracleTempCache

    R, chunks = bench.generate_inputs(cfg, "cpu", seed)
    o = OracleTempCache(cfg.H, cfg.d, cfg.nbits, cfg.tau, cfg.capacity, R.astype(np.float64))
    f = lambda x: x.to(torch.float64).numpy()  # noqa: E731
    checksum = 0.0
    for K, V, Qs in chunks:
        o.append_chunk(f(K), f(V))
        checksum += float(o.attend(f(Qs[0])).sum())
    return o.cache_size().tolist(), checksum


@pytest.mark.timeout(180)
def test_two_rank_independent_rollouts():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rollout_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=150) for _ in procs]
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    assert res[0] == res[1]                       # every rank gathered the same results
    (r0, s0, c0), (r1, s1, c1) = sorted(res[0])
    assert (r0, r1) == (0, 1) and c0 != c1        # the ranks' rollouts are independent
    # a rank's result depends on its seed only: recomputed here in one process
    import bench
    from synthetic import CONFIGS
    cfg = CONFIGS["wan1.3b"].replace(H=2, P=48, F=2, chunks=4, S=24, nbits=6, capacity=1000)
    assert _oracle_rollout(cfg, bench.rank_seed(cfg.seed, 1)) == (s1, c1)
