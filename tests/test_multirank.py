"""The N > 1 path of bench.py on CPU: two ranks over gloo (no GPU).

A decode step shards by request with no exchange between ranks (replicas), so what the
multi-rank path has to get right is host logic: each rank decodes its own requests, the
step time of the whole job is the slowest rank's (all_reduce MAX, every rank agrees), the
reported throughput counts every rank's requests, and the reference arm runs on rank 0 only.
"""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime

    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench
    import qsa_gen as G

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        r, w, lr = bench.dist_env()
        seed = bench.replica_seed(r)
        lens = [int(x) for x in G.decode_128k(seed=seed, batch=4).lens]
        # rank-specific timings: the job takes the slowest rank's
        times = bench.max_over_ranks([10.0 + rank, 20.0 - 5.0 * rank], w)
        value = bench.job_throughput(64, w, times[0])

        class Args:
            batch, steps, warmup = 4, 1, 0

        ref = bench.run_reference(Args, r, w) if r != 0 else "rank 0 skipped here"
        out.put((r, w, lr, seed, lens, times, value, ref))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_requests_and_take_the_slowest_time():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        r, w, lr, seed, lens, times, value, ref = q.get(timeout=120)
        res[r] = (w, lr, seed, lens, times, value, ref)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res[0][0] == res[1][0] == world and res[0][1] == 0 and res[1][1] == 1
    # each replica decodes its own requests
    assert res[0][2] != res[1][2] and res[0][3] != res[1][3]
    # every rank sees the maxima over the ranks: step 11 ms (rank 1), e2e 20 ms (rank 0)
    assert res[0][4] == res[1][4] == [11.0, 20.0]
    # whole-job throughput: both ranks' 64 requests over the slowest step
    assert res[0][5] == pytest.approx(2 * 64 / 11e-3)
    # the reference arm does no work and prints nothing on other ranks
    assert res[1][6] is None
