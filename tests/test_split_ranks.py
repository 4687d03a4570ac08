"""Host side of split-context decode on CPU with two gloo ranks (no GPU).

What the multi-rank path must get right besides its kernels: every page of a request belongs to
exactly one rank in increasing ranges (so candidates gathered in rank order are in block order),
exactly one rank holds the newest position (it appends the new index key and attends to the tail),
and the exchange returns every rank's tensor in rank order on every rank.
"""
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("n_pages,world", [(4096, 2), (4097, 3), (5, 4), (64, 8), (1, 1)])
def test_partition_covers_every_page_once_in_increasing_ranges(n_pages, world):
    from block_sparse_attention_c4_b200.split import holds_position, partition_pages

    lo, cnt = partition_pages(n_pages, world)
    assert len(lo) == len(cnt) == world and lo[0] == 0 and sum(cnt) == n_pages
    assert all(lo[r] + cnt[r] == lo[r + 1] for r in range(world - 1))
    assert max(cnt) - min(cnt) <= 1
    for pos in {0, 63, 64, 64 * n_pages - 1, (64 * n_pages) // 2}:
        if pos >= 64 * n_pages:
            continue
        owners = [r for r in range(world) if holds_position(lo[r], cnt[r], pos)]
        assert len(owners) == 1


def _rank_main(rank, world, port, out):
    import datetime

    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    from block_sparse_attention_c4_b200.split import all_gather_stack

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # a rank's candidates: keys (int32 view of uint32), block ids in its own range, counts
        B = 3
        keys = torch.arange(B * 512, dtype=torch.int32).view(B, 512) * (rank + 1)
        ids = torch.arange(B * 512, dtype=torch.int32).view(B, 512) + 100000 * rank
        n = torch.tensor([512, 7 + rank, 0], dtype=torch.int32)
        lse = torch.full((B, 16), float(rank), dtype=torch.float32)
        got = [all_gather_stack(t) for t in (keys, ids, n, lse)]
        out.put((rank, [g.numpy() for g in got]))
    finally:
        dist.destroy_process_group()


def test_exchange_returns_every_rank_in_rank_order():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        r, got = q.get(timeout=120)
        res[r] = got
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(world):
        keys, ids, n, lse = res[r]
        assert keys.shape == (world, 3, 512) and n.shape == (world, 3) and lse.shape == (world, 3, 16)
        for k in range(world):
            assert (keys[k] == torch.arange(3 * 512).view(3, 512).numpy() * (k + 1)).all()
            assert (ids[k] // 100000 == k).all()  # rank order = block order
            assert list(n[k]) == [512, 7 + k, 0]
            assert (lse[k] == k).all()
