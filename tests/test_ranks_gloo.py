"""The multi-GPU rank logic as two gloo processes on the CPU: every unit owned by exactly
one rank, max-over-ranks timing, the collective retry decision, clean shutdown."""

from __future__ import annotations

import os
import socket

import pytest
import torch.multiprocessing as mp

from chunked_causal_linear_b200.ranks import RankInfo, shard


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from chunked_causal_linear_b200 import ranks
    info = ranks.init(backend="gloo", timeout_s=60)
    units = list(ranks.shard(37, info))
    ranks.barrier(info)
    m = ranks.max_over_ranks(10.0 + rank, info)
    retry = ranks.any_over_ranks(rank == 1, info)
    none = ranks.any_over_ranks(False, info)
    ranks.finish(info)
    q.put((rank, units, m, retry, none))


@pytest.mark.parametrize("world", [2])
def test_two_gloo_ranks(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    results.sort()
    owned = sorted(u for _, units, _, _, _ in results for u in units)
    assert owned == list(range(37))
    for _, _, m, retry, none in results:
        assert m == 10.0 + (world - 1)
        assert retry is True and none is False


@pytest.mark.parametrize("n,world", [(0, 3), (5, 8), (37, 2), (64, 8), (7, 7)])
def test_shard_partitions_units(n, world):
    seen = []
    sizes = []
    for r in range(world):
        rg = shard(n, RankInfo(r, world, r))
        seen.extend(rg)
        sizes.append(len(rg))
    assert seen == list(range(n))
    assert max(sizes) - min(sizes) <= 1


def test_single_rank_needs_no_process_group():
    from chunked_causal_linear_b200 import ranks
    info = RankInfo(0, 1, 0)
    assert ranks.max_over_ranks(3.5, info) == 3.5
    assert ranks.any_over_ranks(True, info) is True
    ranks.barrier(info)
    ranks.finish(info)
