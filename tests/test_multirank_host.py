"""Host logic of the N > 1 path, run as two gloo ranks on the CPU.

Pools on different GPUs exchange nothing on the data path (every sequence's
state is independent), so what N > 1 adds is bookkeeping: the slot partition,
the barrier around the timed region, the slowest rank's time and the
whole-job rate.  These run here with the same ``torch.distributed`` calls the
GPU ranks make, on the gloo backend.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from bit_recurrent_state_pace_b200.ranks import (aggregate_rate, barrier, max_over_ranks,
                                                 rank_of_slot, slot_range)


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, q):
    import datetime
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=30))
    try:
        out = {}
        # each rank's own elapsed time; every rank must see the slowest
        mine = [3.5, 7.25][rank]
        barrier(world)
        out["max"] = max_over_ranks(mine, world, "cpu")
        # the slot partition: gather every rank's share and check it on rank 0
        start, count = slot_range(4099, world, rank)
        t = torch.tensor([start, count], dtype=torch.int64)
        parts = [torch.zeros(2, dtype=torch.int64) for _ in range(world)]
        dist.all_gather(parts, t)
        out["parts"] = [tuple(int(x) for x in p) for p in parts]
        # whole-job rate from per-rank units and the slowest time
        out["rate"] = aggregate_rate(1000, world, out["max"])
        barrier(world)
        q.put((rank, out))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_max_partition_and_rate():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = {}
    for _ in range(world):
        rank, out = q.get(timeout=120)
        results[rank] = out
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(world):
        assert results[r]["max"] == 7.25
        assert results[r]["rate"] == pytest.approx(2 * 1000 / 7.25e-3)
    parts = results[0]["parts"]
    assert parts == results[1]["parts"]
    covered = []
    for start, count in parts:
        covered.extend(range(start, start + count))
    assert covered == list(range(4099))


@pytest.mark.parametrize("slots,world", [(0, 1), (1, 4), (7, 3), (4096, 8), (4099, 8), (5, 5)])
def test_slot_partition_is_balanced_disjoint_and_invertible(slots, world):
    seen = []
    counts = []
    for r in range(world):
        start, count = slot_range(slots, world, r)
        counts.append(count)
        for s in range(start, start + count):
            assert rank_of_slot(s, slots, world) == r
            seen.append(s)
    assert seen == list(range(slots))
    assert max(counts) - min(counts) <= 1


def test_partition_rejects_bad_arguments():
    with pytest.raises(ValueError):
        slot_range(10, 0, 0)
    with pytest.raises(ValueError):
        slot_range(10, 2, 2)
    with pytest.raises(ValueError):
        rank_of_slot(10, 10, 2)
    with pytest.raises(ValueError):
        aggregate_rate(10, 1, 0.0)
