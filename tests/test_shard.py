"""Multi-rank host logic (bit_kv_cache_23_b200.shard) on CPU: the head partition
used to split a layer over GPUs, and the cross-rank reductions that turn per-rank
times into the whole-job rate, run as two gloo ranks."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from bit_kv_cache_23_b200 import shard


@pytest.mark.parametrize("H,world", [(40, 1), (40, 2), (40, 3), (40, 8), (12, 5), (7, 7), (1, 1)])
def test_head_range_partitions(H, world):
    ranges = [shard.head_range(r, world, H) for r in range(world)]
    owned = [h for h0, h1 in ranges for h in range(h0, h1)]
    assert owned == list(range(H))                    # every head once, in order
    sizes = [h1 - h0 for h0, h1 in ranges]
    assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1


def test_head_range_rejects_bad_input():
    with pytest.raises(ValueError):
        shard.head_range(2, 2, 40)
    with pytest.raises(ValueError):
        shard.head_range(0, 4, 3)


def test_single_process_reductions_are_identity():
    assert shard.max_over_ranks(2.5) == 2.5
    assert shard.sum_over_ranks(2.5) == 2.5
    assert shard.throughput(100.0, 4.0) == 25.0


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, outdir):
    os.environ["GLOO_SOCKET_IFNAME"] = os.environ.get("GLOO_SOCKET_IFNAME", "lo")
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        mx = shard.max_over_ranks([3.0, 5.0][rank])
        sm = shard.sum_over_ranks([3.0, 5.0][rank])
        # replicas: each rank a whole layer of 1560 query tokens, times 1.0 s and 2.0 s
        rep = shard.throughput(1560.0, [1.0, 2.0][rank])
        # heads split: each rank the query tokens of its share of the 40 heads
        h0, h1 = shard.head_range(rank, world, 40)
        hd = shard.throughput(1560.0 * (h1 - h0) / 40, [0.5, 0.75][rank])
        got = [None] * world
        dist.all_gather_object(got, (h0, h1))
        with open(os.path.join(outdir, f"r{rank}.txt"), "w") as f:
            f.write(repr((mx, sm, rep, hd, got)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks(tmp_path):
    world = 2
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    res = [eval(open(tmp_path / f"r{r}.txt").read()) for r in range(world)]
    for mx, sm, rep, hd, got in res:
        assert mx == 5.0 and sm == 8.0
        assert rep == pytest.approx(2 * 1560.0 / 2.0)       # all ranks' units / slowest time
        assert hd == pytest.approx(1560.0 / 0.75)           # one layer / slowest rank
        assert got == [(0, 20), (20, 40)]
    assert res[0] == res[1]                                  # every rank sees the same result
