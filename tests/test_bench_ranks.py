"""Host logic of the multi-rank benchmark on CPU: two gloo ranks split the
cameras as replicas (disjoint, covering every camera) and agree on the
max-over-ranks timing that the whole-job throughput divides by."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from scenes import SPECS, make_cameras


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cams = make_cameras(SPECS["train400k_half"])
        mine = bench.my_cameras(cams, rank, world)
        ids = [i for i, c in enumerate(cams) if any(c is m for m in mine)]
        gathered = [None] * world
        dist.all_gather_object(gathered, ids)
        # each rank reports a different time; all must see the same max
        t = bench.max_over_ranks([10.0 + rank, 5.0 * (world - rank)], world, "cpu")
        out[rank] = (gathered, t)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_cameras_split_and_max_over_ranks(world):
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    n_cams = len(make_cameras(SPECS["train400k_half"]))
    gathered = res[0][0]
    flat = sorted(i for ids in gathered for i in ids)
    assert flat == list(range(n_cams))  # disjoint and complete
    assert all(len(ids) == n_cams // world for ids in gathered)
    for r in range(world):
        assert res[r][1] == [10.0 + world - 1, 5.0 * world]


def test_one_rank_keeps_every_camera_and_more_ranks_than_cameras_still_work():
    cams = list(range(3))
    assert bench.my_cameras(cams, 0, 1) == cams
    assert bench.my_cameras(cams, 4, 5) == [0]  # a rank with no camera of its own renders one
    assert bench.max_over_ranks([1.5, 2.5], 1, "cpu") == [1.5, 2.5]
