"""Host logic of the data-parallel training step on CPU: two gloo ranks, each
with its own cameras' mean gradient, make one all-reduce and hand Adam the
mean over ranks ("Training a smaller scene": one model fitted to many
cameras, here split across GPUs)."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from gaussian_splatting_differentiable_tile_b200.raster import _flat_views, data_parallel_step

SHAPES = {"means": (5, 3), "log_scales": (5, 3), "quats": (5, 4), "opacity_logits": (5,), "colors": (5, 3)}


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _local_grads(rank):
    rng = np.random.default_rng(100 + rank)
    return {k: rng.normal(size=sh).astype(np.float32) for k, sh in SHAPES.items()}


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        flat, views = _flat_views(SHAPES, "cpu")
        calls = []

        def local_step():
            calls.append("local")
            for k, v in _local_grads(rank).items():
                views[k].copy_(torch.from_numpy(v))

        def adam_step(scale):
            calls.append("adam")
            out[rank] = (scale, {k: (views[k] * scale).numpy().copy() for k in SHAPES}, list(calls))

        data_parallel_step(local_step, adam_step, flat)
    finally:
        dist.destroy_process_group()


def test_flat_views_are_aligned_and_disjoint():
    flat, views = _flat_views(SHAPES, "cpu")
    spans = []
    for k, v in views.items():
        off = (v.data_ptr() - flat.data_ptr()) // 4
        assert off % 4 == 0 and tuple(v.shape) == SHAPES[k] and v.is_contiguous()
        spans.append((off, off + v.numel()))
    spans.sort()
    assert all(a[1] <= b[0] for a, b in zip(spans, spans[1:]))
    assert spans[-1][1] <= flat.numel()


def test_two_ranks_apply_the_mean_gradient():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    expect = {k: (_local_grads(0)[k].astype(np.float64) + _local_grads(1)[k]) / 2 for k in SHAPES}
    for r in range(world):
        scale, g, calls = res[r]
        assert scale == 0.5 and calls == ["local", "adam"]
        for k in SHAPES:
            np.testing.assert_allclose(g[k], expect[k], rtol=1e-6, atol=1e-7)
