"""gs_bin_and_sort_static: binning for callers that cannot allocate device
memory (a frame loop that must not call cudaMalloc, a plug-in without an
allocator).  It keeps its scratch in a fixed array inside libgs.so; its
results must equal gs_bin_and_sort's, bit for bit (integer work), call after
call on the shared array.

This file is collected last on purpose, so that a run stopping at the first
failure has run every other test; it passes alone in a fresh process too.
"""
import numpy as np
import pytest
import torch

import gaussian_splatting_differentiable_tile_b200 as G
from scenes import Camera, make_cameras, make_scene, tiny_camera

from gpu_common import cuda_params

pytestmark = pytest.mark.gpu


def _project(cam, params):
    n = params["means"].shape[0]
    proj = G.Projected(n)
    G.gs_project(cam, cuda_params(params), proj)
    return proj, n


def _reference(cam, proj, n):
    need = int(proj.count[:n].sum().item()) if n else 0
    bins = G.Bins(n, max(64 * n, need) + cam.tiles + 4096, cam.width, cam.height)
    K = G.gs_bin_and_sort(cam, n, proj, bins)
    return (K, bins.pair_tile[:K].cpu().numpy(), bins.pair_gid[:K].cpu().numpy(),
            bins.ranges.cpu().numpy()[:cam.tiles])


def _static(cam, proj, n, max_pairs):
    pt = torch.full((max_pairs,), -1, dtype=torch.int32, device="cuda")
    pg = torch.full((max_pairs,), -1, dtype=torch.int32, device="cuda")
    rg = torch.full((cam.tiles, 2), -1, dtype=torch.int32, device="cuda")
    K = G.gs_bin_and_sort_static(cam, n, proj, pt, pg, rg)
    return K, pt[:K].cpu().numpy(), pg[:K].cpu().numpy(), rg.cpu().numpy()


def test_static_variant_matches_bin_and_sort_on_consecutive_calls():
    # two calls in a row on the shared array: a larger frame first, then a
    # smaller one, so stale contents of the first would show in the second
    cases = [(make_cameras("student", count=60)[11], make_scene("student", n=30_000, seed=2)),
             (tiny_camera(200, 150, 180.0, distance=3.0), make_scene("tiny", n=1537, seed=9))]
    for cam, params in cases:
        proj, n = _project(cam, params)
        K, tile, gid, ranges = _reference(cam, proj, n)
        Ks, tile_s, gid_s, ranges_s = _static(cam, proj, n, max_pairs=K + 1000)
        assert Ks == K
        np.testing.assert_array_equal(tile_s, tile)
        np.testing.assert_array_equal(gid_s, gid)
        np.testing.assert_array_equal(ranges_s, ranges)


def _synthetic(W, H, n, seed, spread, log_scale):
    """n Gaussians in front of an identity camera looking down +z."""
    cam = Camera(np.eye(4), W * 0.5, W * 0.5, W / 2.0, H / 2.0, W, H)
    rng = np.random.default_rng(seed)
    params = {"means": np.column_stack([rng.uniform(-spread, spread, n), rng.uniform(-spread, spread, n),
                                        rng.uniform(2, 4, n)]).astype(np.float32),
              "log_scales": rng.normal(log_scale, 0.2, (n, 3)).astype(np.float32),
              "quats": rng.normal(size=(n, 4)).astype(np.float32),
              "opacity_logits": rng.normal(0, 1, n).astype(np.float32),
              "colors": rng.uniform(0, 1, (n, 3)).astype(np.float32)}
    return cam, params


def test_static_variant_long_lists_and_large_grids():
    """The two paths of the shared array that short lists on small grids never
    reach, each compared with gs_bin_and_sort: tile lists longer than 8192
    entries (sorted by the long-list radix sort in the array's ping-pong
    space), and a grid of more than 16384 tiles (counted in the array's
    count matrix instead of shared memory, with fewer CTAs)."""
    cases = [_synthetic(48, 32, 10_000, 3, 0.3, -0.5),        # 6 tiles, ~10 000 entries each
             _synthetic(2400, 1800, 3000, 4, 1.0, -3.0)]       # 150 x 113 = 16 950 tiles
    for cam, params in cases:
        proj, n = _project(cam, params)
        K, tile, gid, ranges = _reference(cam, proj, n)
        length = ranges[:, 1] - ranges[:, 0]
        assert length.max() > 8192 or cam.tiles > 16384
        Ks, tile_s, gid_s, ranges_s = _static(cam, proj, n, max_pairs=K + 16)
        assert Ks == K
        np.testing.assert_array_equal(tile_s, tile)
        np.testing.assert_array_equal(gid_s, gid)
        np.testing.assert_array_equal(ranges_s, ranges)


def test_static_variant_rejects_sizes_beyond_its_array():
    cam = tiny_camera()
    proj = G.Projected(16)
    small = torch.empty(16, dtype=torch.int32, device="cuda")
    rg = torch.empty(cam.tiles, 2, dtype=torch.int32, device="cuda")
    big = torch.empty((1 << 20) + 1, dtype=torch.int32, device="cuda")
    with pytest.raises(G.GSError) as ei:  # more pairs than the array holds
        G.gs_bin_and_sort_static(cam, 16, proj, big, big, rg)
    assert ei.value.code == G.GS_ERR_TOO_LARGE
    with pytest.raises(G.GSError) as ei:  # more Gaussians than the array holds
        G.gs_bin_and_sort_static(cam, (1 << 18) + 1, G.Projected((1 << 18) + 1), small, small, rg)
    assert ei.value.code == G.GS_ERR_TOO_LARGE


def test_static_variant_reports_capacity():
    cam = tiny_camera()
    params = make_scene("tiny")
    proj, n = _project(cam, params)
    K, _, _, _ = _reference(cam, proj, n)
    pt = torch.empty(K - 1, dtype=torch.int32, device="cuda")
    rg = torch.full((cam.tiles, 2), -1, dtype=torch.int32, device="cuda")
    with pytest.raises(G.GSError) as ei:
        G.gs_bin_and_sort_static(cam, n, proj, pt, pt.clone(), rg)
    assert ei.value.code == G.GS_ERR_CAPACITY and ei.value.n_pairs == K
    # as documented: every tile's range is left empty, so a render of these
    # ranges draws only background
    assert int(rg.abs().sum().item()) == 0
