"""Pins of the oracle's brute-force binning ("SplatRs: The Week the Gap
Closed", "Throughput: the tile rasterizer": count, emit, sort, range).

The oracle tests every (Gaussian, tile) pair for membership.  Here the same
pair list is built a second way, from the rectangles' row-major expansion and
a numpy lexsort, and the structural invariants of the result are checked.
"""
import numpy as np

import oracle as O
from scenes import make_cameras, make_scene, tiny_camera


def _expand(rect, valid, depth32, tiles_x):
    keys, gids = [], []
    for g in range(rect.shape[0]):
        x0, y0, x1, y1 = rect[g]
        if not valid[g] or x0 > x1 or y0 > y1:
            continue
        for ty in range(y0, y1 + 1):
            for tx in range(x0, x1 + 1):
                t = ty * tiles_x + tx
                keys.append((t << 32) | int(np.float32(depth32[g]).view(np.uint32)))
                gids.append(g)
    keys = np.array(keys, dtype=np.uint64)
    gids = np.array(gids, dtype=np.uint32)
    order = np.lexsort((gids, keys))
    return keys[order], gids[order]


def _check(p, cam):
    b = O.bin_pairs(p["rect"], p["valid"], p["depth32"], cam.width, cam.height)
    keys, gids = _expand(p["rect"], p["valid"], p["depth32"], cam.tiles_x)
    np.testing.assert_array_equal(b["keys"], keys)
    np.testing.assert_array_equal(b["gids"], gids)
    # count = rectangle area for drawable Gaussians, 0 otherwise
    np.testing.assert_array_equal(b["counts"], p["count"])
    assert b["n_pairs"] == int(p["count"].sum())
    # ranges partition [0, K) in tile order; empty tiles are [0, 0)
    r = b["ranges"].astype(np.int64)
    tiles = (b["keys"] >> np.uint64(32)).astype(np.int64)
    pos = 0
    for t in range(cam.tiles):
        s, e = r[t]
        if e == s:
            assert s == 0 and e == 0
            assert not np.any(tiles == t)
            continue
        assert s == pos
        assert np.all(tiles[s:e] == t)
        pos = e
    assert pos == b["n_pairs"]
    # within a tile, Gaussians appear in the global depth order
    order = O.depth_order(p["depth32"], p["rect"], p["valid"])
    rank = np.empty(len(p["valid"]), dtype=np.int64)
    rank[order] = np.arange(len(order))
    for t in range(cam.tiles):
        s, e = r[t]
        if e > s:
            assert np.all(np.diff(rank[b["gids"][s:e]]) > 0)
    return b


def test_binning_tiny_scene():
    cam = tiny_camera()
    p = O.project(make_scene("tiny"), cam)
    b = _check(p, cam)
    assert b["n_pairs"] > 1000


def test_binning_ragged_image_and_offscreen():
    # 100 x 70 px: 7 x 5 tiles, the last column and row partial; many
    # Gaussians project off-screen or behind the camera
    cam = tiny_camera(100, 70, 90.0, distance=0.8)
    params = make_scene("tiny", n=400, seed=5)
    params["log_scales"] = params["log_scales"] + 1.0
    p = O.project(params, cam)
    assert (p["valid"] == 0).sum() > 0 and (p["count"] == 0).sum() > (p["valid"] == 0).sum()
    _check(p, cam)


def test_binning_ring_camera_equal_depths():
    cam = make_cameras("student", count=3)[1]
    params = make_scene("student", n=3000)
    p = O.project(params, cam)
    # force ties in depth: equal keys must be ordered by Gaussian id
    p["depth32"] = np.round(p["depth32"], 1).astype(np.float32)
    b = _check(p, cam)
    k = b["keys"]
    same = k[1:] == k[:-1]
    assert same.any() and np.all(b["gids"][1:][same] > b["gids"][:-1][same])


def test_rect_rule_matches_float_arithmetic():
    """The rectangle is floor((m -+ r)/16) per axis in single precision,
    clamped to the grid; count is its area."""
    rng = np.random.default_rng(2)
    n = 5000
    m = rng.uniform(-200, 1200, (n, 2)).astype(np.float32)
    r = np.ceil(rng.uniform(0.5, 300, n)).astype(np.float32)
    valid = np.ones(n, np.uint8)
    rect, count = O.tile_rects(m, r, valid, 980, 545)
    tx, ty = 62, 35
    lo = np.floor((m - r[:, None]) * np.float32(1 / 16)).astype(np.float64)
    hi = np.floor((m + r[:, None]) * np.float32(1 / 16)).astype(np.float64)
    lo = np.maximum(lo, 0)
    hi = np.minimum(hi, [tx - 1, ty - 1])
    nonempty = np.all(lo <= hi, axis=1)
    area = np.where(nonempty, (hi[:, 0] - lo[:, 0] + 1) * (hi[:, 1] - lo[:, 1] + 1), 0)
    np.testing.assert_array_equal(count, area.astype(np.int32))
    np.testing.assert_array_equal(rect[nonempty, :2], lo[nonempty].astype(np.int32))
    np.testing.assert_array_equal(rect[nonempty, 2:], hi[nonempty].astype(np.int32))
