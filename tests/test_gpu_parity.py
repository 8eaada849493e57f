"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Integer stages (tile counts, the sorted pair list, tile ranges) must match bit
for bit when fed the same records; images within 1e-4; gradients within
1e-6 absolute or 1e-3 relative (cancellation excused against the sum of
absolute terms).  Sizes span several tiles with ragged edges and run on the
oracle in seconds.
"""
import numpy as np
import pytest
import torch

import gaussian_splatting_differentiable_tile_b200 as G
import oracle as O
from oracle import train as OT
from scenes import Camera, make_cameras, make_scene, make_target, tiny_camera

from gpu_common import (IMG_TOL, MARGIN_CUT, MARGIN_RADIUS, MARGIN_TILE, ambiguous_gaussians, ambiguous_pixels,
                        check_ambiguous, cuda_params, fill_projected, gpu_bin, gpu_render, grad_compare,
                        oracle_records, report, tiles_to_pixels)

pytestmark = pytest.mark.gpu


def _student_subset(n, seed=2):
    cam = make_cameras("student", count=60)[7]
    params = make_scene("student", n=n, seed=seed)
    return cam, params


def _ragged_cam():
    # 200 x 150 px: 13 x 10 tiles, last column 8 px wide and last row 6 px tall
    return tiny_camera(200, 150, 180.0, distance=3.0)


SCENES = {
    "tiny": lambda: (tiny_camera(), make_scene("tiny")),
    "ragged": lambda: (_ragged_cam(), make_scene("tiny", n=1537, seed=9)),
    "student3k": lambda: _student_subset(3000),
}


# ------------------------------------------------------------------ project
VARIANTS = (G.GS_FLAG_ANTIALIASED | G.GS_FLAG_RADII_AXIS | G.GS_FLAG_RADII_OPACITY | G.GS_FLAG_CAP_0999 |
            G.GS_FLAG_STOP_INCLUSIVE)


@pytest.mark.parametrize("flags", [0, G.GS_FLAG_TIGHT_TILES, VARIANTS, VARIANTS | G.GS_FLAG_TIGHT_TILES])
@pytest.mark.parametrize("scene", list(SCENES))
def test_project_matches_oracle(scene, flags):
    cam, params = SCENES[scene]()
    cam.flags = flags
    n = params["means"].shape[0]
    proj = G.Projected(n)
    G.gs_project(cam, cuda_params(params), proj)
    torch.cuda.synchronize()
    p = O.project(params, cam)
    xyod = proj.xy_opacity_depth.cpu().numpy().astype(np.float64)
    conr = proj.conic_radius.cpu().numpy().astype(np.float64)
    rgb = proj.rgb.cpu().numpy()
    rect = proj.rect.cpu().numpy()
    count = proj.count.cpu().numpy()
    v = p["valid"].astype(bool)
    np.testing.assert_array_equal(rgb[:, :3], params["colors"])
    np.testing.assert_allclose(xyod[:, 3], p["depth"], rtol=1e-6, atol=1e-6)
    np.testing.assert_allclose(xyod[:, 2], p["opacity"], rtol=1e-6, atol=1e-7)
    np.testing.assert_allclose(xyod[v, :2], p["mean2d"][v], rtol=2e-6, atol=2e-3)
    scale = np.maximum(np.abs(p["conic"][v, 0]), np.abs(p["conic"][v, 2]))[:, None]
    assert np.all(np.abs(conr[v, :3] - p["conic"][v]) <= 1e-4 * scale + 1e-9)
    # integer decisions: equal unless the oracle says the decision was within
    # its stated margin of flipping
    amb = v & ((p["radius_margin"] < MARGIN_RADIUS) | (p["rect_margin"] < MARGIN_TILE) |
               (p["cut_margin"] < MARGIN_CUT))
    diff_r = conr[:, 3] != p["radius"]
    diff_rect = np.any(rect != p["rect"], axis=1) | (count != p["count"])
    assert not np.any(diff_r & ~amb), np.nonzero(diff_r & ~amb)[0][:10]
    assert not np.any(diff_rect & ~amb), np.nonzero(diff_rect & ~amb)[0][:10]
    assert amb.sum() <= max(10, 1e-2 * n)


# ---------------------------------------------------- bin and sort (stage-fed)
def _check_bins(cam, rec, n, bins, K, ob=None):
    if ob is None:
        ob = O.bin_pairs(rec["rect"], rec["valid"], rec["depth32"], cam.width, cam.height)
    assert K == ob["n_pairs"]
    tile = bins.pair_tile[:K].cpu().numpy().astype(np.uint32)
    gid = bins.pair_gid[:K].cpu().numpy().astype(np.uint32)
    np.testing.assert_array_equal(tile.astype(np.uint64), ob["keys"] >> np.uint64(32))
    np.testing.assert_array_equal(gid, ob["gids"])
    # the 64-bit keys of the emitted pairs: tile << 32 | depth bits
    key = (tile.astype(np.uint64) << np.uint64(32)) | rec["depth32"].view(np.uint32)[gid].astype(np.uint64)
    np.testing.assert_array_equal(key, ob["keys"])
    np.testing.assert_array_equal(bins.ranges.cpu().numpy().astype(np.uint32)[:cam.tiles], ob["ranges"])
    assert int(bins.status.item()) == 0


STRATEGIES = [G.GS_BIN_PER_TILE, G.GS_BIN_GLOBAL]


@pytest.mark.parametrize("strategy", STRATEGIES)
@pytest.mark.parametrize("scene", list(SCENES))
def test_bin_and_sort_bit_exact(scene, strategy):
    cam, params = SCENES[scene]()
    n = params["means"].shape[0]
    rec = oracle_records(params, cam)
    proj = fill_projected(rec, n)
    bins, K = gpu_bin(cam, n, proj, strategy=strategy)
    _check_bins(cam, rec, n, bins, K)


@pytest.mark.parametrize("strategy", STRATEGIES)
def test_bin_and_sort_depth_ties_and_many_partitions(strategy):
    """Equal depth keys keep Gaussian-id order; N spans several sort and scan
    partitions with a ragged last one."""
    cam, params = _student_subset(30_000)
    n = 30_000
    rec = oracle_records(params, cam)
    rec["depth32"] = (np.round(rec["depth32"] * 4) / 4).astype(np.float32)
    proj = fill_projected(rec, n)
    bins, K = gpu_bin(cam, n, proj, strategy=strategy)
    _check_bins(cam, rec, n, bins, K)


@pytest.mark.parametrize("strategy", STRATEGIES)
@pytest.mark.parametrize("W,H", [(16, 16), (1, 1), (17, 1), (4112, 4112)])
def test_bin_and_sort_tile_bit_widths(W, H, strategy):
    """One tile, 1 x 2 tiles, and 257 x 257 tiles (66049: the count matrix
    then takes fewer CTAs and rows longer than shared memory)."""
    cam = Camera(np.eye(4), W * 0.5, W * 0.5, W / 2.0, H / 2.0, W, H)
    rng = np.random.default_rng(W + H)
    n = 700
    params = {"means": np.column_stack([rng.uniform(-1, 1, n), rng.uniform(-1, 1, n), rng.uniform(2, 4, n)]),
              "log_scales": rng.normal(-2.5, 0.7, (n, 3)), "quats": rng.normal(size=(n, 4)),
              "opacity_logits": rng.normal(0, 1, n), "colors": rng.uniform(0, 1, (n, 3))}
    rec = oracle_records(params, cam)
    proj = fill_projected(rec, n)
    bins, K = gpu_bin(cam, n, proj, max_pairs=max(int(rec["count"].sum()), n) + 16, strategy=strategy)
    _check_bins(cam, rec, n, bins, K)


@pytest.mark.parametrize("strategy", STRATEGIES)
@pytest.mark.parametrize("n", [900, 5000, 20000])
def test_bin_and_sort_long_tile_lists(n, strategy):
    """Every Gaussian covers the few tiles of a 48 x 32 image, so each tile's
    list has about n entries: the shared-memory sort of short and of long
    lists, and the global-memory sort beyond 16384 entries; a quarter of the
    depths tie."""
    cam = Camera(np.eye(4), 20.0, 20.0, 24.0, 16.0, 48, 32)
    rng = np.random.default_rng(n)
    params = {"means": np.column_stack([rng.uniform(-.3, .3, n), rng.uniform(-.3, .3, n), rng.uniform(2, 4, n)]),
              "log_scales": rng.normal(-0.5, 0.2, (n, 3)), "quats": rng.normal(size=(n, 4)),
              "opacity_logits": rng.normal(0, 1, n), "colors": rng.uniform(0, 1, (n, 3))}
    rec = oracle_records(params, cam)
    tie = rng.random(n) < 0.25
    rec["depth32"] = np.where(tie, np.float32(3.0), rec["depth32"]).astype(np.float32)
    proj = fill_projected(rec, n)
    bins, K = gpu_bin(cam, n, proj, max_pairs=int(rec["count"].sum()) + 16, strategy=strategy)
    r = bins.ranges.cpu().numpy()[:cam.tiles]
    assert (r[:, 1] - r[:, 0]).max() > 0.8 * n
    _check_bins(cam, rec, n, bins, K)


@pytest.mark.parametrize("strategy", STRATEGIES)
def test_bin_and_sort_capacity_error_and_async_status(strategy):
    cam, params = SCENES["tiny"]()
    n = params["means"].shape[0]
    rec = oracle_records(params, cam)
    need = int(rec["count"].sum())
    proj = fill_projected(rec, n)
    bins = G.Bins(n, need - 1, cam.width, cam.height, strategy=strategy)
    with pytest.raises(G.GSError) as ei:
        G.gs_bin_and_sort(cam, n, proj, bins, sync=True)
    assert ei.value.code == G.GS_ERR_CAPACITY and ei.value.n_pairs == need
    # asynchronous mode: nothing raised, the status word says so, ranges are
    # empty, and the render draws background only
    G.gs_bin_and_sort(cam, n, proj, bins, sync=False)
    st, K = G.gs_read_status(bins)
    assert st == G.GS_ERR_CAPACITY and K == need
    assert int(bins.ranges.abs().sum().item()) == 0
    image, T, _ = gpu_render(cam, n, proj, bins)
    assert torch.all(image == 0) and torch.all(T == 1)
    # regrown to the reported need, the same call succeeds
    bins2 = G.Bins(n, need, cam.width, cam.height)
    assert G.gs_bin_and_sort(cam, n, proj, bins2) == need


@pytest.mark.parametrize("depth", [False, True])
@pytest.mark.parametrize("scene", ["tiny", "ragged", "student3k"])
def test_render_fwd_l1_equals_forward_then_l1(scene, depth):
    """gs_render_fwd_l1 (the L1 loss in the forward's epilogue) writes the
    image, T, last and dL/dimage of gs_render_fwd followed by
    gs_l1_loss_grad bit for bit; the loss (summed per CTA instead of per
    thread block of values) agrees to rounding, and is zeroed first."""
    cam, params = SCENES[scene]()
    if depth:
        cam.flags |= G.GS_FLAG_DEPTH
    n = params["means"].shape[0]
    P = cuda_params(params)
    r = G.Rasterizer(n, cam.width, cam.height)
    image = r.forward(cam, P).clone()
    T, last = r.T_final.clone(), r.last.clone()
    ch = G.channels(cam)
    target = torch.from_numpy(make_target(cam.width, cam.height, channels=ch)).cuda()
    dl_ref = torch.empty_like(image)
    loss_ref = torch.zeros(1, device="cuda")
    G.gs_l1_loss_grad(image, target, dl_ref, loss_ref)
    img2, T2, last2, dl2 = (torch.full_like(x, 7) for x in (image, T, last, dl_ref))
    loss2 = torch.full((1,), 7.0, device="cuda")
    G.gs_render_fwd_l1(cam, n, r.proj, r.bins, img2, T2, last2, target, dl2, loss2)
    torch.cuda.synchronize()
    assert torch.equal(img2, image) and torch.equal(T2, T) and torch.equal(last2, last)
    assert torch.equal(dl2, dl_ref)
    assert abs(loss2.item() - loss_ref.item()) <= 1e-6 * max(1.0, loss_ref.item())
    dl3 = torch.full_like(dl_ref, 7)
    G.gs_render_fwd_l1(cam, n, r.proj, r.bins, img2, T2, last2, target, dl3, None)  # no loss wanted
    torch.cuda.synchronize()
    assert torch.equal(dl3, dl_ref)


@pytest.mark.parametrize("count,offset", [(4 * 100_003, 0), (4 * 100_003 + 3, 0), (4 * 100_003, 1)])
def test_l1_loss_grad_sizes_and_offsets(count, offset):
    """gs_l1_loss_grad against the oracle's loss and gradient: a count that is
    a multiple of 4 with aligned arrays, a ragged count, and arrays offset by
    one float.  Values are multiples of 1/64, so image - target is exact in
    fp32 and its sign is unambiguous (zeros included)."""
    rng = np.random.default_rng(count + offset)
    img = rng.integers(-64, 64, count).astype(np.float32) / 64
    tgt = rng.integers(-64, 64, count).astype(np.float32) / 64
    buf = torch.empty(3 * (count + 4), device="cuda")
    base = lambda k: buf[k * (count + 4) + offset:k * (count + 4) + offset + count]
    image, target, dl = base(0), base(1), base(2)
    image.copy_(torch.from_numpy(img))
    target.copy_(torch.from_numpy(tgt))
    loss = torch.zeros(1, device="cuda")
    G.gs_l1_loss_grad(image, target, dl, loss)
    torch.cuda.synchronize()
    loss_ref, dl_ref = OT.l1_loss_grad(img, tgt)
    np.testing.assert_allclose(dl.cpu().numpy().astype(np.float64), dl_ref, rtol=1e-7, atol=0)
    assert abs(loss.item() - loss_ref) <= 1e-5 * max(loss_ref, 1.0)


def test_argument_errors_launch_nothing():
    cam = tiny_camera()
    proj = G.Projected(10)
    bins = G.Bins(10, 100, cam.width, cam.height)
    bad = tiny_camera()
    bad.near_z = 0.0
    with pytest.raises(G.GSError) as ei:
        G.gs_bin_and_sort(bad, 10, proj, bins)
    assert ei.value.code == G.GS_ERR_INVALID_ARG
    with pytest.raises(G.GSError) as ei:
        G.gs_bin_and_sort(cam, 11, proj, bins)  # more Gaussians than carved for
    assert ei.value.code == G.GS_ERR_INVALID_ARG
    big = tiny_camera(512, 512)
    with pytest.raises(G.GSError):
        G.gs_render_fwd(big, 10, proj, bins, torch.empty(512, 512, 3, device="cuda"),
                        torch.empty(512, 512, device="cuda"),
                        torch.empty(512, 512, dtype=torch.int32, device="cuda"))


# ------------------------------------------------------- forward (stage-fed)
def _fwd_stage_fed(cam, params, tile_mask=None):
    n = params["means"].shape[0]
    rec = oracle_records(params, cam)
    proj = fill_projected(rec, n)
    bins, K = gpu_bin(cam, n, proj)
    image, T, last = gpu_render(cam, n, proj, bins)
    ref = O.render(rec, cam, tile_mask=tile_mask)
    return rec, proj, bins, K, image.cpu().numpy(), T.cpu().numpy(), last.cpu().numpy(), ref


def _assert_fwd(cam, bins, image, T, last, ref, sel):
    """Every selected pixel matches (image and T within 1e-4, the same last
    entry) unless one of its threshold decisions sat within the stated margin
    of flipping; such actual flips must be rare."""
    amb = ambiguous_pixels(ref) & sel
    check_ambiguous(amb, sel, "forward")
    d_img = np.abs(image - ref["image"]).max(axis=2)
    d_T = np.abs(T - ref["T_final"])
    ranges = bins.ranges.cpu().numpy()
    ty, tx = np.mgrid[0:cam.height, 0:cam.width]
    start = ranges[(ty // 16) * cam.tiles_x + tx // 16, 0]
    differs = sel & ((d_img > IMG_TOL) | (d_T > IMG_TOL) | ((last - start) != ref["n_walk"]))
    unexplained = differs & ~amb
    assert not unexplained.any(), (f"{int(unexplained.sum())} pixels differ away from any threshold; max "
                                   f"|d image| {d_img[unexplained].max():.3e}")
    report("forward", flipped_pixels=int(differs.sum()), max_abs_image_diff=f"{float(d_img[sel & ~amb].max(initial=0)):.2e}")
    assert differs.sum() <= max(2, 1e-4 * sel.sum()), f"{int(differs.sum())} flipped pixels"
    assert np.all(np.isfinite(image)) and np.all(T > 0) and np.all(T <= 1)


@pytest.mark.parametrize("scene", list(SCENES))
def test_render_fwd_matches_oracle(scene):
    cam, params = SCENES[scene]()
    rec, proj, bins, K, image, T, last, ref = _fwd_stage_fed(cam, params)
    _assert_fwd(cam, bins, image, T, last, ref, np.ones((cam.height, cam.width), bool))


def test_render_fwd_student_sampled_tiles():
    """The 30k-Gaussian student at 980 x 545 on 120 sampled tiles."""
    cam, params = _student_subset(30_000)
    rng = np.random.default_rng(0)
    mask = np.zeros(cam.tiles, np.uint8)
    mask[rng.choice(cam.tiles, 120, replace=False)] = 1
    mask[-1] = 1  # ragged corner tile
    rec, proj, bins, K, image, T, last, ref = _fwd_stage_fed(cam, params, tile_mask=mask)
    sel = tiles_to_pixels(mask.reshape(cam.tiles_y, cam.tiles_x).astype(bool), cam)
    _assert_fwd(cam, bins, image, T, last, ref, sel)


@pytest.mark.parametrize("scene", ["ragged", "student3k"])
def test_render_stats_match_oracle_counts(scene):
    """gs_render_stats counts the work the method must do: entries visited up
    to and including each pixel's stopping entry, entries added, and the
    backward's walk [start, last).  The oracle counts the same per pixel;
    pixels whose decisions sit within the stated margins may differ."""
    cam, params = SCENES[scene]()
    rec, proj, bins, K, image, T, last, ref = _fwd_stage_fed(cam, params)
    n = params["means"].shape[0]
    st = G.gs_render_stats(cam, n, proj, bins, torch.from_numpy(last).cuda())
    amb = ambiguous_pixels(ref)
    slack = int(ref["e_visit"][amb].sum()) + int(amb.sum())
    assert st["pixels"] == cam.width * cam.height
    assert abs(st["fwd_visits"] - int(ref["e_visit"].sum())) <= slack
    assert abs(st["contributions"] - int(ref["e_contrib"].sum())) <= slack
    assert abs(st["bwd_visits"] - int(ref["n_walk"].sum())) <= slack
    assert st["contributions"] > 0 and st["fwd_visits"] >= st["contributions"]


def test_render_fwd_background_and_white_invariant():
    cam, params = SCENES["ragged"]()
    cam.bg = (0.2, 0.4, 0.6)
    params = dict(params)
    params["colors"] = np.ones_like(params["colors"])
    rec, proj, bins, K, image, T, last, ref = _fwd_stage_fed(cam, params)
    _assert_fwd(cam, bins, image, T, last, ref, np.ones((cam.height, cam.width), bool))
    # white splats: C = 1 - T, so image = (1 - T) + T bg
    np.testing.assert_allclose(image, (1 - T)[..., None] + T[..., None] * np.array(cam.bg), atol=2e-6)


# ------------------------------------------------------ backward (stage-fed)
def _bwd_stage_fed(cam, params, seed=0, tile_mask=None):
    n = params["means"].shape[0]
    rec, proj, bins, K, image, T, last, ref = _fwd_stage_fed(cam, params, tile_mask=tile_mask)
    rng = np.random.default_rng(seed)
    dl = rng.normal(size=(cam.height, cam.width, G.channels(cam)))
    sel = np.ones((cam.height, cam.width), bool)
    if tile_mask is not None:
        sel = tiles_to_pixels(tile_mask.reshape(cam.tiles_y, cam.tiles_x).astype(bool), cam)
    amb = ambiguous_pixels(ref, with_clamp=True)
    check_ambiguous(amb, sel, "backward (dL/dimage zeroed)")
    keep = sel & ~amb
    dl = np.where(keep[..., None], dl, 0.0).astype(np.float32)
    P = cuda_params(params)
    grads = {k: torch.full_like(v, float("nan")) for k, v in P.items()}
    grad2d = torch.full((n, 12), float("nan"), device="cuda")
    G.gs_render_bwd(cam, n, P, proj, bins, torch.from_numpy(T).cuda(), torch.from_numpy(last).cuda(),
                    torch.from_numpy(dl).cuda(), grad2d, grads)
    torch.cuda.synchronize()
    assert int(bins.status.item()) == 0  # a checked build records an index out of range here
    g2_ref, g2_abs = O.render_bwd(rec, cam, dl.astype(np.float64), tile_mask=tile_mask)
    return rec, grad2d.cpu().numpy(), {k: v.cpu().numpy() for k, v in grads.items()}, g2_ref, g2_abs, params


@pytest.mark.parametrize("scene", list(SCENES))
def test_render_bwd_matches_oracle(scene):
    cam, params = SCENES[scene]()
    rec, g2, grads, g2_ref, g2_abs, params = _bwd_stage_fed(cam, params)
    assert np.all(g2[:, 9:] == 0)
    grad_compare(g2[:, :g2_ref.shape[1]], g2_ref, g2_abs, "grad2d")
    raw_ref = O.project_bwd(params, cam, g2_ref)
    bound = O.grad_bound(params, cam, g2_abs)
    for k in G.PARAM_KEYS:
        grad_compare(grads[k], raw_ref[k], bound[k], k)
        assert np.all(np.isfinite(grads[k]))


def test_render_bwd_student_sampled_tiles():
    cam, params = _student_subset(30_000)
    rng = np.random.default_rng(1)
    mask = np.zeros(cam.tiles, np.uint8)
    mask[rng.choice(cam.tiles, 80, replace=False)] = 1
    rec, g2, grads, g2_ref, g2_abs, params = _bwd_stage_fed(cam, params, tile_mask=mask)
    grad_compare(g2[:, :g2_ref.shape[1]], g2_ref, g2_abs, "grad2d")
    raw_ref = O.project_bwd(params, cam, g2_ref)
    bound = O.grad_bound(params, cam, g2_abs)
    for k in G.PARAM_KEYS:
        grad_compare(grads[k], raw_ref[k], bound[k], k)


# --------------------------------------------- opacity-aware tile cut
@pytest.mark.parametrize("scene", ["ragged", "student3k"])
def test_tight_tiles_stage_fed(scene):
    """Forward and backward on the oracle's cut rectangles."""
    cam, params = SCENES[scene]()
    cam.flags = G.GS_FLAG_TIGHT_TILES
    rec, proj, bins, K, image, T, last, ref = _fwd_stage_fed(cam, params)
    _assert_fwd(cam, bins, image, T, last, ref, np.ones((cam.height, cam.width), bool))
    rec, g2, grads, g2_ref, g2_abs, params = _bwd_stage_fed(cam, params)
    grad_compare(g2[:, :g2_ref.shape[1]], g2_ref, g2_abs, "grad2d")
    raw_ref = O.project_bwd(params, cam, g2_ref)
    bound = O.grad_bound(params, cam, g2_abs)
    for k in G.PARAM_KEYS:
        grad_compare(grads[k], raw_ref[k], bound[k], k)


@pytest.mark.parametrize("flags", [G.GS_FLAG_CAP_0999 | G.GS_FLAG_STOP_INCLUSIVE, VARIANTS, G.GS_FLAG_DEPTH,
                                   VARIANTS | G.GS_FLAG_DEPTH | G.GS_FLAG_TIGHT_TILES])
def test_variants_stage_fed(flags):
    """The pages' variants (antialiased compensation, gsplat radii, inclusive
    stop test, 0.999 cap): forward and backward on the oracle's records."""
    cam, params = SCENES["student3k"]()
    cam.flags = flags
    rec, proj, bins, K, image, T, last, ref = _fwd_stage_fed(cam, params)
    _assert_fwd(cam, bins, image, T, last, ref, np.ones((cam.height, cam.width), bool))
    rec, g2, grads, g2_ref, g2_abs, params = _bwd_stage_fed(cam, params)
    grad_compare(g2[:, :g2_ref.shape[1]], g2_ref, g2_abs, "grad2d")
    raw_ref = O.project_bwd(params, cam, g2_ref)
    bound = O.grad_bound(params, cam, g2_abs)
    for k in G.PARAM_KEYS:
        grad_compare(grads[k], raw_ref[k], bound[k], k)


def test_tight_tiles_leave_image_and_gradients_unchanged():
    """The 30k student at 980 x 545 through the CUDA path with and without
    the cut: the same entries pass the alpha test in the same order, so the
    image and transmittance are equal bit for bit, with fewer pairs."""
    cam, params = _student_subset(30_000)
    n = params["means"].shape[0]
    P = cuda_params(params)
    target = torch.from_numpy(make_target(cam.width, cam.height)).cuda()
    out = {}
    for flags in (0, G.GS_FLAG_TIGHT_TILES):
        cam.flags = flags
        r = G.Rasterizer(n, cam.width, cam.height)
        image = r.forward(cam, P).clone()
        T = r.T_final.clone()
        dl = torch.empty_like(image)
        G.gs_l1_loss_grad(image, target, dl, torch.zeros(1, device="cuda"))
        grads = {k: v.clone() for k, v in r.backward(cam, P, dl).items()}
        torch.cuda.synchronize()
        out[flags] = (image.cpu().numpy(), T.cpu().numpy(), grads, r.n_pairs)
    (i0, t0, g0, k0), (i1, t1, g1, k1) = out[0], out[G.GS_FLAG_TIGHT_TILES]
    assert k1 < 0.85 * k0
    np.testing.assert_array_equal(i1, i0)
    np.testing.assert_array_equal(t1, t0)
    for k in G.PARAM_KEYS:  # same sums, atomics in another order
        a, b = g1[k].cpu().numpy(), g0[k].cpu().numpy()
        assert np.abs(a - b).max() <= 1e-5 * max(np.abs(b).max(), 1e-30), k


# ------------------------------------------------------------ end to end
def _without_ambiguous(params, cam):
    """The scene with every Gaussian whose projection sits within the stated
    margin of an integer decision (radius ceiling, tile edge, depth order)
    moved behind the camera, so that fp32 and fp64 bin it the same way."""
    p = O.project(params, cam)
    bad = ambiguous_gaussians(p)
    out = {k: v.copy() for k, v in params.items()}
    out["means"][bad] = np.linalg.inv(cam.viewmat.astype(np.float64))[:3, :3] @ [0.0, 0.0, -50.0] + \
        np.linalg.inv(cam.viewmat.astype(np.float64))[:3, 3]
    return out, int(bad.sum())


@pytest.mark.parametrize("flags", [0, G.GS_FLAG_TIGHT_TILES, VARIANTS, VARIANTS | G.GS_FLAG_DEPTH])
def test_end_to_end_from_raw_parameters(flags):
    """Raw parameters through all four calls vs the oracle from the same raw
    parameters in double precision, L1 loss against a seeded target."""
    cam, params = SCENES["ragged"]()
    cam.flags = flags
    params, removed = _without_ambiguous(params, cam)
    assert removed <= 20
    n = params["means"].shape[0]
    P = cuda_params(params)
    r = G.Rasterizer(n, cam.width, cam.height)
    image = r.forward(cam, P).clone()
    tgt = make_target(cam.width, cam.height)
    if G.channels(cam) == 4:  # a target depth channel as well
        tgt = np.concatenate([tgt, np.random.default_rng(5).uniform(2, 5, tgt.shape[:2] + (1,))], axis=2)
    target = torch.from_numpy(np.ascontiguousarray(tgt, np.float32)).cuda()
    dl = torch.empty_like(image)
    loss = torch.zeros(1, device="cuda")
    G.gs_l1_loss_grad(image, target, dl, loss)
    torch.cuda.synchronize()
    p = O.project(params, cam)
    assert not ambiguous_gaussians(p).any()
    ref = O.render(p, cam)
    amb = ambiguous_pixels(ref, with_clamp=True)
    check_ambiguous(amb, np.ones_like(amb), "end to end")
    sel = ~amb
    img = image.cpu().numpy()
    assert np.abs(img - ref["image"]).max(axis=2)[sel].max() <= IMG_TOL
    tgt = target.cpu().numpy().astype(np.float64)
    # the L1 gradient of each side from its own image; pixels whose sign of
    # image - target the fp32 image could flip are masked out with the
    # ambiguous ones
    loss_ref, dl_ref = OT.l1_loss_grad(ref["image"], tgt)
    assert abs(loss.item() - loss_ref) <= 1e-5
    sign_amb = (np.abs(ref["image"] - tgt) <= IMG_TOL).any(axis=2) & sel
    # |image - target| <= 1e-4 in one of three channels: about 6e-4 of the
    # pixels for a U(0, 1) target
    report("end to end", l1_sign_ambiguous_pixels=int(sign_amb.sum()), pixels=sel.size)
    assert sign_amb.sum() <= 2e-3 * sel.size
    sel &= ~sign_amb
    dl_gpu = dl.cpu().numpy().astype(np.float64)
    np.testing.assert_allclose(dl_gpu[sel], dl_ref[sel], rtol=1e-7, atol=0)
    dlm = torch.where(torch.from_numpy(sel[..., None]).cuda(), dl, torch.zeros_like(dl))
    grads = r.backward(cam, P, dlm)
    torch.cuda.synchronize()
    g2_ref, g2_abs = O.render_bwd(p, cam, np.where(sel[..., None], dl_ref, 0.0))
    raw_ref = O.project_bwd(params, cam, g2_ref)
    bound = O.grad_bound(params, cam, g2_abs)
    for k in G.PARAM_KEYS:
        grad_compare(grads[k].cpu().numpy(), raw_ref[k], bound[k], k)


# --------------------------------------------------------------- edge cases
def test_empty_scene_renders_background():
    cam = tiny_camera(40, 24, bg=(0.1, 0.2, 0.3))
    r = G.Rasterizer(0, cam.width, cam.height)
    P = {k: torch.zeros((0,) + s, device="cuda") for k, s in
         (("means", (3,)), ("log_scales", (3,)), ("quats", (4,)), ("opacity_logits", ()), ("colors", (3,)))}
    img = r.forward(cam, P)
    torch.cuda.synchronize()
    assert r.n_pairs == 0
    np.testing.assert_array_equal(img.cpu().numpy(), np.broadcast_to(np.float32([0.1, 0.2, 0.3]), (24, 40, 3)))
    grads = r.backward(cam, P, torch.ones_like(img))
    assert all(v.numel() == 0 for v in grads.values())


def test_culled_nan_and_zero_quaternion_inputs():
    """Gaussians behind the camera, on the near plane, with a NaN parameter
    or a non-finite colour: no tiles, exactly zero gradient, and the others are unaffected.  A zero
    quaternion renders as the identity rotation."""
    cam = tiny_camera(64, 48, 60.0)
    rng = np.random.default_rng(4)
    n = 40
    params = {"means": np.column_stack([rng.uniform(-.5, .5, n), rng.uniform(-.5, .5, n), rng.uniform(-.5, .5, n)]),
              "log_scales": rng.normal(-2.3, 0.3, (n, 3)), "quats": rng.normal(size=(n, 4)),
              "opacity_logits": rng.normal(0, 1, n), "colors": rng.uniform(0, 1, (n, 3))}
    params["means"][0, 2] = -4.0            # z_cam = 0: culled
    params["means"][1, 2] = -10.0           # behind the camera
    params["means"][2] = [0.3, 0.3, -3.995]  # in front of the near plane
    params["log_scales"][3, 1] = np.nan     # NaN parameter
    params["quats"][4] = 0.0                # zero quaternion
    params["colors"][5, 2] = np.inf         # non-finite colour
    params = {k: v.astype(np.float32) for k, v in params.items()}
    P = cuda_params(params)
    r = G.Rasterizer(n, cam.width, cam.height)
    r.forward(cam, P)
    cnt = r.proj.count.cpu().numpy()
    assert cnt[0] == 0 and cnt[1] == 0 and cnt[2] == 0 and cnt[3] == 0 and cnt[4] > 0 and cnt[5] == 0
    grads = r.backward(cam, P, torch.ones(cam.height, cam.width, 3, device="cuda"))
    torch.cuda.synchronize()
    for k, v in grads.items():
        v = v.cpu().numpy()
        assert np.all(np.isfinite(v)), k
        assert np.all(v[:4] == 0) and np.all(v[5] == 0), k
    p = O.project(params, cam)
    assert p["count"][:4].tolist() == [0, 0, 0, 0] and p["count"][5] == 0
    assert np.all(np.isfinite(r.image.cpu().numpy()))


def test_huge_splat_covers_every_tile():
    cam = _ragged_cam()
    params = {"means": np.zeros((2, 3), np.float32), "log_scales": np.full((2, 3), 1.0, np.float32),
              "quats": np.tile(np.float32([1, 0, 0, 0]), (2, 1)), "opacity_logits": np.float32([2.0, -1.0]),
              "colors": np.float32([[1, 0, 0], [0, 1, 0]])}
    rec = oracle_records(params, cam)
    assert rec["count"][0] == cam.tiles
    proj = fill_projected(rec, 2)
    bins, K = gpu_bin(cam, 2, proj)
    _check_bins(cam, rec, 2, bins, K)
    image, T, last = gpu_render(cam, 2, proj, bins)
    ref = O.render(rec, cam)
    _assert_fwd(cam, bins, image.cpu().numpy(), T.cpu().numpy(), last.cpu().numpy(), ref,
                np.ones((cam.height, cam.width), bool))


def test_saturating_stack_terminates_early():
    """Many opaque splats: every pixel stops at T < 1e-4 long before the end
    of its list, as in the pages' termination example."""
    cam = tiny_camera(48, 40, 60.0)
    n = 300
    rng = np.random.default_rng(8)
    params = {"means": np.column_stack([rng.uniform(-.2, .2, n), rng.uniform(-.2, .2, n), rng.uniform(-.5, .5, n)]),
              "log_scales": np.full((n, 3), -0.5), "quats": rng.normal(size=(n, 4)),
              "opacity_logits": np.full(n, 3.0), "colors": rng.uniform(0, 1, (n, 3))}
    params = {k: v.astype(np.float32) for k, v in params.items()}
    rec, proj, bins, K, image, T, last, ref = _fwd_stage_fed(cam, params)
    _assert_fwd(cam, bins, image, T, last, ref, np.ones((cam.height, cam.width), bool))
    assert (ref["e_visit"] < n).mean() > 0.75 and (T < 1e-3).mean() > 0.75
