"""Pins of the oracle's opacity-aware tile cut ("Gaussian splatting in
PyTorch", s4 "The low-pass filter, the conic and the radius": gsplat's extent
of sqrt(2 ln(255 o)) standard deviations, beyond which a splat has faded
below 1/255).

The cut narrows each tile rectangle to the columns and rows in which some
pixel centre can still reach alpha >= 1/255.  What pins it, independently of
its own formula:
  * a hand-worked axis-aligned case (the bounds written out below);
  * brute force over pixels: every tile the cut removes has alpha < 1/255 at
    all of its pixel centres, and the cut rectangle lies inside the 3-sigma
    one;
  * the rendered image, final transmittance and gradients are the same with
    and without the cut, bit for bit, while the pair count drops.
"""
import math

import numpy as np

import oracle as O
from scenes import make_cameras, make_scene, tiny_camera

W, H = 980, 545  # 62 x 35 tiles


def _rects(mean2d, radius, conic, opacity, tight=True, width=W, height=H):
    n = len(radius)
    return O.tile_rects(np.asarray(mean2d, np.float32).reshape(n, 2), np.asarray(radius, np.float32),
                        np.ones(n, np.uint8), width, height,
                        np.asarray(conic, np.float32).reshape(n, 3),
                        np.asarray(opacity, np.float32), tight)


def test_axis_aligned_hand_worked_bounds():
    # Sigma'' = diag(10^2, 4^2): conic (1/100, 0, 1/16), o = 0.5, centre
    # (100.3, 60.7), radius 64 (so the 3-sigma rectangle is tiles x 2..10,
    # y 0..7).  ell = ln(127.5) + 0.01 = 4.858116; sqrt(2 ell) = 3.117087;
    # D_x = 10 * 3.117087 = 31.1709, D_y = 4 * 3.117087 = 12.4683.
    #   x: ceil((100.3 - 31.1709 - 15.5) / 16) = ceil(3.3518) = 4,
    #      floor((100.3 + 31.1709 - 0.5) / 16) = floor(8.1857) = 8
    #   y: ceil((60.7 - 12.4683 - 15.5) / 16) = ceil(2.0457) = 3,
    #      floor((60.7 + 12.4683 - 0.5) / 16) = floor(4.5418) = 4
    rect, count = _rects([100.3, 60.7], [64.0], [0.01, 0.0, 1.0 / 16], [0.5])
    assert rect[0].tolist() == [4, 3, 8, 4] and count[0] == 10
    rect3, count3 = _rects([100.3, 60.7], [64.0], [0.01, 0.0, 1.0 / 16], [0.5], tight=False)
    assert rect3[0].tolist() == [2, 0, 10, 7] and count3[0] == 72
    # at mx = 113.13: mx + D_x = 144.30, so column 9 (nearest centre 144.5)
    # is out and column 8 (nearest centre 143.5) in: x = ceil(4.154) = 5 ..
    # floor((144.30 - 0.5) / 16) = floor(8.9875) = 8
    rect, count = _rects([113.13, 60.7], [64.0], [0.01, 0.0, 1.0 / 16], [0.5])
    assert rect[0].tolist() == [5, 3, 8, 4] and count[0] == 8
    # the kept edge column 4 reaches alpha = 0.5 exp(-(20.8^2/100 + 0.2^2/16)/2)
    # = 0.0574 at pixel (79.5, 60.5); the cut column 3 peaks at pixel
    # (63.5, 60.5) with 0.5 exp(-(36.8^2/100 + 0.04/16)/2) = 5.7e-4 < 1/255
    assert 0.5 * math.exp(-0.5 * (20.8 ** 2 / 100 + 0.2 ** 2 / 16)) > 1 / 255
    assert 0.5 * math.exp(-0.5 * (36.8 ** 2 / 100 + 0.2 ** 2 / 16)) < 1 / 255


def test_faint_splats_touch_nothing():
    # ell = ln(255 o) + 0.01 <= 0 iff o <= e^-0.01 / 255 = 0.0038826
    rect, count = _rects([[100.0, 100.0]] * 2, [30.0, 30.0], [[0.01, 0.0, 0.01]] * 2, [0.0038, 0.0040])
    assert count.tolist()[0] == 0 and count.tolist()[1] > 0
    assert rect[0, 0] > rect[0, 2] or rect[0, 1] > rect[0, 3]


def test_ill_conditioned_conic_keeps_the_three_sigma_rectangle():
    # a 45-degree needle with eigenvalues 3e3 and 0.3: A C / (A C - B^2) > 1024
    lam1, lam2, th = 3e3, 0.3, math.pi / 4
    c, s = math.cos(th), math.sin(th)
    a = lam1 * c * c + lam2 * s * s
    b = (lam1 - lam2) * c * s
    cc = lam1 * s * s + lam2 * c * c
    det = a * cc - b * b
    conic = [cc / det, -b / det, a / det]
    cond = conic[0] * conic[2] / (conic[0] * conic[2] - conic[1] ** 2)
    assert cond > 1024
    r = math.ceil(3 * math.sqrt(lam1))
    args = ([[500.0, 270.0]], [float(r)], [conic], [0.02])
    np.testing.assert_array_equal(_rects(*args)[0], _rects(*args, tight=False)[0])
    # the same needle at half the length is cut
    lam1 = 3e2
    a, b, cc = lam1 * c * c + lam2 * s * s, (lam1 - lam2) * c * s, lam1 * s * s + lam2 * c * c
    det = a * cc - b * b
    conic = [cc / det, -b / det, a / det]
    args = ([[500.0, 270.0]], [float(math.ceil(3 * math.sqrt(lam1)))], [conic], [0.02])
    assert _rects(*args)[1][0] < _rects(*args, tight=False)[1][0]


def _alpha_max_in_tile(mx, my, A, B, C, o, tx, ty):
    xs = 16 * tx + 0.5 + np.arange(16.0)
    ys = 16 * ty + 0.5 + np.arange(16.0)
    dx = mx - xs[None, :]
    dy = my - ys[:, None]
    sig = 0.5 * (A * dx * dx + C * dy * dy) + B * dx * dy
    return float((o * np.exp(-sig)).max())


def _line_alpha_max(mx, my, A, B, C, o, x):
    """Largest alpha on the vertical line through pixel-centre column x,
    by dense sampling of y (never above the true maximum)."""
    sy = math.sqrt(A / (A * C - B * B))  # standard deviation along y
    ys = my + np.linspace(-4 * sy, 4 * sy, 200001)
    dx, dy = mx - x, my - ys
    return float((o * np.exp(-(0.5 * (A * dx * dx + C * dy * dy) + B * dx * dy))).max())


def _brute_force_check(p, limit):
    v = np.nonzero(p["valid"])[0]
    checked = tight = 0
    for g in v[:limit]:
        x0, y0, x1, y1 = p["rect3"][g]
        a0, b0, a1, b1 = p["rect"][g]
        if p["count"][g] > 0:  # inside the 3-sigma rectangle
            assert x0 <= a0 <= a1 <= x1 and y0 <= b0 <= b1 <= y1
        mx, my = p["mean2d"][g]
        A, B, C = p["conic"][g]
        o = p["opacity"][g]
        for ty in range(y0, y1 + 1):
            for tx in range(x0, x1 + 1):
                kept = p["count"][g] > 0 and a0 <= tx <= a1 and b0 <= ty <= b1
                if not kept:
                    assert _alpha_max_in_tile(mx, my, A, B, C, o, tx, ty) < math.exp(-0.01) / 255
                    checked += 1
        # tight in x: a kept edge column that the cut placed (inside the
        # 3-sigma rectangle and the grid) reaches the cut's threshold on the
        # line through its pixel centre nearest to the mean
        if p["count"][g] > 0 and A * C < 1024 * (A * C - B * B):
            for edge, inner in ((a0, a0 > x0), (a1, a1 < x1)):
                if inner:
                    xc = min(max(mx, 16 * edge + 0.5), 16 * edge + 15.5)
                    assert _line_alpha_max(mx, my, A, B, C, o, xc) >= math.exp(-0.01) / 255 * (1 - 1e-6)
                    tight += 1
    return checked, tight


def _project_both(params, cam):
    cam.flags = 0
    p3 = O.project(params, cam)
    cam.flags = O.TIGHT_TILES
    p = O.project(params, cam)
    p["rect3"], p["count3"] = p3["rect"], p3["count"]
    return p, p3


def test_cut_tiles_hold_no_visible_pixel_random_scenes():
    # anisotropic, rotated splats over a range of sizes and opacities
    cam = make_cameras("student", count=60)[7]
    params = make_scene("student", n=4000, seed=5)
    p, _ = _project_both(params, cam)
    checked, tight = _brute_force_check(p, 1500)
    assert checked > 1000 and tight > 100
    K3, K = int(p["count3"].sum()), int(p["count"].sum())
    assert K < 0.9 * K3
    cam = tiny_camera(200, 150, 180.0, distance=3.0)
    params = make_scene("tiny", n=800, seed=12)
    params["log_scales"] = params["log_scales"] + np.array([1.5, 0.0, -0.5], np.float32)
    p, _ = _project_both(params, cam)
    checked, tight = _brute_force_check(p, 800)
    assert checked > 100 and tight > 20


def test_image_and_gradients_unchanged_by_the_cut():
    cam = tiny_camera(200, 150, 180.0, distance=3.0)
    params = make_scene("tiny", n=1500, seed=21)
    params["opacity_logits"] = np.random.default_rng(3).normal(-1.0, 2.5, 1500).astype(np.float32)
    p, p3 = _project_both(params, cam)
    assert int(p["count"].sum()) < int(p3["count"].sum())
    f = O.render(p, cam)
    f3 = O.render(p3, cam)
    np.testing.assert_array_equal(f["image"], f3["image"])
    np.testing.assert_array_equal(f["T_final"], f3["T_final"])
    np.testing.assert_array_equal(f["e_contrib"], f3["e_contrib"])
    g = np.random.default_rng(4).normal(size=(cam.height, cam.width, 3))
    grad2d, grad_abs = O.render_bwd(p, cam, g)
    grad2d3, grad_abs3 = O.render_bwd(p3, cam, g)
    assert np.abs(grad2d).max() > 0
    np.testing.assert_array_equal(grad2d, grad2d3)
    np.testing.assert_array_equal(grad_abs, grad_abs3)
    # the same holds for records rounded to single precision
    r = O.records_f32(p3, cam.width, cam.height, tight=True)
    r3 = O.records_f32(p3, cam.width, cam.height)
    assert int(r["count"].sum()) < int(r3["count"].sum())
    np.testing.assert_array_equal(O.render(r, cam)["image"], O.render(r3, cam)["image"])
