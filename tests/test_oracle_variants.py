"""Pins of the oracle's variants of the method ("Gaussian splatting in
PyTorch": s4 the gsplat radii and the antialiased compensation, s5 gsplat's
inclusive stop test, s6 the older 0.999 alpha cap), each selected by a camera
flag.  The default (no flag) is the 3DGS method pinned elsewhere."""
import math

import numpy as np

import oracle as O

from test_oracle_pins import _identity_cam, _records


def _one_pixel_cam(flags=0):
    cam = _identity_cam(1, 1, 10.0, 10.0, 0.5, 0.5)
    cam.flags = flags
    return cam


def test_inclusive_stop_test():
    """s5: 3DGS stops when next_T < 1e-4, gsplat when next_T <= 1e-4.  Two
    splats at the pixel centre: the first capped at 0.99, the second's opacity
    chosen so that T (1 - alpha) rounds to exactly 1e-4f; 3DGS adds it,
    gsplat stops before it."""
    a1 = float(np.float32(0.99))
    T1 = 1.0 - a1
    t_min = float(np.float32(1e-4))
    o2 = 1.0 - t_min / T1
    assert np.float32(T1 * (1.0 - o2)) == np.float32(1e-4) and not np.float32(o2) > np.float32(0.99)
    rec = _records([[0.5, 0.5], [0.5, 0.5]], [[1.0, 0.0, 1.0]] * 2, [0.995, o2],
                   [[1.0, 0.0, 0.0], [0.0, 1.0, 0.0]], [1.0, 2.0], [[0, 0, 0, 0]] * 2)
    f3 = O.render(rec, _one_pixel_cam(), nthreads=1)
    fg = O.render(rec, _one_pixel_cam(O.STOP_INCLUSIVE), nthreads=1)
    # 3DGS: both added; gsplat: only the first
    np.testing.assert_allclose(f3["image"][0, 0], [a1, o2 * T1, 0.0], rtol=1e-12)
    np.testing.assert_allclose(fg["image"][0, 0], [a1, 0.0, 0.0], rtol=1e-12)
    assert f3["e_contrib"][0, 0] == 2 and fg["e_contrib"][0, 0] == 1
    assert fg["T_final"][0, 0] == T1


def test_cap_0999():
    """s6: alpha = min(cap, o G) with cap 0.99 (3DGS, current gsplat) or
    0.999 (older gsplat); at the centre G = 1."""
    rec = _records([[0.5, 0.5]], [[1.0, 0.0, 1.0]], [0.9995], [[1.0, 1.0, 1.0]], [1.0], [[0, 0, 0, 0]])
    f = O.render(rec, _one_pixel_cam(), nthreads=1)
    f9 = O.render(rec, _one_pixel_cam(O.CAP_0999), nthreads=1)
    assert f["image"][0, 0, 0] == float(np.float32(0.99))
    assert f9["image"][0, 0, 0] == float(np.float32(0.999))
    # below both caps nothing changes
    rec["opacity"][0] = 0.5
    assert O.render(rec, _one_pixel_cam(), nthreads=1)["image"][0, 0, 0] == \
        O.render(rec, _one_pixel_cam(O.CAP_0999), nthreads=1)["image"][0, 0, 0] == 0.5


def _isotropic(s, z, f, logit, flags):
    cam = _identity_cam(64, 64, f, f, 32.0, 32.0)
    cam.flags = flags
    params = {"means": np.array([[0.0, 0.0, z]]), "log_scales": np.full((1, 3), math.log(s)),
              "quats": np.array([[1.0, 0.0, 0.0, 0.0]]), "opacity_logits": np.array([logit]),
              "colors": np.ones((1, 3))}
    return cam, params, O.project(params, cam)


def test_antialiased_compensation_closed_form():
    """s4: with the antialiased flag the opacity is multiplied by
    sqrt(det S' / det(S' + 0.3 I)).  An isotropic splat on the axis has
    S' = v I, v = (s f / z)^2, so the factor is v / (v + 0.3)."""
    for s, z, f in [(0.01, 2.0, 60.0), (0.05, 3.0, 100.0), (0.002, 1.5, 50.0)]:
        v = (s * f / z) ** 2
        o = 1.0 / (1.0 + math.exp(-0.4))
        _, _, p0 = _isotropic(s, z, f, 0.4, 0)
        _, _, pa = _isotropic(s, z, f, 0.4, O.ANTIALIASED)
        assert p0["opacity"][0] == o
        assert abs(pa["opacity"][0] - o * v / (v + 0.3)) <= 1e-15
        np.testing.assert_array_equal(pa["conic"], p0["conic"])


def test_gsplat_radii_page_values_and_opacity_extent():
    """s4: gsplat's per-axis radii ceil(3.33 sqrt(S''_xx)), ceil(3.33
    sqrt(S''_yy)) are [18, 17] in the page's example (3DGS: 16); with the
    opacity-aware extent they become ceil(e sqrt(S''_ii)), e = min(3.33,
    sqrt(2 ln(255 o))), and a splat with 255 o <= 1 touches no tile."""
    import json
    import os
    gold = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_examples.json")))
    g = gold["projection_example"]
    ls = np.full(3, 0.5 * math.log(g["cov_camera_isotropic_variance"]))
    params = {"means": np.array(g["means_camera"][:1]), "log_scales": ls[None, :],
              "quats": np.array([[1.0, 0, 0, 0]]), "opacity_logits": np.zeros(1), "colors": np.ones((1, 3))}
    cam = _identity_cam(g["W"], g["H"], g["fx"], g["fy"], g["cx"], g["cy"])
    assert O.project(params, cam)["radius_xy"][0].tolist() == [g["first_radius_3dgs"]] * 2
    cam.flags = O.RADII_AXIS
    p = O.project(params, cam)
    assert p["radius_xy"][0].tolist() == g["first_radii_gsplat"]
    assert p["radius"][0] == max(g["first_radii_gsplat"])
    # the rectangle follows the per-axis radii
    mx, my = p["mean2d"][0]
    rx, ry = g["first_radii_gsplat"]
    expect = [max(0, math.floor((mx - rx) / 16)), max(0, math.floor((my - ry) / 16)),
              min(cam.tiles_x - 1, math.floor((mx + rx) / 16)), min(cam.tiles_y - 1, math.floor((my + ry) / 16))]
    assert p["rect"][0].tolist() == expect
    # opacity-aware extent: o = 0.5 -> e = sqrt(2 ln 127.5) = 3.115
    cam.flags = O.RADII_AXIS | O.RADII_OPACITY
    p = O.project(params, cam)
    a, _, c = p["cov2d"][0]
    e = math.sqrt(2 * math.log(127.5))
    assert p["radius_xy"][0].tolist() == [math.ceil(e * math.sqrt(a)), math.ceil(e * math.sqrt(c))]
    params["opacity_logits"] = np.array([math.log(0.0035 / (1 - 0.0035))])  # 255 o < 1
    p = O.project(params, cam)
    assert p["count"][0] == 0 and p["radius_xy"][0].tolist() == [0, 0]


def test_depth_channel():
    """s5: "C channels of any kind cost the same": with the depth flag each
    record carries its camera z as a fourth colour, blended with the same
    weights and no background (image[..., 3] = sum_i w_i z_i)."""
    rec = _records([[0.5, 0.5], [0.5, 0.5]], [[1.0, 0.0, 1.0]] * 2, [0.6, 0.5],
                   [[1.0, 0.0, 0.0], [0.0, 1.0, 0.0]], [2.0, 3.0], [[0, 0, 0, 0]] * 2)
    rec["color"] = np.array([[1.0, 0.0, 0.0, 2.0], [0.0, 1.0, 0.0, 3.0]])
    cam = _one_pixel_cam(O.DEPTH)
    cam.bg = (0.25, 0.25, 0.25)
    img = O.render(rec, cam, nthreads=1)["image"][0, 0]
    T1 = 1.0 - 0.6
    np.testing.assert_allclose(img, [0.6 + T1 * 0.5 * 0 + T1 * 0.5 * 0.25, T1 * 0.5 + T1 * 0.5 * 0.25,
                                     T1 * 0.5 * 0.25, 0.6 * 2.0 + T1 * 0.5 * 3.0], rtol=1e-12)
    # the projection fills the fourth colour with the camera z
    cam2 = _identity_cam(64, 64, 50.0, 50.0, 32.0, 32.0)
    cam2.flags = O.DEPTH
    params = {"means": np.array([[0.1, -0.2, 3.0], [0.0, 0.1, 5.0]]), "log_scales": np.full((2, 3), -2.0),
              "quats": np.tile([1.0, 0, 0, 0], (2, 1)), "opacity_logits": np.zeros(2),
              "colors": np.array([[0.1, 0.2, 0.3], [0.4, 0.5, 0.6]])}
    p = O.project(params, cam2)
    np.testing.assert_array_equal(p["color"][:, :3], params["colors"])
    np.testing.assert_array_equal(p["color"][:, 3], p["depth"])
    assert O.render(p, cam2, nthreads=1)["image"].shape == (64, 64, 4)
