"""Pins of the CPU oracle to values the pages print, closed forms and invariants.

Each test fails on a plausible mistake in the oracle (a dropped term, a
transposed operand, a wrong sign or index, a wrong threshold) without
restating the oracle's own code.  Page citations are by title and section;
the printed values live in ``tests/golden/page_examples.json``.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle as O
from oracle import dense
from scenes import Camera, make_scene, tiny_camera

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_examples.json")))


def _identity_cam(W, H, fx, fy, cx, cy, bg=(0.0, 0.0, 0.0)):
    return Camera(np.eye(4), fx, fy, cx, cy, W, H, 0.01, bg)


def _records(mean2d, conic, opacity, color, depth, rect, valid=None):
    n = len(opacity)
    return {
        "mean2d": np.asarray(mean2d, dtype=np.float64).reshape(n, 2),
        "conic": np.asarray(conic, dtype=np.float64).reshape(n, 3),
        "opacity": np.asarray(opacity, dtype=np.float64).reshape(n),
        "color": np.asarray(color, dtype=np.float64).reshape(n, 3),
        "depth32": np.asarray(depth, dtype=np.float32).reshape(n),
        "rect": np.asarray(rect, dtype=np.int32).reshape(n, 4),
        "valid": np.ones(n, dtype=np.uint8) if valid is None else np.asarray(valid, np.uint8),
    }


# ---------------------------------------------------------------- s2: Sigma
def test_sigma_45_degrees_page_values():
    """Gaussian splatting in PyTorch, s2: 45 degrees about z, s = (2, .5, 1)."""
    g = GOLD["sigma_45deg"]
    h = math.radians(45.0) / 2.0
    S = O.covariance3d([math.cos(h), 0.0, 0.0, math.sin(h)], np.log(g["scales"]))
    assert S[0, 0] == pytest.approx(g["sigma_00"], abs=1e-12)
    assert S[1, 1] == pytest.approx(g["sigma_11"], abs=1e-12)
    assert S[0, 1] == pytest.approx(g["sigma_01"], abs=1e-12)
    assert S[1, 0] == pytest.approx(g["sigma_01"], abs=1e-12)
    assert S[2, 2] == pytest.approx(g["sigma_22"], abs=1e-12)
    assert S[0, 2] == pytest.approx(0.0, abs=1e-12) and S[1, 2] == pytest.approx(0.0, abs=1e-12)
    # the page's named bug, S R instead of R S, gives diag(4, 0.25, 1): reject it
    assert not np.allclose(np.diag(S), g["wrong_broadcast_diag"])


def test_zero_quaternion_is_identity():
    """Gaussian splatting in PyTorch, s2: normalising with the clamp maps the
    zero quaternion to the identity."""
    np.testing.assert_array_equal(O.quat_to_rotmat([0.0, 0.0, 0.0, 0.0]),
                                  np.array(GOLD["zero_quat"]["rotation"], dtype=np.float64))


def test_rotation_and_covariance_invariants():
    """R is a proper rotation, invariant to the quaternion's scale; Sigma is
    symmetric PSD with eigenvalues exp(log_scale)^2 (s2: 'must stay symmetric
    positive semi-definite')."""
    rng = np.random.default_rng(7)
    for _ in range(50):
        q = rng.normal(size=4)
        ls = rng.normal(-1.0, 1.0, size=3)
        R = O.quat_to_rotmat(q)
        np.testing.assert_allclose(R.T @ R, np.eye(3), atol=1e-12)
        assert np.linalg.det(R) == pytest.approx(1.0, abs=1e-12)
        np.testing.assert_allclose(O.quat_to_rotmat(3.7 * q), R, atol=1e-12)
        # a unit quaternion rotates by 2 acos(w) about (x, y, z)
        qn = q / np.linalg.norm(q)
        axis = qn[1:] / np.linalg.norm(qn[1:])
        np.testing.assert_allclose(R @ axis, axis, atol=1e-12)
        S = O.covariance3d(q, ls)
        np.testing.assert_allclose(S, S.T, atol=1e-14)
        ev = np.sort(np.linalg.eigvalsh(S))
        np.testing.assert_allclose(ev, np.sort(np.exp(2.0 * ls)), rtol=1e-10)
        # eigenvector of the largest scale is the matching column of R
        j = int(np.argmax(ls))
        np.testing.assert_allclose(S @ R[:, j], np.exp(2.0 * ls[j]) * R[:, j], rtol=1e-9, atol=1e-12)


def test_rotation_matches_axis_angle():
    """Rodrigues' formula (a textbook routine) agrees with the quaternion map."""
    rng = np.random.default_rng(11)
    for _ in range(20):
        axis = rng.normal(size=3)
        axis /= np.linalg.norm(axis)
        ang = rng.uniform(-math.pi, math.pi)
        q = [math.cos(ang / 2)] + list(math.sin(ang / 2) * axis)
        K = np.array([[0, -axis[2], axis[1]], [axis[2], 0, -axis[0]], [-axis[1], axis[0], 0]])
        R_ref = np.eye(3) + math.sin(ang) * K + (1 - math.cos(ang)) * K @ K
        np.testing.assert_allclose(O.quat_to_rotmat(q), R_ref, atol=1e-12)


# ---------------------------------------------------------- s3-s4: projection
def test_projection_example_page_values():
    """Gaussian splatting in PyTorch, s3 example and the s4 radius bullets."""
    g = GOLD["projection_example"]
    d = GOLD["projection_example_derived"]
    cam = _identity_cam(g["W"], g["H"], g["fx"], g["fy"], g["cx"], g["cy"])
    ls = np.full(3, 0.5 * math.log(g["cov_camera_isotropic_variance"]))
    first = O.project_debug(g["means_camera"][0], ls, [1, 0, 0, 0], 0.0, cam)
    second = O.project_debug(g["means_camera"][1], ls, [1, 0, 0, 0], 0.0, cam)
    # second Gaussian: J built at the widened frustum edge, mean not clamped
    assert second["clamped_xz"] == pytest.approx(g["second_clamped_x_over_z"], abs=1e-12)
    assert second["clamped_x"] and not second["clamped_y"]
    assert second["mean2d"][0] == pytest.approx(g["second_mean2d_x"], abs=1e-9)
    # first Gaussian: radii by both rules
    assert math.ceil(first["radius_value"]) == g["first_radius_3dgs"]
    a, _, c = first["cov2d"]
    assert [math.ceil(3.33 * math.sqrt(a)), math.ceil(3.33 * math.sqrt(c))] == g["first_radii_gsplat"]
    # hand-derived intermediates
    np.testing.assert_allclose(first["mean2d"], d["first_mean2d"], atol=1e-9)
    np.testing.assert_allclose(first["cov2d"], d["first_cov2d_dilated"], rtol=1e-12)
    assert first["det"] == pytest.approx(d["first_det"], rel=1e-12)
    np.testing.assert_allclose(first["conic"], d["first_conic"], rtol=1e-12)
    assert first["lambda_max"] == pytest.approx(d["first_lambda_max"], rel=1e-12)
    np.testing.assert_allclose(first["J"], [[50.0, 0.0, -10.0], [0.0, 50.0, 5.0]], atol=1e-12)
    # the batched projection takes the same decisions
    params = {"means": np.array(g["means_camera"]), "log_scales": np.tile(ls, (2, 1)),
              "quats": np.array([[1.0, 0, 0, 0]] * 2), "opacity_logits": np.zeros(2),
              "colors": np.ones((2, 3))}
    p = O.project(params, cam)
    assert p["radius"][0] == g["first_radius_3dgs"]
    assert p["count"][1] == 0  # mean at x = 182 px, outside the 64 px image


def test_near_plane_and_view_transform():
    """s3/s6: camera-space mean is W mu + t; z <= 0.01 is culled."""
    rng = np.random.default_rng(3)
    V = np.eye(4)
    R = O.quat_to_rotmat(rng.normal(size=4))
    V[:3, :3] = R
    V[:3, 3] = [0.3, -0.2, 5.0]
    cam = Camera(V, 100, 100, 32, 24, 64, 48)
    mu = rng.normal(size=3)
    d = O.project_debug(mu, [-2, -2, -2], [1, 0, 0, 0], 0.0, cam)
    np.testing.assert_allclose(d["t"], cam.viewmat[:3, :3].astype(np.float64) @ mu +
                               cam.viewmat[:3, 3].astype(np.float64), atol=1e-12)
    near = float(np.float32(0.01))  # the camera holds near_z in single precision
    for z, ok in ((0.0101, True), (near, False), (0.0, False), (-1.0, False)):
        dd = O.project_debug([0.0, 0.0, z], [-2, -2, -2], [1, 0, 0, 0], 0.0,
                             _identity_cam(64, 48, 100, 100, 32, 24))
        assert dd["valid"] == ok


def test_single_isotropic_gaussian_closed_form():
    """A lone isotropic Gaussian on the optical axis: J = diag(f/z) so the
    dilated screen covariance is v I, v = s^2 f^2 / z^2 + 0.3; the image is
    c min(0.99, o exp(-d^2 / 2v)) inside the rectangle where alpha >= 1/255;
    the radius is ceil(3 sqrt(v + sqrt(0.1))) (the 0.1 floor applies since
    mid^2 - det = 0)."""
    for s, logit, f, z in ((0.03, 1.0, 150.0, 4.0), (0.01, 3.0, 150.0, 4.0), (0.2, -0.5, 100.0, 6.0)):
        W = H = 128
        cam = tiny_camera(W, H, f, distance=z)
        params = {"means": np.zeros((1, 3)), "log_scales": np.full((1, 3), math.log(s)),
                  "quats": np.array([[1.0, 0, 0, 0]]), "opacity_logits": np.array([logit]),
                  "colors": np.array([[0.2, 0.5, 0.9]])}
        p = O.project(params, cam)
        v = s * s * f * f / (z * z) + 0.3
        np.testing.assert_allclose(p["cov2d"][0], [v, 0.0, v], rtol=1e-12, atol=1e-15)
        r = math.ceil(3.0 * math.sqrt(v + math.sqrt(0.1)))
        assert p["radius"][0] == r
        o = 1.0 / (1.0 + math.exp(-logit))
        img = O.render(p, cam, nthreads=2)["image"]
        lo, hi = math.floor((64 - r) / 16), math.floor((64 + r) / 16)
        ys, xs = np.mgrid[0:H, 0:W]
        d2 = (xs + 0.5 - 64.0) ** 2 + (ys + 0.5 - 64.0) ** 2
        alpha = np.minimum(np.float64(np.float32(0.99)), o * np.exp(-d2 / (2 * v)))
        tile_in = ((xs // 16 >= max(lo, 0)) & (xs // 16 <= min(hi, 7)) &
                   (ys // 16 >= max(lo, 0)) & (ys // 16 <= min(hi, 7)))
        keep = tile_in & (alpha.astype(np.float32) >= np.float32(1.0) / np.float32(255.0))
        expect = np.where(keep[..., None], alpha[..., None] * params["colors"][0], 0.0)
        np.testing.assert_allclose(img, expect, atol=1e-12)


# ---------------------------------------------------------------- s5: blend
def test_alpha_field_argmax_tie():
    """s5: the first splat sits on the edge between pixels (1, 1) and (1, 2),
    which get the same, largest alpha."""
    g = GOLD["alpha_field"]
    cam = _identity_cam(g["W"], g["H"], 1.0, 1.0, 0.0, 0.0)
    rec = _records([g["means2d"][0]], [g["conics"][0]], [g["opacities"][0]], [[1, 1, 1]], [1.0],
                   [[0, 0, 0, 0]])
    img = O.render(rec, cam, nthreads=1)["image"][..., 0]
    top = np.argwhere(np.isclose(img, img.max(), rtol=0, atol=1e-15)).tolist()
    assert sorted(top) == sorted(g["first_splat_argmax_pixels_row_col"])
    assert img.max() == pytest.approx(0.9 * math.exp(-0.0625), rel=1e-12)
    # the dense form agrees at every pixel
    np.testing.assert_allclose(dense.render_dense(rec, cam)["image"][..., 0], img, atol=1e-15)


def _stack_at_pixel(alphas, colors):
    """Splats centred on the single pixel's centre (sigma = 0, alpha = o)."""
    n = len(alphas)
    return _records([[0.5, 0.5]] * n, [[1.0, 0.0, 1.0]] * n, alphas, colors,
                    np.arange(1, n + 1, dtype=np.float32), [[0, 0, 0, 0]] * n)


def test_compositing_weights():
    """s5: alpha = (.6, .5, .9, .8) gives exclusive T = (1, .4, .2, .02) and
    weights alpha T = (.6, .2, .18, .016), summing to .996."""
    g = GOLD["compositing"]
    cam = _identity_cam(1, 1, 1.0, 1.0, 0.0, 0.0)
    onehot = [[1, 0, 0], [0, 1, 0], [0, 0, 1], [0, 0, 0]]
    out = O.render(_stack_at_pixel(g["alpha"], onehot), cam, nthreads=1)
    w = list(out["image"][0, 0]) + [1.0 - out["T_final"][0, 0] - out["image"][0, 0].sum()]
    np.testing.assert_allclose(w, g["weights"], atol=1e-12)
    assert 1.0 - out["T_final"][0, 0] == pytest.approx(g["weights_sum"], abs=1e-12)
    assert out["n_walk"][0, 0] == 4 and out["e_contrib"][0, 0] == 4
    dn = dense.render_dense(_stack_at_pixel(g["alpha"], onehot), cam)
    np.testing.assert_allclose(dn["weights"][:, 0, 0], g["weights"], atol=1e-12)
    np.testing.assert_allclose(dn["weights"][:, 0, 0] / np.array(g["alpha"]), g["T"], atol=1e-12)


def test_early_termination():
    """s5: four splats of alpha .98 -> T = (1, 2e-2, 4e-4, 8e-6); the third
    would take T below 1e-4, so the loop stops without it and the pixel's
    alpha is 1 - 4e-4."""
    g = GOLD["termination"]
    cam = _identity_cam(1, 1, 1.0, 1.0, 0.0, 0.0)
    out = O.render(_stack_at_pixel(g["alpha"], [[1, 1, 1]] * 4), cam, nthreads=1)
    assert out["image"][0, 0, 0] == pytest.approx(g["accumulated_alpha"], abs=1e-12)
    assert out["T_final"][0, 0] == pytest.approx(g["T"][2], rel=1e-12)
    assert out["n_walk"][0, 0] == sum(g["kept"])
    assert out["e_visit"][0, 0] == 3  # the stopping entry is visited, not added
    dn = dense.render_dense(_stack_at_pixel(g["alpha"], [[1, 1, 1]] * 4), cam)
    assert dn["keep"][:, 0, 0].tolist() == g["kept"]


def test_skip_tests_and_cap():
    """s5 listing: alpha = min(.99, o G); entries with alpha < 1/255 are
    skipped and leave T unchanged; a capped entry has alpha exactly .99."""
    cam = _identity_cam(1, 1, 1.0, 1.0, 0.0, 0.0)
    # 1/255 in float: the entry just below is skipped, just above is kept
    lo = float(np.nextafter(np.float32(1.0) / np.float32(255.0), np.float32(0.0)))
    hi = float(np.nextafter(np.float32(1.0) / np.float32(255.0), np.float32(1.0)))
    out = O.render(_stack_at_pixel([lo, hi, 1.0], [[1, 0, 0], [0, 1, 0], [0, 0, 1]]), cam, nthreads=1)
    im = out["image"][0, 0]
    assert im[0] == 0.0
    assert im[1] == pytest.approx(hi, rel=1e-12)
    assert im[2] == pytest.approx(0.99 * (1 - hi), rel=1e-6)
    assert out["e_visit"][0, 0] == 3 and out["e_contrib"][0, 0] == 2 and out["n_walk"][0, 0] == 3


def test_rect_cutoff_and_background():
    """The tile rectangle is the cutoff: a splat whose rectangle misses a
    tile adds nothing there even where its alpha is large; the background
    is weighted by the final transmittance (s5, last paragraph)."""
    cam = _identity_cam(32, 16, 1.0, 1.0, 0.0, 0.0, bg=(0.25, 0.5, 1.0))
    rec = _records([[15.5, 8.0]], [[0.01, 0.0, 0.01]], [0.8], [[1, 0, 0]], [1.0], [[0, 0, 0, 0]])
    out = O.render(rec, cam, nthreads=1)
    assert np.all(out["image"][:, 16:] == np.array([0.25, 0.5, 1.0]))   # tile 1 not in rect
    assert np.all(out["T_final"][:, 16:] == 1.0)
    np.testing.assert_allclose(out["image"][:, :16, 1], 0.5 * out["T_final"][:, :16], atol=1e-15)
    assert np.all(out["image"][:, :16, 0] > 0.25)


def test_invariants_and_dense_form_random_scenes():
    """For random scenes: T_final in (0, 1]; with white splats and a black
    background sum(w) + T_final = 1; the loop equals the dense cumprod form
    at every pixel."""
    for seed in range(4):
        cam = tiny_camera(40, 36, 60.0)
        params = make_scene("tiny", n=80, seed=seed)
        p = O.project(params, cam)
        out = O.render(p, cam, nthreads=2)
        assert np.all(out["T_final"] > 0) and np.all(out["T_final"] <= 1)
        assert np.all(out["n_walk"] <= out["e_visit"])
        dn = dense.render_dense(p, cam)
        np.testing.assert_allclose(out["image"], dn["image"], atol=1e-12)
        np.testing.assert_allclose(out["T_final"], dn["T_final"], atol=1e-12)
        white = dict(p)
        white["color"] = np.ones_like(p["color"])
        ow = O.render(white, cam, nthreads=2)
        np.testing.assert_allclose(ow["image"][..., 0] + ow["T_final"], 1.0, atol=1e-12)
        assert np.all(out["image"] >= 0) and np.all(out["image"] <= p["color"].max() + 1e-12)


def test_depth_order_is_global_and_stable():
    """s5: one global sort by depth; equal depths keep id order."""
    d = np.array([3.0, 1.0, 2.0, 1.0, 5.0], dtype=np.float32)
    rect = np.array([[0, 0, 0, 0]] * 5, dtype=np.int32)
    valid = np.array([1, 1, 1, 1, 0], dtype=np.uint8)
    assert O.depth_order(d, rect, valid).tolist() == [1, 3, 2, 0]


# ---------------------------------------------------- s6: culled gradients
def test_culled_gaussians_get_exact_zero_gradient():
    """s6: z in {2, 0, -1}; only the first contributes, the others get
    gradients exactly 0, never NaN."""
    g = GOLD["culled_gradient"]
    cam = _identity_cam(32, 32, 40.0, 40.0, 16.0, 16.0)
    n = len(g["camera_z"])
    params = {"means": np.array([[0.0, 0.0, z] for z in g["camera_z"]]),
              "log_scales": np.full((n, 3), -2.0), "quats": np.tile([1.0, 0, 0, 0], (n, 1)),
              "opacity_logits": np.zeros(n), "colors": np.full((n, 3), 0.5)}
    p = O.project(params, cam)
    assert p["valid"].astype(bool).tolist() == g["contributes"]
    dl = np.ones((32, 32, 3))
    g2, _ = O.render_bwd(p, cam, dl, nthreads=1)
    grads = O.project_bwd(params, cam, g2)
    for name, v in grads.items():
        assert np.all(np.isfinite(v)), name
        for k in range(n):
            if not g["contributes"][k]:
                assert np.all(v[k] == 0.0), (name, k)
    assert np.abs(grads["means"][0]).sum() > 0 and np.abs(grads["colors"][0]).sum() > 0


def test_non_finite_colour_is_culled():
    """s6: a Gaussian whose colour is not finite never enters the blend; the
    image of the others is unchanged and its gradients are exactly 0."""
    cam = _identity_cam(32, 32, 40.0, 40.0, 16.0, 16.0)
    params = {"means": np.array([[0.0, 0.0, 2.0], [0.05, 0.0, 2.5]]),
              "log_scales": np.full((2, 3), -2.0), "quats": np.tile([1.0, 0, 0, 0], (2, 1)),
              "opacity_logits": np.zeros(2), "colors": np.array([[0.5, 0.5, 0.5], [0.2, np.nan, 0.1]])}
    p = O.project(params, cam)
    assert p["valid"].tolist() == [1, 0] and p["count"][1] == 0
    one = {k: v[:1] for k, v in params.items()}
    np.testing.assert_array_equal(O.render(p, cam, nthreads=1)["image"],
                                  O.render(O.project(one, cam), cam, nthreads=1)["image"])
    g2, _ = O.render_bwd(p, cam, np.ones((32, 32, 3)), nthreads=1)
    grads = O.project_bwd(params, cam, g2)
    for name, v in grads.items():
        assert np.all(v[1] == 0.0), name
    assert np.abs(grads["means"][0]).sum() > 0 and np.abs(grads["colors"][0]).sum() > 0
