"""Finite-difference pins of the oracle's analytic backward.

"Gaussian splatting in PyTorch", s6: differentiable code is tested in float64
against finite differences.  Here the oracle's forward (float64) is
differentiated numerically by central differences and compared with its
analytic backward: first with respect to the projected records (pins the
blend backward alone), then with respect to every raw parameter (pins the
chain rule through conic, dilation, J and its clamp, view rotation, R S,
quaternion normalisation, exp and sigmoid).

Scenes are tiny and chosen away from every discontinuity: no alpha, cap or
transmittance test within 1e-4 (relative) of its threshold, no radius or tile
edge within 1e-4 of an integer, distinct depths; a perturbation of 1e-6
then flips no decision.
"""
import math

import numpy as np
import pytest

import oracle as O
from scenes import Camera, tiny_camera

H_STEP = 1e-6


def _scene(seed, n=6, clamp_case=False, bg=(0.0, 0.0, 0.0), flags=0):
    rng = np.random.default_rng(seed)
    W, H, f = 40, 36, 60.0
    cam = tiny_camera(W, H, f, distance=4.0, bg=bg)
    cam.flags = flags
    means = np.column_stack([rng.uniform(-0.4, 0.4, n), rng.uniform(-0.4, 0.4, n),
                             rng.uniform(-0.5, 0.5, n)])
    params = {"means": means, "log_scales": rng.normal(-2.2, 0.3, (n, 3)),
              "quats": rng.normal(size=(n, 4)), "opacity_logits": rng.normal(0.0, 1.0, n),
              "colors": rng.uniform(0.0, 1.0, (n, 3))}
    if clamp_case:
        # x/z = 0.5 lies beyond the widened frustum edge (20/60 + 0.1 = 0.433);
        # the splat is large enough to reach into the image
        params["means"] = np.vstack([params["means"], [2.0, 0.1, 0.0]])
        params["log_scales"] = np.vstack([params["log_scales"], [0.2, -0.1, 0.1]])
        params["quats"] = np.vstack([params["quats"], rng.normal(size=(1, 4))])
        params["opacity_logits"] = np.append(params["opacity_logits"], 0.5)
        params["colors"] = np.vstack([params["colors"], [0.9, 0.1, 0.4]])
    return cam, params


def _clean(cam, params):
    p = O.project(params, cam)
    out = O.render(p, cam, nthreads=2)
    v = p["valid"].astype(bool)
    d = np.sort(p["depth32"][v])
    return (out["margin_alpha"].min() > 1e-4 and out["margin_T"].min() > 1e-4 and
            out["margin_clamp"].min() > 1e-4 and
            p["rect_margin"][v].min() > 1e-4 and p["radius_margin"][v].min() > 1e-4 and
            (len(d) < 2 or np.diff(d).min() > 1e-5) and p["count"].sum() > 0)


def _find_clean(seed0, **kw):
    for seed in range(seed0, seed0 + 200):
        cam, params = _scene(seed, **kw)
        if _clean(cam, params):
            return cam, params
    raise RuntimeError("no clean scene found")


def _loss_weights(cam, seed=99):
    return np.random.default_rng(seed).normal(size=(cam.height, cam.width, O.channels(cam)))


def _loss_from_records(rec, cam, w):
    return float((O.render(rec, cam, nthreads=2)["image"] * w).sum())


def _loss_from_params(params, cam, w):
    return _loss_from_records(O.project(params, cam), cam, w)


@pytest.mark.parametrize("bg,flags", [((0.0, 0.0, 0.0), 0), ((0.3, 0.2, 0.1), 0), ((0.3, 0.2, 0.1), O.DEPTH)])
def test_blend_backward_matches_finite_differences(bg, flags):
    cam, params = _find_clean(100, bg=bg, flags=flags)
    w = _loss_weights(cam)
    rec = O.project(params, cam)
    g2, g2abs = O.render_bwd(rec, cam, w, nthreads=2)
    nc = O.channels(cam)
    fields = [("mean2d", 2, [0, 1]), ("conic", 3, [2, 3, 4]), ("opacity", 1, [5]),
              ("color", nc, list(range(6, 6 + nc)))]
    checked = 0
    for g in range(len(rec["opacity"])):
        if rec["count"][g] == 0:
            continue
        for name, width, cols in fields:
            for k in range(width):
                r_p = {kk: (vv.copy() if isinstance(vv, np.ndarray) else vv) for kk, vv in rec.items()}
                r_m = {kk: (vv.copy() if isinstance(vv, np.ndarray) else vv) for kk, vv in rec.items()}
                if width == 1:
                    r_p[name][g] += H_STEP
                    r_m[name][g] -= H_STEP
                else:
                    r_p[name][g, k] += H_STEP
                    r_m[name][g, k] -= H_STEP
                fd = (_loss_from_records(r_p, cam, w) - _loss_from_records(r_m, cam, w)) / (2 * H_STEP)
                an = g2[g, cols[k]]
                assert abs(fd - an) <= 1e-6 + 1e-5 * abs(an), (g, name, k, fd, an)
                checked += 1
    assert checked >= 27
    assert np.all(g2abs >= np.abs(g2) - 1e-15)


ALL_VARIANTS = O.ANTIALIASED | O.RADII_AXIS | O.RADII_OPACITY | O.CAP_0999 | O.STOP_INCLUSIVE


@pytest.mark.parametrize("clamp_case,flags", [(False, 0), (True, 0), (False, O.ANTIALIASED),
                                              (True, ALL_VARIANTS), (False, O.DEPTH),
                                              (True, ALL_VARIANTS | O.DEPTH)])
def test_raw_parameter_gradients_match_finite_differences(clamp_case, flags):
    """With the antialiased flag the chain also runs through the
    compensation sqrt(det S' / det S'') into S' and the sigmoid."""
    cam, params = _find_clean(300, clamp_case=clamp_case, bg=(0.1, 0.2, 0.3), flags=flags)
    if clamp_case:
        d = O.project_debug(params["means"][-1], params["log_scales"][-1], params["quats"][-1],
                            params["opacity_logits"][-1], cam)
        assert d["clamped_x"] and d["valid"]
        assert O.project(params, cam)["count"][-1] > 0
    w = _loss_weights(cam)
    rec = O.project(params, cam)
    g2, _ = O.render_bwd(rec, cam, w, nthreads=2)
    grads = O.project_bwd(params, cam, g2)
    n = len(params["opacity_logits"])
    for name in ("means", "log_scales", "quats", "opacity_logits", "colors"):
        for g in range(n):
            width = 1 if params[name].ndim == 1 else params[name].shape[1]
            for k in range(width):
                pp = {kk: vv.copy() for kk, vv in params.items()}
                pm = {kk: vv.copy() for kk, vv in params.items()}
                if width == 1:
                    pp[name][g] += H_STEP
                    pm[name][g] -= H_STEP
                    an = grads[name][g]
                else:
                    pp[name][g, k] += H_STEP
                    pm[name][g, k] -= H_STEP
                    an = grads[name][g, k]
                fd = (_loss_from_params(pp, cam, w) - _loss_from_params(pm, cam, w)) / (2 * H_STEP)
                assert abs(fd - an) <= 1e-6 + 2e-5 * abs(an), (name, g, k, fd, an)


def test_gradient_bound_dominates():
    """The absolute-contribution bound used for the cancellation-aware
    tolerance is never below the gradient it bounds."""
    cam, params = _find_clean(500)
    w = _loss_weights(cam)
    rec = O.project(params, cam)
    g2, g2abs = O.render_bwd(rec, cam, w, nthreads=2)
    grads = O.project_bwd(params, cam, g2)
    bound = O.grad_bound(params, cam, g2abs)
    for name in grads:
        assert np.all(bound[name] >= np.abs(grads[name]) * (1 - 1e-12)), name


def test_zero_quaternion_gradient_is_finite():
    """s2/s6: the clamp makes the zero quaternion a legal input; its gradient
    is finite (zero, as every rotation entry is stationary there)."""
    cam = tiny_camera(32, 32, 40.0)
    params = {"means": np.zeros((1, 3)), "log_scales": np.array([[-1.5, -2.0, -2.5]]),
              "quats": np.zeros((1, 4)), "opacity_logits": np.zeros(1), "colors": np.ones((1, 3))}
    rec = O.project(params, cam)
    g2, _ = O.render_bwd(rec, cam, np.ones((32, 32, 3)), nthreads=1)
    grads = O.project_bwd(params, cam, g2)
    assert np.all(np.isfinite(grads["quats"])) and np.all(grads["quats"] == 0.0)
    assert np.abs(grads["log_scales"]).sum() > 0
