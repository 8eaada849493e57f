"""Pins of the oracle's feature channels ("Gaussian splatting in PyTorch",
s5: the final weighted sum costs the same for channels of any kind, RGB,
depth or features; s6: their backward, in float64 against finite
differences)."""
import copy

import numpy as np
import pytest

import oracle as O
from oracle import features as OF

from test_oracle_gradients import H_STEP, _find_clean


def test_features_equal_to_colours_reproduce_the_image():
    cam, params = _find_clean(10)
    cam = copy.copy(cam)
    cam.bg = (0.0, 0.0, 0.0)
    p = O.project(params, cam)
    n = params["means"].shape[0]
    feats = np.column_stack([params["colors"], np.zeros(n)])
    out = OF.render_features(p, cam, feats, nthreads=2)
    img = O.render(p, cam, nthreads=2)["image"]
    np.testing.assert_array_equal(out[..., :3], img)
    assert np.all(out[..., 3] == 0.0)


def test_a_constant_feature_gives_the_coverage_and_chunks_are_independent():
    """A feature of 1 on every Gaussian blends to sum_i w_i = 1 - T_final;
    the second chunk of [f, 2 f + 1] is twice the first plus the coverage."""
    cam, params = _find_clean(20, bg=(0.3, 0.2, 0.1))
    p = O.project(params, cam)
    n = params["means"].shape[0]
    f = np.random.default_rng(3).uniform(-1, 1, (n, 4))
    out = OF.render_features(p, cam, np.hstack([f, 2 * f + 1]), nthreads=2)
    cover = 1.0 - O.render(p, cam, nthreads=2)["T_final"]
    np.testing.assert_allclose(out[..., 4:], 2 * out[..., :4] + cover[..., None], rtol=1e-12, atol=1e-14)
    ones = OF.render_features(p, cam, np.ones((n, 4)), nthreads=2)
    np.testing.assert_allclose(ones, np.repeat(cover[..., None], 4, axis=2), rtol=1e-12, atol=1e-14)
    with pytest.raises(ValueError):
        OF.render_features(p, cam, np.ones((n, 6)))


def test_features_backward_matches_finite_differences():
    """loss = sum(out * W) over 8 feature channels: dL/dfeatures (linear, so
    the differences are exact up to rounding) and the features' share of the
    raw-parameter gradient, through projection, blend weights and the chain
    rule, against central differences of the float64 oracle."""
    cam, params = _find_clean(30)
    n = params["means"].shape[0]
    rng = np.random.default_rng(7)
    feats = rng.uniform(-1, 1, (n, 8))
    W = rng.normal(size=(cam.height, cam.width, 8))

    def loss(prm, fts):
        return float((OF.render_features(O.project(prm, cam), cam, fts, nthreads=2) * W).sum())

    p = O.project(params, cam)
    dfeat, g2, _ = OF.render_features_bwd(p, cam, feats, W, nthreads=2)
    for idx in [(0, 0), (1, 5), (2, 7), (n - 1, 3)]:
        fp, fm = feats.copy(), feats.copy()
        fp[idx] += H_STEP
        fm[idx] -= H_STEP
        fd = (loss(params, fp) - loss(params, fm)) / (2 * H_STEP)
        assert abs(fd - dfeat[idx]) <= 1e-7 + 1e-6 * abs(dfeat[idx]), (idx, fd, dfeat[idx])
    raw = O.project_bwd(params, cam, np.hstack([g2, np.zeros((n, 3))]))
    assert np.all(raw["colors"] == 0.0)  # the features do not touch the colours
    checked = 0
    for k in ("means", "log_scales", "quats", "opacity_logits"):
        for idx in np.ndindex(params[k].shape):
            if idx[0] not in (0, 2):
                continue
            pp = {q: v.copy() for q, v in params.items()}
            pm = {q: v.copy() for q, v in params.items()}
            pp[k][idx] += H_STEP
            pm[k][idx] -= H_STEP
            fd = (loss(pp, feats) - loss(pm, feats)) / (2 * H_STEP)
            an = raw[k][idx]
            assert abs(fd - an) <= 1e-6 + 1e-4 * abs(an), (k, idx, fd, an)
            checked += 1
    assert checked == 2 * 11
