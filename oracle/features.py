"""Feature channels of the oracle: F per-Gaussian values blended with the
forward's weights, and their backward, in double precision.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Source: "Gaussian splatting in PyTorch" s5 (the final weighted sum
image = sum_i w_i c_i + (1 - sum_i w_i) bg costs the same for channels of any
kind: RGB, depth, features).  Reading: features blend without a background;
their backward is the colours' (s6) with the features' dL/dout in place of
dL/dimage and a zero background, so its geometric part (through alpha) adds
to the colours'.  Computed here by running the oracle's own blend and
backward on chunks of four channels (the fourth channel of that path has no
background, and the background is set to zero for all four).
"""
from __future__ import annotations

import copy

import numpy as np

from . import oracle as _o

__all__ = ["render_features", "render_features_bwd"]


def _chunk_setup(proj: dict, cam, features, k: int):
    rec = dict(proj)
    rec["color"] = np.ascontiguousarray(np.asarray(features, np.float64)[:, 4 * k:4 * k + 4])
    c = copy.copy(cam)
    c.flags = int(getattr(cam, "flags", 0)) | _o.DEPTH
    c.bg = (0.0, 0.0, 0.0)
    return rec, c


def _check_F(features) -> int:
    F = int(np.asarray(features).shape[1])
    if F < 4 or F % 4:
        raise ValueError("F must be a positive multiple of 4")
    return F


def render_features(proj: dict, cam, features, tile_mask=None, nthreads: int | None = None) -> np.ndarray:
    """out[p][f] = sum_i w_i features[g_i][f] with the forward's weights of
    `proj` for this camera; returns (H, W, F)."""
    F = _check_F(features)
    out = np.zeros((int(cam.height), int(cam.width), F))
    for k in range(F // 4):
        rec, c = _chunk_setup(proj, cam, features, k)
        out[..., 4 * k:4 * k + 4] = _o.render(rec, c, tile_mask=tile_mask, nthreads=nthreads)["image"]
    return out


def render_features_bwd(proj: dict, cam, features, dL_dout, tile_mask=None, nthreads: int | None = None):
    """Returns (dL_dfeatures (n, F), grad2d (n, 6), grad2d_abs (n, 6)): the
    feature gradients and the features' share of the blend gradient with
    respect to (mean2d x, y, A, B, C, opacity), with the sums of absolute
    terms for tolerances."""
    F = _check_F(features)
    dL = np.asarray(dL_dout, np.float64)
    n = np.asarray(features).shape[0]
    dfeat = np.zeros((n, F))
    g2 = np.zeros((n, 6))
    g2a = np.zeros((n, 6))
    for k in range(F // 4):
        rec, c = _chunk_setup(proj, cam, features, k)
        g, ga = _o.render_bwd(rec, c, np.ascontiguousarray(dL[..., 4 * k:4 * k + 4]), tile_mask=tile_mask,
                              nthreads=nthreads)
        dfeat[:, 4 * k:4 * k + 4] = g[:, 6:10]
        g2 += g[:, :6]
        g2a += ga[:, :6]
    return dfeat, g2, g2a
