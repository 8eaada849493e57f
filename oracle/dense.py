"""Dense [M, H, W] formulation of the blend, in numpy float64.

TEST INFRASTRUCTURE ONLY.  This is a second, independent statement of the
forward render, written from "Gaussian splatting in PyTorch" s5
("Compositing as tensor ops"): every drawable splat is evaluated at every
pixel centre as one tensor, the transmittance is the exclusive cumulative
product of (1 - alpha) along the depth-sorted axis, and early termination is
a prefix mask.  The tile-rectangle cutoff of the tiled method is applied as
one more mask.  It is used to pin the C oracle's per-pixel loop; it is only
practical for small scenes (memory grows as M x H x W).
"""
from __future__ import annotations

import numpy as np

TILE = 16
ALPHA_CAP_F = np.float32(0.99)
ALPHA_MIN_F = np.float32(1.0) / np.float32(255.0)
T_MIN_F = np.float32(1e-4)


def depth_sort(depth32: np.ndarray, rect: np.ndarray, valid: np.ndarray) -> np.ndarray:
    """Drawable splats (valid, non-empty rectangle) ordered by (float bits of
    depth, id): one global stable sort ([GSP] s5)."""
    n = depth32.shape[0]
    draw = valid.astype(bool) & (rect[:, 0] <= rect[:, 2]) & (rect[:, 1] <= rect[:, 3])
    ids = np.nonzero(draw)[0]
    bits = depth32.astype(np.float32).view(np.uint32)[ids]
    return ids[np.lexsort((ids, bits))] if n else ids


def render_dense(proj: dict, cam) -> dict:
    H, W = int(cam.height), int(cam.width)
    order = depth_sort(np.asarray(proj["depth32"], dtype=np.float32), np.asarray(proj["rect"]),
                       np.asarray(proj["valid"]))
    bg = np.asarray(cam.bg, dtype=np.float64).reshape(3)
    M = order.shape[0]
    if M == 0:
        return {"image": np.broadcast_to(bg, (H, W, 3)).copy(), "T_final": np.ones((H, W)),
                "weights": np.zeros((0, H, W))}
    mean2d = np.asarray(proj["mean2d"], dtype=np.float64)[order]
    conic = np.asarray(proj["conic"], dtype=np.float64)[order]
    opac = np.asarray(proj["opacity"], dtype=np.float64)[order]
    colors = np.asarray(proj["color"], dtype=np.float64)[order]
    rect = np.asarray(proj["rect"])[order]

    xs = np.arange(W, dtype=np.float64) + 0.5          # pixel centres at +0.5
    ys = np.arange(H, dtype=np.float64) + 0.5
    dx = mean2d[:, 0, None, None] - xs[None, None, :]   # [M, 1, W]
    dy = mean2d[:, 1, None, None] - ys[None, :, None]   # [M, H, 1]
    A, B, C = (conic[:, k, None, None] for k in range(3))
    sigma = 0.5 * (A * dx ** 2 + C * dy ** 2) + B * dx * dy
    oG = opac[:, None, None] * np.exp(-sigma)
    alpha = np.where(oG.astype(np.float32) > ALPHA_CAP_F, np.float64(ALPHA_CAP_F), oG)

    tx = (np.arange(W) // TILE)[None, None, :]
    ty = (np.arange(H) // TILE)[None, :, None]
    in_rect = ((tx >= rect[:, 0, None, None]) & (tx <= rect[:, 2, None, None]) &
               (ty >= rect[:, 1, None, None]) & (ty <= rect[:, 3, None, None]))
    alpha = np.where(in_rect & (sigma >= 0) & (alpha.astype(np.float32) >= ALPHA_MIN_F), alpha, 0.0)

    one_minus = 1.0 - alpha
    inclusive = np.cumprod(one_minus, axis=0)
    T = np.concatenate([np.ones((1, H, W)), inclusive[:-1]], axis=0)     # exclusive
    keep = (T * one_minus).astype(np.float32) >= T_MIN_F                # a prefix along M
    w = alpha * T * keep
    T_final = np.prod(np.where(keep, one_minus, 1.0), axis=0)
    image = np.einsum("mhw,mc->hwc", w, colors) + T_final[..., None] * bg
    return {"image": image, "T_final": T_final, "weights": w, "keep": keep, "order": order}
