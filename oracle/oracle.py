"""ctypes face of the C oracle (``gs_oracle.c``), double precision.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Every function takes and returns numpy arrays.  A camera is any object with
the attributes ``viewmat`` (4x4, row-major world-to-camera, OpenCV axes),
``fx, fy, cx, cy, width, height, near_z`` and ``bg`` (3,), e.g.
``scenes.Camera``; its single-precision values are promoted exactly to
double.

Page citations (by title and section):
  [GSP]  "Gaussian splatting in PyTorch"
  [WEEK] "SplatRs: The Week the Gap Closed", "Throughput: the tile rasterizer"
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

__all__ = [
    "TILE", "TIGHT_TILES", "ANTIALIASED", "STOP_INCLUSIVE", "CAP_0999", "RADII_AXIS",
    "RADII_OPACITY", "DEPTH", "channels", "OrcCamera", "lib", "quat_to_rotmat", "covariance3d", "project_debug", "project", "tile_rects",
    "records_f32", "bin_pairs", "depth_order", "render", "render_bwd", "project_bwd",
    "grad_bound", "default_threads",
]

TILE = 16
# Camera flag bits of the variants (the values the library's camera struct
# uses for the same options).
TIGHT_TILES = 1       # opacity-aware tile cut
ANTIALIASED = 2       # opacity x sqrt(det S' / det S'')
STOP_INCLUSIVE = 4    # stop once next_T <= 1e-4 (gsplat)
CAP_0999 = 8          # alpha cap 0.999 (older gsplat)
RADII_AXIS = 16       # gsplat per-axis 3.33-sigma radii
RADII_OPACITY = 32    # with RADII_AXIS: min(3.33, sqrt(2 ln(255 o))) sigmas
DEPTH = 64            # a fourth channel, camera z, blended with the colours' weights


def channels(cam) -> int:
    """Channels of the rendered image: RGB, plus depth with the DEPTH flag."""
    return 4 if int(getattr(cam, "flags", 0)) & DEPTH else 3

_c_double_p = ctypes.POINTER(ctypes.c_double)
_c_float_p = ctypes.POINTER(ctypes.c_float)
_c_int32_p = ctypes.POINTER(ctypes.c_int32)
_c_int64_p = ctypes.POINTER(ctypes.c_int64)
_c_uint8_p = ctypes.POINTER(ctypes.c_uint8)
_c_uint32_p = ctypes.POINTER(ctypes.c_uint32)
_c_uint64_p = ctypes.POINTER(ctypes.c_uint64)


class OrcCamera(ctypes.Structure):
    _fields_ = [
        ("viewmat", ctypes.c_double * 16),
        ("fx", ctypes.c_double), ("fy", ctypes.c_double),
        ("cx", ctypes.c_double), ("cy", ctypes.c_double),
        ("width", ctypes.c_int32), ("height", ctypes.c_int32),
        ("near_z", ctypes.c_double),
        ("bg", ctypes.c_double * 3),
        ("flags", ctypes.c_int32),
    ]


_LIB = None


def lib() -> ctypes.CDLL:
    """Loads (building if needed) ``libgs_oracle.so``."""
    global _LIB
    if _LIB is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        L.orc_quat_to_rotmat.argtypes = [_c_double_p, _c_double_p]
        L.orc_covariance3d.argtypes = [_c_double_p, _c_double_p, _c_double_p]
        L.orc_project.argtypes = [ctypes.c_int64] + [_c_double_p] * 5 + [ctypes.POINTER(OrcCamera)] + \
            [_c_double_p] * 6 + [_c_float_p, _c_float_p, _c_int32_p, _c_int32_p, _c_uint8_p, _c_double_p,
                                 _c_double_p, _c_double_p]
        L.orc_project.restype = ctypes.c_int
        L.orc_tile_rects.argtypes = [ctypes.c_int64, _c_float_p, _c_float_p, _c_float_p, _c_float_p,
                                     _c_uint8_p, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                     _c_int32_p, _c_int32_p]
        L.orc_bin.argtypes = [ctypes.c_int64, _c_int32_p, _c_uint8_p, _c_float_p, ctypes.c_int32,
                              ctypes.c_int32, ctypes.c_int64, _c_int32_p, _c_uint64_p, _c_uint32_p,
                              _c_uint32_p]
        L.orc_bin.restype = ctypes.c_int64
        L.orc_depth_order.argtypes = [ctypes.c_int64, _c_float_p, _c_int32_p, _c_uint8_p, _c_int64_p]
        L.orc_depth_order.restype = ctypes.c_int64
        L.orc_render.argtypes = [ctypes.c_int64, _c_double_p, _c_double_p, _c_double_p, _c_double_p,
                                 _c_float_p, _c_int32_p, _c_uint8_p, ctypes.POINTER(OrcCamera),
                                 _c_uint8_p, ctypes.c_int, _c_double_p, _c_double_p, _c_int32_p,
                                 _c_int64_p, _c_int64_p, _c_double_p, _c_double_p, _c_double_p]
        L.orc_render_bwd.argtypes = [ctypes.c_int64, _c_double_p, _c_double_p, _c_double_p,
                                     _c_double_p, _c_float_p, _c_int32_p, _c_uint8_p,
                                     ctypes.POINTER(OrcCamera), _c_uint8_p, ctypes.c_int, _c_double_p,
                                     _c_double_p, _c_double_p]
        L.orc_project_debug.argtypes = [_c_double_p, _c_double_p, _c_double_p, ctypes.c_double,
                                        ctypes.POINTER(OrcCamera), _c_double_p]
        L.orc_project_bwd.argtypes = [ctypes.c_int64] + [_c_double_p] * 4 + [ctypes.POINTER(OrcCamera)] + \
            [_c_double_p] * 6
        _LIB = L
    return _LIB


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count() or 1)


def _ptr(a: np.ndarray, ctype):
    return a.ctypes.data_as(ctype)


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _cam(cam) -> OrcCamera:
    c = OrcCamera()
    vm = np.asarray(cam.viewmat, dtype=np.float64).reshape(16)
    for k in range(16):
        c.viewmat[k] = float(vm[k])
    c.fx, c.fy, c.cx, c.cy = (float(np.float64(v)) for v in (cam.fx, cam.fy, cam.cx, cam.cy))
    c.width, c.height = int(cam.width), int(cam.height)
    c.near_z = float(np.float64(cam.near_z))
    bg = np.asarray(cam.bg, dtype=np.float64).reshape(3)
    for k in range(3):
        c.bg[k] = float(bg[k])
    c.flags = int(getattr(cam, "flags", 0))
    return c


def quat_to_rotmat(q) -> np.ndarray:
    """[GSP] s2: (w, x, y, z) -> R, normalised with max(|q|, 1e-12)."""
    q = _f64(q).reshape(4)
    R = np.zeros(9, dtype=np.float64)
    lib().orc_quat_to_rotmat(_ptr(q, _c_double_p), _ptr(R, _c_double_p))
    return R.reshape(3, 3)


def covariance3d(q, log_scale) -> np.ndarray:
    """[GSP] s2: Sigma = R S S^T R^T."""
    q = _f64(q).reshape(4)
    ls = _f64(log_scale).reshape(3)
    S = np.zeros(9, dtype=np.float64)
    lib().orc_covariance3d(_ptr(q, _c_double_p), _ptr(ls, _c_double_p), _ptr(S, _c_double_p))
    return S.reshape(3, 3)


def project_debug(mean, log_scale, quat, opacity_logit, cam) -> dict:
    """Intermediates of one Gaussian's projection ([GSP] s1-s4)."""
    m, ls, q = _f64(mean).reshape(3), _f64(log_scale).reshape(3), _f64(quat).reshape(4)
    out = np.zeros(40)
    c = _cam(cam)
    lib().orc_project_debug(_ptr(m, _c_double_p), _ptr(ls, _c_double_p), _ptr(q, _c_double_p),
                            float(opacity_logit), ctypes.byref(c), _ptr(out, _c_double_p))
    return {"valid": bool(out[0]), "clamped_xz": out[1], "clamped_yz": out[2],
            "J": out[3:9].reshape(2, 3), "cov2d_raw": out[9:12], "cov2d": out[12:15],
            "det": out[15], "conic": out[16:19], "lambda_max": out[19], "radius_value": out[20],
            "mean2d": out[21:23], "t": out[23:26], "Sigma": out[26:35].reshape(3, 3),
            "opacity": out[35], "clamped_x": bool(out[36]), "clamped_y": bool(out[37]),
            "det_clamped": bool(out[38])}


def project(params: dict, cam) -> dict:
    """[GSP] s1-s4, s6 for every Gaussian.  ``params`` holds means (n,3),
    log_scales (n,3), quats (n,4), opacity_logits (n,), colors (n,3)."""
    means = _f64(params["means"]).reshape(-1, 3)
    n = means.shape[0]
    log_scales = _f64(params["log_scales"]).reshape(n, 3)
    quats = _f64(params["quats"]).reshape(n, 4)
    logits = _f64(params["opacity_logits"]).reshape(n)
    colors = _f64(params["colors"]).reshape(n, 3)
    out = {
        "mean2d": np.zeros((n, 2)), "conic": np.zeros((n, 3)), "cov2d": np.zeros((n, 3)),
        "opacity": np.zeros(n), "depth": np.zeros(n), "color": np.zeros((n, channels(cam))),
        "radius": np.zeros(n, dtype=np.float32), "radius_xy": np.zeros((n, 2), dtype=np.float32),
        "rect": np.zeros((n, 4), dtype=np.int32),
        "count": np.zeros(n, dtype=np.int32), "valid": np.zeros(n, dtype=np.uint8),
        "radius_margin": np.zeros(n), "rect_margin": np.zeros(n), "cut_margin": np.zeros(n),
    }
    c = _cam(cam)
    rc = lib().orc_project(
        n, _ptr(means, _c_double_p), _ptr(log_scales, _c_double_p), _ptr(quats, _c_double_p),
        _ptr(logits, _c_double_p), _ptr(colors, _c_double_p), ctypes.byref(c),
        _ptr(out["mean2d"], _c_double_p), _ptr(out["conic"], _c_double_p),
        _ptr(out["cov2d"], _c_double_p), _ptr(out["opacity"], _c_double_p),
        _ptr(out["depth"], _c_double_p), _ptr(out["color"], _c_double_p),
        _ptr(out["radius"], _c_float_p), _ptr(out["radius_xy"], _c_float_p), _ptr(out["rect"], _c_int32_p),
        _ptr(out["count"], _c_int32_p), _ptr(out["valid"], _c_uint8_p),
        _ptr(out["radius_margin"], _c_double_p), _ptr(out["rect_margin"], _c_double_p),
        _ptr(out["cut_margin"], _c_double_p))
    if rc != 0:
        raise ValueError("orc_project: bad arguments")
    out["depth32"] = out["depth"].astype(np.float32)
    return out


def tile_rects(mean2d32, radius32, valid, width: int, height: int, conic32=None, opacity32=None,
               tight: bool = False):
    """The tile-rectangle rule alone, on single-precision records: radius32 is
    one radius per Gaussian (n,) or per-axis radii (n, 2); with ``tight`` the
    opacity-aware cut is taken on conic32 and opacity32."""
    m = np.ascontiguousarray(mean2d32, dtype=np.float32).reshape(-1, 2)
    n = m.shape[0]
    r = np.asarray(radius32, dtype=np.float32)
    r = np.ascontiguousarray(np.repeat(r.reshape(n, 1), 2, axis=1) if r.ndim == 1 else r.reshape(n, 2))
    v = np.ascontiguousarray(valid, dtype=np.uint8).reshape(n)
    cn = np.ascontiguousarray(np.zeros((n, 3)) if conic32 is None else conic32, dtype=np.float32).reshape(n, 3)
    op = np.ascontiguousarray(np.zeros(n) if opacity32 is None else opacity32, dtype=np.float32).reshape(n)
    if tight and (conic32 is None or opacity32 is None):
        raise ValueError("tile_rects: the opacity-aware cut needs conic32 and opacity32")
    rect = np.zeros((n, 4), dtype=np.int32)
    count = np.zeros(n, dtype=np.int32)
    lib().orc_tile_rects(n, _ptr(m, _c_float_p), _ptr(r, _c_float_p), _ptr(cn, _c_float_p),
                         _ptr(op, _c_float_p), _ptr(v, _c_uint8_p), int(width), int(height),
                         1 if tight else 0, _ptr(rect, _c_int32_p), _ptr(count, _c_int32_p))
    return rect, count


def records_f32(proj: dict, width: int, height: int, tight: bool = False) -> dict:
    """Rounds projected records once to single precision (the precision the
    CUDA path stores them in) and re-derives the rectangles from the rounded
    mean2d and radius (and, with ``tight``, the opacity-aware cut from the
    rounded conic and opacity).  Rendering these records in double with
    ``render`` isolates the blend from the projection."""
    out = dict(proj)
    for k in ("mean2d", "conic", "opacity", "color", "depth"):
        out[k] = np.asarray(proj[k], dtype=np.float32).astype(np.float64)
    out["depth32"] = np.asarray(proj["depth"], dtype=np.float32)
    rxy = np.asarray(proj["radius_xy"], dtype=np.float32)
    draws = proj["valid"].astype(bool) & np.any(rxy > 0, axis=1)  # an empty opacity extent draws nothing
    rect, count = tile_rects(out["mean2d"].astype(np.float32), rxy, draws, width, height,
                             out["conic"].astype(np.float32), out["opacity"].astype(np.float32), tight)
    out["rect"], out["count"] = rect, count
    return out


def bin_pairs(rect, valid, depth32, width: int, height: int, max_pairs: int | None = None) -> dict:
    """[WEEK] count, emit, sort, range, by brute force over (Gaussian, tile)."""
    rect = np.ascontiguousarray(rect, dtype=np.int32).reshape(-1, 4)
    n = rect.shape[0]
    valid = np.ascontiguousarray(valid, dtype=np.uint8).reshape(n)
    depth32 = np.ascontiguousarray(depth32, dtype=np.float32).reshape(n)
    tiles = ((width + TILE - 1) // TILE) * ((height + TILE - 1) // TILE)
    counts = np.zeros(n, dtype=np.int32)
    if max_pairs is None:
        nx = np.where(valid.astype(bool) & (rect[:, 2] >= rect[:, 0]) & (rect[:, 3] >= rect[:, 1]),
                      (rect[:, 2] - rect[:, 0] + 1).astype(np.int64) *
                      (rect[:, 3] - rect[:, 1] + 1).astype(np.int64), 0)
        max_pairs = int(nx.sum())
    keys = np.zeros(max(max_pairs, 1), dtype=np.uint64)
    gids = np.zeros(max(max_pairs, 1), dtype=np.uint32)
    ranges = np.zeros((tiles, 2), dtype=np.uint32)
    k = lib().orc_bin(n, _ptr(rect, _c_int32_p), _ptr(valid, _c_uint8_p), _ptr(depth32, _c_float_p),
                      int(width), int(height), int(max_pairs), _ptr(counts, _c_int32_p),
                      _ptr(keys, _c_uint64_p), _ptr(gids, _c_uint32_p), _ptr(ranges, _c_uint32_p))
    if k < 0:
        raise ValueError("orc_bin: pair list exceeds max_pairs" if k == -1 else "orc_bin: out of memory")
    return {"counts": counts, "keys": keys[:k], "gids": gids[:k], "ranges": ranges, "n_pairs": int(k)}


def depth_order(depth32, rect, valid) -> np.ndarray:
    depth32 = np.ascontiguousarray(depth32, dtype=np.float32)
    n = depth32.shape[0]
    rect = np.ascontiguousarray(rect, dtype=np.int32).reshape(n, 4)
    valid = np.ascontiguousarray(valid, dtype=np.uint8).reshape(n)
    order = np.zeros(max(n, 1), dtype=np.int64)
    m = lib().orc_depth_order(n, _ptr(depth32, _c_float_p), _ptr(rect, _c_int32_p),
                              _ptr(valid, _c_uint8_p), _ptr(order, _c_int64_p))
    return order[:m]


def _render_inputs(proj: dict, nc: int = 3):
    n = np.asarray(proj["mean2d"]).reshape(-1, 2).shape[0]
    return (n, _f64(proj["mean2d"]).reshape(n, 2), _f64(proj["conic"]).reshape(n, 3),
            _f64(proj["opacity"]).reshape(n), _f64(proj["color"]).reshape(n, nc),
            np.ascontiguousarray(proj["depth32"], dtype=np.float32).reshape(n),
            np.ascontiguousarray(proj["rect"], dtype=np.int32).reshape(n, 4),
            np.ascontiguousarray(proj["valid"], dtype=np.uint8).reshape(n))


def _mask(cam, tile_mask):
    if tile_mask is None:
        return None, None
    tiles = ((cam.width + TILE - 1) // TILE) * ((cam.height + TILE - 1) // TILE)
    m = np.ascontiguousarray(tile_mask, dtype=np.uint8).reshape(tiles)
    return m, _ptr(m, _c_uint8_p)


def render(proj: dict, cam, tile_mask=None, nthreads: int | None = None) -> dict:
    """[WEEK] naive renderer with the tile-rectangle cutoff; [GSP] s5 loop."""
    nc = channels(cam)
    n, m2, con, op, col, d32, rect, valid = _render_inputs(proj, nc)
    H, W = int(cam.height), int(cam.width)
    out = {"image": np.zeros((H, W, nc)), "T_final": np.zeros((H, W)),
           "n_walk": np.zeros((H, W), dtype=np.int32), "e_visit": np.zeros((H, W), dtype=np.int64),
           "e_contrib": np.zeros((H, W), dtype=np.int64),
           "margin_alpha": np.full((H, W), np.inf), "margin_T": np.full((H, W), np.inf),
           "margin_clamp": np.full((H, W), np.inf)}
    c = _cam(cam)
    mk, mkp = _mask(cam, tile_mask)
    rc = lib().orc_render(
        n, _ptr(m2, _c_double_p), _ptr(con, _c_double_p), _ptr(op, _c_double_p),
        _ptr(col, _c_double_p), _ptr(d32, _c_float_p), _ptr(rect, _c_int32_p),
        _ptr(valid, _c_uint8_p), ctypes.byref(c), mkp, int(nthreads or default_threads()),
        _ptr(out["image"], _c_double_p), _ptr(out["T_final"], _c_double_p),
        _ptr(out["n_walk"], _c_int32_p), _ptr(out["e_visit"], _c_int64_p),
        _ptr(out["e_contrib"], _c_int64_p), _ptr(out["margin_alpha"], _c_double_p),
        _ptr(out["margin_T"], _c_double_p), _ptr(out["margin_clamp"], _c_double_p))
    if rc != 0:
        raise ValueError("orc_render failed")
    return out


def render_bwd(proj: dict, cam, dL_dimage, tile_mask=None, nthreads: int | None = None):
    """[GSP] s6 back-to-front analytic backward of the blend.  Returns
    (grad2d, grad2d_abs), each (n, 9): dmean2d x/y, dA, dB, dC, dopacity,
    dr, dg, db (and a tenth column, the depth channel, with the DEPTH flag),
    and the sums of absolute contributions."""
    nc = channels(cam)
    n, m2, con, op, col, d32, rect, valid = _render_inputs(proj, nc)
    H, W = int(cam.height), int(cam.width)
    g = _f64(dL_dimage).reshape(H, W, nc)
    grad2d = np.zeros((n, 6 + nc))
    grad_abs = np.zeros((n, 6 + nc))
    c = _cam(cam)
    mk, mkp = _mask(cam, tile_mask)
    rc = lib().orc_render_bwd(
        n, _ptr(m2, _c_double_p), _ptr(con, _c_double_p), _ptr(op, _c_double_p),
        _ptr(col, _c_double_p), _ptr(d32, _c_float_p), _ptr(rect, _c_int32_p),
        _ptr(valid, _c_uint8_p), ctypes.byref(c), mkp, int(nthreads or default_threads()),
        _ptr(g, _c_double_p), _ptr(grad2d, _c_double_p), _ptr(grad_abs, _c_double_p))
    if rc != 0:
        raise ValueError("orc_render_bwd failed")
    return grad2d, grad_abs


def project_bwd(params: dict, cam, grad2d) -> dict:
    """[GSP] s6 chain rule from the 2D gradients to the raw parameters."""
    means = _f64(params["means"]).reshape(-1, 3)
    n = means.shape[0]
    log_scales = _f64(params["log_scales"]).reshape(n, 3)
    quats = _f64(params["quats"]).reshape(n, 4)
    logits = _f64(params["opacity_logits"]).reshape(n)
    g2 = _f64(grad2d).reshape(n, 6 + channels(cam))
    out = {"means": np.zeros((n, 3)), "log_scales": np.zeros((n, 3)), "quats": np.zeros((n, 4)),
           "opacity_logits": np.zeros(n), "colors": np.zeros((n, 3))}
    c = _cam(cam)
    lib().orc_project_bwd(
        n, _ptr(means, _c_double_p), _ptr(log_scales, _c_double_p), _ptr(quats, _c_double_p),
        _ptr(logits, _c_double_p), ctypes.byref(c), _ptr(g2, _c_double_p),
        _ptr(out["means"], _c_double_p), _ptr(out["log_scales"], _c_double_p),
        _ptr(out["quats"], _c_double_p), _ptr(out["opacity_logits"], _c_double_p),
        _ptr(out["colors"], _c_double_p))
    return out


def grad_bound(params: dict, cam, grad2d_abs) -> dict:
    """Propagates the per-element sums of absolute 2D contributions through
    the absolute value of the (linear) chain rule, giving for each raw
    gradient element a bound on the magnitude of the terms it sums.  Used for
    the cancellation-aware gradient tolerance."""
    n = np.asarray(params["means"]).reshape(-1, 3).shape[0]
    ng = 6 + channels(cam)
    ga = _f64(grad2d_abs).reshape(n, ng)
    total = {k: np.zeros_like(v) for k, v in project_bwd(params, cam, np.zeros((n, ng))).items()}
    for k in range(ng):
        e = np.zeros((n, ng))
        e[:, k] = 1.0
        col = project_bwd(params, cam, e)
        for name, v in col.items():
            shape = v.shape
            total[name] = total[name] + np.abs(v) * ga[:, k].reshape((n,) + (1,) * (len(shape) - 1))
    return total
