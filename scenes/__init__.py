"""Seeded synthetic scenes and cameras.

This module only draws inputs.  It holds none of the rasterizer's arithmetic
(no activation, covariance, projection or blending): raw parameters come out
exactly as an optimiser would store them (log-scales, opacity logits,
unnormalised quaternions, RGB colours), and the cameras as a world-to-camera
matrix plus pinhole intrinsics.  Both the CUDA path and the CPU oracle take
their inputs from here.

Shapes follow the workloads the pages describe: a 30k-Gaussian student and a
742k-Gaussian teacher seen from 60 ring cameras at 980x545 ("The backward pass
I deleted trained the model the Nano runs"), and a 400k-Gaussian full-
resolution training scene ("SplatRs: We Gave the Model 4x More Pixels and It
Got Worse", Lesson 2).  No dataset is read: scenes are mixtures of
anisotropic 3D Gaussian clusters in a 10 m box.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

__all__ = ["Camera", "SceneSpec", "SPECS", "make_scene", "make_cameras", "make_target",
           "look_at", "tiny_camera"]


@dataclasses.dataclass
class Camera:
    """Pinhole camera.  ``viewmat`` is the row-major 4x4 world-to-camera
    matrix [R | t; 0 0 0 1] in OpenCV axes (+x right, +y down, +z forward);
    fx, fy, cx, cy are in pixels; pixel (row i, col j) is sampled at
    (j + 0.5, i + 0.5).  All values are single precision.  ``flags`` holds
    option bits of the renderer (bit 0: the opacity-aware tile cut)."""
    viewmat: np.ndarray
    fx: float
    fy: float
    cx: float
    cy: float
    width: int
    height: int
    near_z: float = 0.01
    bg: tuple = (0.0, 0.0, 0.0)
    flags: int = 0

    def __post_init__(self):
        self.viewmat = np.asarray(self.viewmat, dtype=np.float32).reshape(4, 4)
        self.fx, self.fy, self.cx, self.cy, self.near_z = (
            float(np.float32(v)) for v in (self.fx, self.fy, self.cx, self.cy, self.near_z))
        self.bg = tuple(float(np.float32(v)) for v in self.bg)
        self.width, self.height = int(self.width), int(self.height)
        self.flags = int(self.flags)

    @property
    def tiles_x(self) -> int:
        return (self.width + 15) // 16

    @property
    def tiles_y(self) -> int:
        return (self.height + 15) // 16

    @property
    def tiles(self) -> int:
        return self.tiles_x * self.tiles_y

    @property
    def pixels(self) -> int:
        return self.width * self.height


@dataclasses.dataclass(frozen=True)
class SceneSpec:
    name: str
    n: int
    clusters: int            # 0 = means uniform in [-1, 1]^3
    log_scale_mean: float
    log_scale_std: float
    logit_mean: float
    logit_std: float
    width: int
    height: int
    focal: float
    cameras: str             # "front", "ring", "orbit"
    n_cameras: int
    seed: int


# The workloads.  Log-scale and logit distributions, resolutions and focal
# lengths are those of the configurations this library is measured on.
SPECS = {
    "tiny": SceneSpec("tiny: 1k Gaussians, 128x128, f=150", 1000, 0, -3.5, 0.5, 0.0, 1.5,
                      128, 128, 150.0, "front", 1, 0),
    "student": SceneSpec("student: 30k Gaussians, 20 clusters, 980x545, f=1000", 30_000, 20,
                         -4.0, 0.6, 1.0, 1.5, 980, 545, 1000.0, "ring", 60, 2),
    "teacher": SceneSpec("teacher: 742k Gaussians, 200 clusters, 980x545, f=1000", 742_000, 200,
                         -5.0, 0.7, 0.0, 2.0, 980, 545, 1000.0, "orbit", 16, 3),
    # full resolution, the log-scale mean raised from -4.0 in steps of 0.25
    # until a frame's pair list (opacity-aware cut) exceeds 2^24 entries
    "train400k": SceneSpec("train400k: 400k Gaussians, 120 clusters, log-scales N(-2.5,0.6), 1960x1090, "
                           "f=2000, > 2^24 pairs", 400_000, 120, -2.5, 0.6, 1.0, 1.5, 1960, 1090, 2000.0,
                           "ring", 16, 4),
    "train400k_half": SceneSpec("train400k_half: 400k Gaussians, 120 clusters, 980x545, f=1000",
                                400_000, 120, -4.0, 0.6, 1.0, 1.5, 980, 545, 1000.0, "ring", 16, 4),
    "large_splats": SceneSpec("large_splats: 30k Gaussians, log-scales N(-2.5,0.6), 1960x1090",
                              30_000, 20, -2.5, 0.6, 1.0, 1.5, 1960, 1090, 2000.0, "ring", 16, 5),
    "million": SceneSpec("million: 1M Gaussians, 200 clusters, log-scales N(-5.5,0.5), 1960x1090",
                         1_000_000, 200, -5.5, 0.5, 0.0, 2.0, 1960, 1090, 2000.0, "ring", 16, 6),
}


def _random_rotation(rng: np.random.Generator) -> np.ndarray:
    """A random orthonormal 3x3 matrix (QR of a Gaussian matrix, sign-fixed)."""
    a = rng.normal(size=(3, 3))
    q, r = np.linalg.qr(a)
    q = q * np.sign(np.diag(r))[None, :]
    if np.linalg.det(q) < 0:
        q[:, 0] = -q[:, 0]
    return q


def _cluster_means(rng: np.random.Generator, n: int, clusters: int, box: float = 5.0) -> np.ndarray:
    centres = rng.uniform(-box, box, size=(clusters, 3))
    stds = rng.uniform(0.2, 1.5, size=(clusters, 3))
    rots = np.stack([_random_rotation(rng) for _ in range(clusters)])
    out = np.empty((n, 3), dtype=np.float64)
    filled = 0
    while filled < n:
        m = (n - filled) * 2
        cid = rng.integers(0, clusters, size=m)
        z = rng.normal(size=(m, 3)) * stds[cid]
        pts = centres[cid] + np.einsum("mij,mj->mi", rots[cid], z)
        pts = pts[np.all(np.abs(pts) <= box, axis=1)]
        take = min(n - filled, pts.shape[0])
        out[filled:filled + take] = pts[:take]
        filled += take
    return out


def make_scene(spec: SceneSpec | str, n: int | None = None, seed: int | None = None) -> dict:
    """Raw parameters of a seeded scene, float32, contiguous:
    means (n,3), log_scales (n,3), quats (n,4) with N(0,1) entries (not
    normalised: the rasterizer normalises), opacity_logits (n,),
    colors (n,3) uniform in [0, 1)."""
    if isinstance(spec, str):
        spec = SPECS[spec]
    n = spec.n if n is None else int(n)
    rng = np.random.default_rng(spec.seed if seed is None else seed)
    if spec.clusters == 0:
        means = rng.uniform(-1.0, 1.0, size=(n, 3))
    else:
        means = _cluster_means(rng, n, spec.clusters)
    log_scales = rng.normal(spec.log_scale_mean, spec.log_scale_std, size=(n, 3))
    quats = rng.normal(size=(n, 4))
    logits = rng.normal(spec.logit_mean, spec.logit_std, size=n)
    colors = rng.uniform(0.0, 1.0, size=(n, 3))
    f = lambda a: np.ascontiguousarray(a, dtype=np.float32)  # noqa: E731
    return {"means": f(means), "log_scales": f(log_scales), "quats": f(quats),
            "opacity_logits": f(logits), "colors": f(colors)}


def look_at(position, target=(0.0, 0.0, 0.0), down=(0.0, 1.0, 0.0)) -> np.ndarray:
    """World-to-camera matrix of a camera at ``position`` looking at
    ``target``, OpenCV axes: z forward, x = down x z (right), y = z x x."""
    p = np.asarray(position, dtype=np.float64)
    z = np.asarray(target, dtype=np.float64) - p
    z = z / np.linalg.norm(z)
    x = np.cross(np.asarray(down, dtype=np.float64), z)
    x = x / np.linalg.norm(x)
    y = np.cross(z, x)
    R = np.stack([x, y, z])
    V = np.eye(4)
    V[:3, :3] = R
    V[:3, 3] = -R @ p
    return V.astype(np.float32)


def tiny_camera(width: int = 128, height: int = 128, focal: float = 150.0, distance: float = 4.0,
                bg=(0.0, 0.0, 0.0)) -> Camera:
    """Camera at (0, 0, -distance) with R = I, looking down +z."""
    V = np.eye(4, dtype=np.float32)
    V[2, 3] = distance
    return Camera(V, focal, focal, width / 2.0, height / 2.0, width, height, 0.01, bg)


def make_cameras(spec: SceneSpec | str, count: int | None = None) -> list:
    if isinstance(spec, str):
        spec = SPECS[spec]
    count = spec.n_cameras if count is None else int(count)
    W, H, f = spec.width, spec.height, spec.focal
    if spec.cameras == "front":
        return [tiny_camera(W, H, f) for _ in range(count)]
    cams = []
    if spec.cameras == "ring":
        for k in range(count):
            th = 2.0 * math.pi * k / count
            pos = (8.0 * math.cos(th), 0.0, 8.0 * math.sin(th))
            cams.append(Camera(look_at(pos), f, f, W / 2.0, H / 2.0, W, H))
    elif spec.cameras == "orbit":
        rng = np.random.default_rng(1000 + spec.seed)
        for _ in range(count):
            az = rng.uniform(0.0, 2.0 * math.pi)
            el = math.radians(rng.uniform(-30.0, 30.0))
            pos = (8.0 * math.cos(el) * math.cos(az), 8.0 * math.sin(el), 8.0 * math.cos(el) * math.sin(az))
            cams.append(Camera(look_at(pos), f, f, W / 2.0, H / 2.0, W, H))
    else:
        raise ValueError(spec.cameras)
    return cams


def make_target(width: int, height: int, seed: int = 0, channels: int = 3) -> np.ndarray:
    """A seeded U(0, 1) target image, (H, W, 3) float32; with channels=4 a
    fourth, depth channel U(2, 8) follows (drawn after the colours, so the
    colours do not depend on it)."""
    rng = np.random.default_rng(10_000 + seed)
    rgb = rng.uniform(0.0, 1.0, size=(height, width, 3))
    if channels == 4:
        rgb = np.concatenate([rgb, rng.uniform(2.0, 8.0, size=(height, width, 1))], axis=2)
    elif channels != 3:
        raise ValueError("channels must be 3 or 4")
    return np.ascontiguousarray(rgb, dtype=np.float32)
