"""B200 tile-binned differentiable 3D Gaussian splatting rasterizer.

A thin Python binding over libgs.so (include/gs.h).  The functions below carry
the C entry points' names and only marshal arguments: every step of the path
runs in the library's CUDA kernels.  PyTorch provides device memory and the
current CUDA stream.

    proj = Projected(n)
    bins = Bins(n, max_pairs, width, height)
    gs_project(cam, params, proj)
    K = gs_bin_and_sort(cam, n, proj, bins)           # sync=True reads K back
    gs_render_fwd(cam, n, proj, bins, image, T_final, last)
    gs_render_bwd(cam, n, params, proj, bins, T_final, last, dL_dimage, grad2d, grads)

``params`` and ``grads`` are dicts of contiguous float32 CUDA tensors with
keys means (N,3), log_scales (N,3), quats (N,4), opacity_logits (N,),
colors (N,3).  A camera is any object with viewmat (4x4 world-to-camera,
OpenCV axes), fx, fy, cx, cy, width, height, near_z and bg.
"""
from __future__ import annotations

import ctypes

import torch

from . import _abi
from ._abi import (GS_BIN_AUTO, GS_BIN_GLOBAL, GS_BIN_PER_TILE, GS_ERR_ALIGNMENT, GS_ERR_CAPACITY, GS_ERR_CUDA, GS_ERR_DEVICE_TIMEOUT,  # noqa: F401
                   GS_ERR_INVALID_ARG, GS_ERR_TOO_LARGE, GS_FLAG_ANTIALIASED, GS_FLAG_CAP_0999, GS_FLAG_DEPTH,
                   GS_FLAG_RADII_AXIS, GS_FLAG_RADII_OPACITY, GS_FLAG_STOP_INCLUSIVE, GS_FLAG_TIGHT_TILES, GS_OK,
                   GS_TILE)

__all__ = [
    "GSError", "Projected", "Bins", "make_camera", "channels", "gs_project", "gs_bin_and_sort",
    "gs_bin_and_sort_static", "gs_render_fwd", "gs_render_fwd_l1", "gs_render_features_fwd", "gs_render_features_bwd",
    "gs_render_bwd", "gs_render_stats", "gs_l1_loss_grad", "gs_read_status", "gs_last_device_error",
    "gs_sort_bytes", "gs_error_string", "profile_begin",
    "profile_end", "lib", "PARAM_KEYS",
]

PARAM_KEYS = ("means", "log_scales", "quats", "opacity_logits", "colors")


def lib() -> ctypes.CDLL:
    return _abi.load()


class GSError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {gs_error_string(code)} (code {code})")
        self.code = code


def gs_error_string(code: int) -> str:
    return lib().gs_error_string(int(code)).decode()


def _check(rc: int, what: str) -> int:
    if rc < 0:
        raise GSError(rc, what)
    return rc


def _dev(t: torch.Tensor | None, name: str, dtype=None) -> ctypes.c_void_p:
    if t is None:
        return ctypes.c_void_p(0)
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def channels(cam) -> int:
    """Image channels for a camera: RGB, plus depth with GS_FLAG_DEPTH."""
    return 4 if int(getattr(cam, "flags", 0)) & GS_FLAG_DEPTH else 3


def make_camera(cam) -> _abi.GsCamera:
    """A gs_camera from a camera-like object (returned as is if it already is one)."""
    if isinstance(cam, _abi.GsCamera):
        return cam
    c = _abi.GsCamera()
    vm = [float(v) for v in torch.as_tensor(cam.viewmat, dtype=torch.float32).reshape(16).tolist()]
    for k in range(16):
        c.viewmat[k] = vm[k]
    c.fx, c.fy, c.cx, c.cy = float(cam.fx), float(cam.fy), float(cam.cx), float(cam.cy)
    c.width, c.height = int(cam.width), int(cam.height)
    c.near_z = float(cam.near_z)
    for k in range(3):
        c.bg[k] = float(cam.bg[k])
    c.flags = int(getattr(cam, "flags", 0))
    return c


def _params_struct(params: dict, cls=_abi.GsParams):
    s = cls()
    for k in PARAM_KEYS:
        setattr(s, k, _dev(params[k], k, torch.float32).value)
    return s


class _Carved:
    """A caller-owned device buffer carved into the library's arrays."""

    def _view(self, ptr: int, count: int, dtype: torch.dtype, shape) -> torch.Tensor:
        off = ptr - self.buffer.data_ptr()
        nbytes = count * torch.tensor([], dtype=dtype).element_size()
        return self.buffer[off:off + nbytes].view(dtype).view(*shape)


class Projected(_Carved):
    """gs_projected records for n Gaussians, in one device buffer."""

    def __init__(self, n: int, device="cuda"):
        self.n = int(n)
        nbytes = max(int(lib().gs_projected_bytes(self.n)), 256)
        self.buffer = torch.empty(nbytes, dtype=torch.uint8, device=device)
        self.struct = _abi.GsProjected()
        _check(lib().gs_projected_carve(ctypes.c_void_p(self.buffer.data_ptr()), self.n,
                                        ctypes.byref(self.struct)), "gs_projected_carve")
        n = self.n
        self.xy_opacity_depth = self._view(self.struct.xy_opacity_depth, 4 * n, torch.float32, (n, 4))
        self.conic_radius = self._view(self.struct.conic_radius, 4 * n, torch.float32, (n, 4))
        self.rgb = self._view(self.struct.rgb, 4 * n, torch.float32, (n, 4))
        self.rect = self._view(self.struct.rect, 4 * n, torch.int32, (n, 4))
        self.count = self._view(self.struct.count, n, torch.int32, (n,))


class Bins(_Carved):
    """gs_bins for at most n Gaussians, max_pairs pairs, a width x height image.
    strategy: GS_BIN_AUTO (default), GS_BIN_PER_TILE or GS_BIN_GLOBAL (the
    same result; see include/gs.h)."""

    def __init__(self, n: int, max_pairs: int, width: int, height: int, device="cuda", strategy: int = 0):
        self.n, self.max_pairs = int(n), int(max_pairs)
        self.width, self.height = int(width), int(height)
        nbytes = int(lib().gs_bins_bytes(self.n, self.max_pairs, self.width, self.height))
        if nbytes == 0:
            raise GSError(GS_ERR_INVALID_ARG, "gs_bins_bytes")
        self.buffer = torch.empty(nbytes, dtype=torch.uint8, device=device)
        self.struct = _abi.GsBins()
        _check(lib().gs_bins_carve(ctypes.c_void_p(self.buffer.data_ptr()), self.n, self.max_pairs,
                                   self.width, self.height, ctypes.byref(self.struct)), "gs_bins_carve")
        self.struct.strategy = int(strategy)
        tiles = int(self.struct.max_tiles)
        self.tiles = tiles
        self.pair_tile = self._view(self.struct.pair_tile, self.max_pairs, torch.int32, (self.max_pairs,))
        self.pair_gid = self._view(self.struct.pair_gid, self.max_pairs, torch.int32, (self.max_pairs,))
        self.ranges = self._view(self.struct.ranges, 2 * tiles, torch.int32, (tiles, 2))
        self.n_pairs = self._view(self.struct.n_pairs, 1, torch.int64, (1,))
        self.status = self._view(self.struct.status, 1, torch.int32, (1,))


def gs_project(cam, params: dict, proj: Projected, stream=None) -> None:
    n = int(params["means"].shape[0])
    if n > proj.n:
        raise ValueError("Projected buffer too small")
    c = make_camera(cam)
    p = _params_struct(params)
    _check(lib().gs_project(ctypes.byref(c), n, ctypes.byref(p), ctypes.byref(proj.struct), _stream(stream)),
           "gs_project")


def gs_bin_and_sort(cam, n: int, proj: Projected, bins: Bins, sync: bool = True, stream=None):
    """Returns K (sync=True; raises GSError with .code GS_ERR_CAPACITY when K
    exceeds bins.max_pairs, the required K in .n_pairs) or None (sync=False)."""
    c = make_camera(cam)
    k = ctypes.c_int64(0)
    rc = lib().gs_bin_and_sort(ctypes.byref(c), int(n), ctypes.byref(proj.struct), ctypes.byref(bins.struct),
                               ctypes.byref(k) if sync else None, _stream(stream))
    if rc < 0:
        err = GSError(rc, "gs_bin_and_sort")
        err.n_pairs = int(k.value)
        raise err
    return int(k.value) if sync else None


def gs_bin_and_sort_static(cam, n: int, proj: Projected, pair_tile: torch.Tensor, pair_gid: torch.Tensor,
                           ranges: torch.Tensor, stream=None) -> int:
    """gs_bin_and_sort without a caller scratch buffer (the library's fixed
    array holds it; see include/gs.h).  Writes the sorted pairs and ranges into
    the given int32 CUDA tensors and returns K; raises GSError on any error
    (with .n_pairs set for GS_ERR_CAPACITY).  The C call cannot see the
    arrays' sizes, so they are checked here, before anything is launched:
    pair_gid must hold as many entries as pair_tile (the capacity passed on)
    and ranges two per tile of the camera's grid."""
    tiles = ((int(cam.width) + GS_TILE - 1) // GS_TILE) * ((int(cam.height) + GS_TILE - 1) // GS_TILE)
    if pair_gid.numel() < pair_tile.numel():
        raise ValueError(f"pair_gid holds {pair_gid.numel()} entries, fewer than pair_tile's {pair_tile.numel()}")
    if ranges.numel() < 2 * tiles:
        raise ValueError(f"ranges holds {ranges.numel()} entries; the camera's {tiles} tiles need {2 * tiles}")
    c = make_camera(cam)
    k = ctypes.c_int64(0)
    rc = lib().gs_bin_and_sort_static(ctypes.byref(c), int(n), ctypes.byref(proj.struct),
                                      _dev(pair_tile, "pair_tile", torch.int32),
                                      _dev(pair_gid, "pair_gid", torch.int32),
                                      _dev(ranges, "ranges", torch.int32), int(pair_tile.numel()),
                                      ctypes.byref(k), _stream(stream))
    if rc < 0:
        err = GSError(rc, "gs_bin_and_sort_static")
        err.n_pairs = int(k.value)
        raise err
    return int(k.value)


def gs_render_fwd(cam, n: int, proj: Projected, bins: Bins, image: torch.Tensor, T_final: torch.Tensor,
                  last: torch.Tensor, stream=None) -> None:
    H, W = int(cam.height), int(cam.width)
    ch = channels(cam)
    if image.numel() != H * W * ch or T_final.numel() != H * W or last.numel() != H * W:
        raise ValueError(f"output tensors must be [H,W,{ch}], [H,W], [H,W]")
    c = make_camera(cam)
    _check(lib().gs_render_fwd(ctypes.byref(c), int(n), ctypes.byref(proj.struct), ctypes.byref(bins.struct),
                               _dev(image, "image", torch.float32), _dev(T_final, "T_final", torch.float32),
                               _dev(last, "last", torch.int32), _stream(stream)), "gs_render_fwd")


def gs_render_fwd_l1(cam, n: int, proj: Projected, bins: Bins, image: torch.Tensor, T_final: torch.Tensor,
                     last: torch.Tensor, target: torch.Tensor, dL_dimage: torch.Tensor,
                     loss: torch.Tensor | None = None, stream=None) -> None:
    """gs_render_fwd plus the L1 loss (into loss, zeroed first) and its
    gradient dL_dimage in the same kernel."""
    H, W = int(cam.height), int(cam.width)
    ch = channels(cam)
    if image.numel() != H * W * ch or T_final.numel() != H * W or last.numel() != H * W:
        raise ValueError(f"output tensors must be [H,W,{ch}], [H,W], [H,W]")
    if target.numel() != H * W * ch or dL_dimage.numel() != H * W * ch:
        raise ValueError(f"target and dL_dimage must be [H,W,{ch}]")
    if loss is not None and loss.numel() < 1:
        raise ValueError("loss must hold one float")
    c = make_camera(cam)
    _check(lib().gs_render_fwd_l1(ctypes.byref(c), int(n), ctypes.byref(proj.struct), ctypes.byref(bins.struct),
                                  _dev(image, "image", torch.float32), _dev(T_final, "T_final", torch.float32),
                                  _dev(last, "last", torch.int32), _dev(target, "target", torch.float32),
                                  _dev(dL_dimage, "dL_dimage", torch.float32), _dev(loss, "loss", torch.float32),
                                  _stream(stream)), "gs_render_fwd_l1")


def gs_render_bwd(cam, n: int, params: dict, proj: Projected, bins: Bins, T_final: torch.Tensor,
                  last: torch.Tensor, dL_dimage: torch.Tensor, grad2d: torch.Tensor, grads: dict,
                  stream=None) -> None:
    if grad2d.numel() < 12 * int(n):
        raise ValueError("grad2d must hold [N,12] floats")
    if dL_dimage.numel() != int(cam.height) * int(cam.width) * channels(cam):
        raise ValueError(f"dL_dimage must be [H,W,{channels(cam)}]")
    c = make_camera(cam)
    p = _params_struct(params)
    g = _params_struct(grads, _abi.GsGrads)
    _check(lib().gs_render_bwd(ctypes.byref(c), int(n), ctypes.byref(p), ctypes.byref(proj.struct),
                               ctypes.byref(bins.struct), _dev(T_final, "T_final", torch.float32),
                               _dev(last, "last", torch.int32), _dev(dL_dimage, "dL_dimage", torch.float32),
                               _dev(grad2d, "grad2d", torch.float32), ctypes.byref(g), _stream(stream)),
           "gs_render_bwd")


def gs_render_features_fwd(cam, n: int, proj: Projected, bins: Bins, features: torch.Tensor, out: torch.Tensor,
                           stream=None) -> None:
    """Blends features [N, F] (F a multiple of 4) with the forward's weights
    into out [H, W, F] (no background)."""
    F = int(features.shape[-1]) if features.dim() == 2 else -1
    if F < 0 or out.numel() != int(cam.height) * int(cam.width) * F:
        raise ValueError("features must be [N, F] and out [H, W, F]")
    c = make_camera(cam)
    _check(lib().gs_render_features_fwd(ctypes.byref(c), int(n), ctypes.byref(proj.struct), ctypes.byref(bins.struct),
                                        _dev(features, "features", torch.float32), F,
                                        _dev(out, "out", torch.float32), _stream(stream)), "gs_render_features_fwd")


def gs_render_features_bwd(cam, n: int, params: dict, proj: Projected, bins: Bins, T_final: torch.Tensor,
                           last: torch.Tensor, features: torch.Tensor, dL_dout: torch.Tensor, grad2d: torch.Tensor,
                           dL_dfeatures: torch.Tensor, grads: dict, stream=None) -> None:
    """dL/dfeatures (overwritten) and the features' share of the raw-parameter
    gradients, added into grads (call after gs_render_bwd)."""
    F = int(features.shape[-1]) if features.dim() == 2 else -1
    if F < 0 or dL_dout.numel() != int(cam.height) * int(cam.width) * F or dL_dfeatures.shape != features.shape:
        raise ValueError("features [N, F], dL_dout [H, W, F], dL_dfeatures [N, F]")
    if grad2d.numel() < 12 * int(n):
        raise ValueError("grad2d must hold [N,12] floats")
    c = make_camera(cam)
    p = _params_struct(params)
    g = _params_struct(grads, _abi.GsGrads)
    _check(lib().gs_render_features_bwd(ctypes.byref(c), int(n), ctypes.byref(p), ctypes.byref(proj.struct),
                                        ctypes.byref(bins.struct), _dev(T_final, "T_final", torch.float32),
                                        _dev(last, "last", torch.int32), _dev(features, "features", torch.float32),
                                        F, _dev(dL_dout, "dL_dout", torch.float32),
                                        _dev(grad2d, "grad2d", torch.float32),
                                        _dev(dL_dfeatures, "dL_dfeatures", torch.float32), ctypes.byref(g),
                                        _stream(stream)), "gs_render_features_bwd")


def gs_render_stats(cam, n: int, proj: Projected, bins: Bins, last: torch.Tensor, stream=None) -> dict:
    """Exact work counts of the frame (synchronizes to read them back)."""
    counts = torch.zeros(4, dtype=torch.int64, device=last.device)
    c = make_camera(cam)
    _check(lib().gs_render_stats(ctypes.byref(c), int(n), ctypes.byref(proj.struct), ctypes.byref(bins.struct),
                                 _dev(last, "last", torch.int32), _dev(counts, "counts"), _stream(stream)),
           "gs_render_stats")
    v = counts.cpu().tolist()
    return {"fwd_visits": v[0], "contributions": v[1], "bwd_visits": v[2], "pixels": v[3]}


def gs_l1_loss_grad(image: torch.Tensor, target: torch.Tensor, dL_dimage: torch.Tensor,
                    loss: torch.Tensor | None = None, stream=None) -> None:
    if image.numel() != target.numel() or image.numel() != dL_dimage.numel():
        raise ValueError("image, target and dL_dimage must have the same size")
    _check(lib().gs_l1_loss_grad(_dev(image, "image", torch.float32), _dev(target, "target", torch.float32),
                                 image.numel(), _dev(dL_dimage, "dL_dimage", torch.float32),
                                 _dev(loss, "loss", torch.float32), _stream(stream)), "gs_l1_loss_grad")


def gs_read_status(bins: Bins, stream=None):
    """Synchronizes and returns (status code, K) of the last gs_bin_and_sort."""
    k = ctypes.c_int64(0)
    rc = lib().gs_read_status(ctypes.byref(bins.struct), ctypes.byref(k), _stream(stream))
    if rc == GS_ERR_CUDA:
        raise GSError(rc, "gs_read_status")
    return rc, int(k.value)


def gs_last_device_error(bins: Bins, stream=None) -> int:
    """Synchronizes and returns the status word of the last gs_bin_and_sort
    on these bins (GS_OK or a GS_ERR_* code)."""
    rc = lib().gs_last_device_error(ctypes.byref(bins.struct), _stream(stream))
    if rc == GS_ERR_CUDA:
        raise GSError(rc, "gs_last_device_error")
    return rc


def gs_sort_bytes(max_pairs: int, tiles: int) -> int:
    """Scratch bytes of one bin-and-sort for max_pairs pairs and `tiles` tiles."""
    return int(lib().gs_sort_bytes(int(max_pairs), int(tiles)))


def profile_begin(max_launches: int = 1 << 16) -> None:
    _check(lib().gs_profile_begin(int(max_launches)), "gs_profile_begin")


def profile_end(max_stats: int = 64) -> dict:
    """Returns {kernel name: (launches, total ms)} for launches since profile_begin."""
    arr = (_abi.GsProfileStat * max_stats)()
    m = _check(lib().gs_profile_end(arr, max_stats), "gs_profile_end")
    return {arr[i].name.decode(): (int(arr[i].launches), float(arr[i].total_ms)) for i in range(m)}


# ------------------------------------------------------------------ training
def adam_config(lr: dict, beta1: float = 0.9, beta2: float = 0.999, eps: float = 1e-8) -> _abi.GsAdamConfig:
    """gs_adam_config from a {group: learning rate} dict over PARAM_KEYS."""
    c = _abi.GsAdamConfig()
    for i, k in enumerate(PARAM_KEYS):
        c.lr[i] = float(lr[k])
    c.beta1, c.beta2, c.eps = float(beta1), float(beta2), float(eps)
    return c


def _set_struct(d: dict | None):
    return None if d is None else ctypes.byref(_params_struct(d, _abi.GsGrads))


def gs_adam_step(params: dict, slots: list, m: dict, v: dict, cfg: _abi.GsAdamConfig, step: torch.Tensor,
                 grad_scale: float = 1.0, grad_out: dict | None = None, stream=None) -> None:
    """One Adam step, in place, with g = grad_scale * sum of the slots' gradients;
    `step` is a CUDA int64 tensor of one element (steps taken), advanced by one."""
    n = int(params["means"].shape[0])
    arr = (_abi.GsGrads * max(1, len(slots)))()
    for i, sl in enumerate(slots):
        arr[i] = _params_struct(sl, _abi.GsGrads)
    _check(lib().gs_adam_step(n, _set_struct(params), arr, len(slots), float(grad_scale), _set_struct(m),
                              _set_struct(v), ctypes.byref(cfg), _dev(step, "step", torch.int64),
                              _set_struct(grad_out), _stream(stream)), "gs_adam_step")


class TrainLane:
    """The buffers of one camera chain of gs_train_step (include/gs.h
    gs_train_lane): records, pair list, image state and a gradient slot.
    `stream` None runs the lane on the step's own stream; otherwise a
    torch.cuda.Stream of its own, joined through an event."""

    def __init__(self, n: int, width: int, height: int, channels: int, max_pairs: int, own_stream: bool,
                 device="cuda"):
        self.n, self.width, self.height = int(n), int(width), int(height)
        self.device = device
        self.proj = Projected(self.n, device)
        self.bins = Bins(self.n, max_pairs, width, height, device)
        self.image = torch.empty((height, width, channels), dtype=torch.float32, device=device)
        self.dL_dimage = torch.empty_like(self.image)
        self.T_final = torch.empty((height, width), dtype=torch.float32, device=device)
        self.last = torch.empty((height, width), dtype=torch.int32, device=device)
        self.grad2d = torch.empty((max(self.n, 1), 12), dtype=torch.float32, device=device)
        self.grads = {k: torch.empty(sh, dtype=torch.float32, device=device)
                      for k, sh in _param_shapes(self.n).items()}
        self.stream = torch.cuda.Stream(device=device) if own_stream else None
        self.done = torch.cuda.Event()
        self.done.record()  # creates the event

    def regrow(self, max_pairs: int) -> None:
        self.bins = Bins(self.n, int(max_pairs), self.width, self.height, self.device)

    def struct(self, step_stream) -> _abi.GsTrainLane:
        ln = _abi.GsTrainLane()
        ln.proj = self.proj.struct
        ln.bins = self.bins.struct
        ln.image = self.image.data_ptr()
        ln.T_final = self.T_final.data_ptr()
        ln.last = self.last.data_ptr()
        ln.dL_dimage = self.dL_dimage.data_ptr()
        ln.grad2d = self.grad2d.data_ptr()
        ln.grads = _params_struct(self.grads, _abi.GsGrads)
        ln.stream = (self.stream.cuda_stream if self.stream is not None else step_stream.value) or None
        ln.done = self.done.cuda_event
        return ln


def _param_shapes(n: int) -> dict:
    return {"means": (n, 3), "log_scales": (n, 3), "quats": (n, 4), "opacity_logits": (n,), "colors": (n, 3)}


def gs_train_step(cams, params: dict, targets: torch.Tensor, lanes: list, fork: torch.cuda.Event,
                  m: dict | None, v: dict | None, cfg: _abi.GsAdamConfig | None, step: torch.Tensor | None,
                  losses: torch.Tensor | None = None, cam_stats: torch.Tensor | None = None,
                  grad_out: dict | None = None, stream=None) -> None:
    """One training step over the cameras (include/gs.h gs_train_step): camera
    b on lane b mod len(lanes), Adam on the mean gradient (cfg None: only
    grad_out).  targets is [B, H, W, C]; losses [B] float32 and cam_stats
    [B, 2] int64 (status, K) are optional outputs."""
    B = len(cams)
    n = int(params["means"].shape[0])
    if targets.dim() != 4 or targets.shape[0] != B:
        raise ValueError("targets must be [B, H, W, C]")
    carr = (_abi.GsCamera * B)(*[make_camera(c) for c in cams])
    s = _stream(stream)
    larr = (_abi.GsTrainLane * len(lanes))(*[ln.struct(s) for ln in lanes])
    _check(lib().gs_train_step(carr, B, n, _set_struct(params), _dev(targets, "targets", torch.float32), larr,
                               len(lanes), ctypes.c_void_p(fork.cuda_event), _set_struct(m), _set_struct(v),
                               None if cfg is None else ctypes.byref(cfg),
                               _dev(step, "step", torch.int64) if step is not None else None,
                               _dev(losses, "losses", torch.float32), _dev(cam_stats, "cam_stats", torch.int64),
                               _set_struct(grad_out), s), "gs_train_step")


__all__ += ["adam_config", "gs_adam_step", "TrainLane", "gs_train_step"]

from .raster import Rasterizer, Trainer, rasterize  # noqa: E402,F401

__all__ += ["Rasterizer", "Trainer", "rasterize"]
