"""Convenience layer over the C-ABI calls: buffer reuse, pair-list regrowth,
and a torch.autograd.Function.  Every step still runs in libgs.so.
"""
from __future__ import annotations

import math

import torch

from . import (GS_ERR_CAPACITY, PARAM_KEYS, Bins, GSError, Projected, TrainLane, adam_config, channels,
               gs_adam_step, gs_bin_and_sort, gs_project, gs_render_bwd, gs_render_fwd, gs_train_step)


class Rasterizer:
    """Owns the device buffers of one image size and up to n Gaussians.

    The pair list starts at ``max_pairs`` (default 16 per Gaussian) and is
    regrown by 25 % over the reported need when a frame overflows it
    ("SplatRs: We Gave the Model 4x More Pixels and It Got Worse", Lesson 2:
    a full-resolution 400k scene needs more than 16.7M pairs).
    """

    def __init__(self, n: int, width: int, height: int, max_pairs: int | None = None, device="cuda",
                 strategy: int = 0):
        self.n, self.width, self.height = int(n), int(width), int(height)
        self.device = device
        self.strategy = int(strategy)  # gs_bins.strategy (GS_BIN_*)
        self.proj = Projected(self.n, device)
        self.bins = Bins(self.n, int(max_pairs) if max_pairs else max(1024, 16 * self.n), width, height, device,
                         strategy=self.strategy)
        P = self.width * self.height
        self.image = torch.empty((self.height, self.width, 3), dtype=torch.float32, device=device)
        self.T_final = torch.empty((self.height, self.width), dtype=torch.float32, device=device)
        self.last = torch.empty((self.height, self.width), dtype=torch.int32, device=device)
        self.grad2d = torch.empty((max(self.n, 1), 12), dtype=torch.float32, device=device)
        self.n_pairs = 0
        assert P > 0

    def _grow(self, need: int) -> None:
        self.bins = Bins(self.n, int(math.ceil(need * 1.25)) + 1024, self.width, self.height, self.device,
                         strategy=self.strategy)

    def _global_for(self, capacity: int, n: int) -> bool:
        """The automatic binning strategy's choice for a pair list of this
        capacity (include/gs.h GS_BIN_AUTO)."""
        return capacity >= 1024 * self.bins.tiles and n <= capacity

    def _fit(self, need: int, n: int) -> bool:
        """With the automatic strategy, re-carves the pair list near the frame's
        need when its current capacity would pick the other strategy than a
        list sized to the frame (a roomy default would send short tile lists
        down the long-list path).  Returns whether it re-carved."""
        if self.strategy != 0:
            return False
        fitted = int(math.ceil(need * 1.25)) + 1024
        if self._global_for(self.bins.max_pairs, n) == self._global_for(fitted, n):
            return False
        self._grow(need)
        return True

    def forward(self, cam, params: dict, sync: bool = True) -> torch.Tensor:
        """Renders into self.image (returned).  With sync=False no host
        synchronization happens and the pair list must already be large
        enough (errors land in self.bins.status)."""
        n = int(params["means"].shape[0])
        gs_project(cam, params, self.proj)
        if sync:
            try:
                self.n_pairs = gs_bin_and_sort(cam, n, self.proj, self.bins, sync=True)
            except GSError as e:
                if e.code != GS_ERR_CAPACITY:
                    raise
                self._grow(e.n_pairs)
                self.n_pairs = gs_bin_and_sort(cam, n, self.proj, self.bins, sync=True)
            if self._fit(self.n_pairs, n):
                self.n_pairs = gs_bin_and_sort(cam, n, self.proj, self.bins, sync=True)
        else:
            gs_bin_and_sort(cam, n, self.proj, self.bins, sync=False)
        ch = channels(cam)
        if self.image.shape[-1] != ch:  # RGB, or RGB + depth with GS_FLAG_DEPTH
            self.image = torch.empty((self.height, self.width, ch), dtype=torch.float32, device=self.device)
        gs_render_fwd(cam, n, self.proj, self.bins, self.image, self.T_final, self.last)
        return self.image

    def backward(self, cam, params: dict, dL_dimage: torch.Tensor, grads: dict | None = None) -> dict:
        n = int(params["means"].shape[0])
        if grads is None:
            grads = {k: torch.empty_like(v) for k, v in params.items()}
        gs_render_bwd(cam, n, params, self.proj, self.bins, self.T_final, self.last,
                      dL_dimage.contiguous(), self.grad2d, grads)
        return grads


class _RasterizeFn(torch.autograd.Function):
    @staticmethod
    def forward(ctx, means, log_scales, quats, opacity_logits, colors, cam, rasterizer):
        params = {"means": means.contiguous(), "log_scales": log_scales.contiguous(),
                  "quats": quats.contiguous(), "opacity_logits": opacity_logits.contiguous(),
                  "colors": colors.contiguous()}
        image = rasterizer.forward(cam, params).clone()
        ctx.cam, ctx.rasterizer, ctx.params = cam, rasterizer, params
        return image

    @staticmethod
    def backward(ctx, grad_image):
        g = ctx.rasterizer.backward(ctx.cam, ctx.params, grad_image.contiguous())
        return g["means"], g["log_scales"], g["quats"], g["opacity_logits"], g["colors"], None, None


def rasterize(means, log_scales, quats, opacity_logits, colors, cam, rasterizer: Rasterizer) -> torch.Tensor:
    """Differentiable render of one camera; the backward recomputes the blend
    weights from the saved per-pixel final transmittance and last index.  The
    rasterizer's buffers hold the forward state until backward runs, so one
    rasterizer serves one forward/backward pair at a time."""
    return _RasterizeFn.apply(means, log_scales, quats, opacity_logits, colors, cam, rasterizer)


# Learning rates of "Gaussian splatting in PyTorch" s7 (3DGS's latest code):
# means 1.6e-4 x the scene extent (decayed over training; the caller scales
# it), scales 5e-3, opacities 2.5e-2, quaternions 1e-3.  The pages give none
# for colours; 2.5e-3 is used.
DEFAULT_LR = {"means": 1.6e-4, "log_scales": 5e-3, "quats": 1e-3, "opacity_logits": 2.5e-2, "colors": 2.5e-3}


class Trainer:
    """A batched multi-camera training step with Adam ("Gaussian splatting in
    PyTorch" s7; "Training a smaller scene": one model fitted to renders from
    many cameras).  Owns `lanes` camera chains that run concurrently (lane 0
    on the caller's stream, the others on streams of their own), Adam's
    moments and its device step counter.  Every step is one gs_train_step
    call, so it can be captured in a CUDA graph."""

    def __init__(self, n: int, width: int, height: int, lanes: int = 2, channels: int = 3,
                 max_pairs: int | None = None, lr: dict | None = None, betas=(0.9, 0.999), eps: float = 1e-8,
                 device="cuda"):
        self.n, self.width, self.height, self.channels = int(n), int(width), int(height), int(channels)
        self.device = device
        mp = int(max_pairs) if max_pairs else max(1024, 16 * self.n)
        self.lanes = [TrainLane(self.n, width, height, channels, mp, own_stream=(i > 0), device=device)
                      for i in range(int(lanes))]
        self.cfg = adam_config(lr or DEFAULT_LR, betas[0], betas[1], eps)
        shapes = {k: v.shape for k, v in self.lanes[0].grads.items()}
        self.m = {k: torch.zeros(shapes[k], dtype=torch.float32, device=device) for k in PARAM_KEYS}
        self.v = {k: torch.zeros(shapes[k], dtype=torch.float32, device=device) for k in PARAM_KEYS}
        self.step_count = torch.zeros(1, dtype=torch.int64, device=device)
        self.fork = torch.cuda.Event()
        self.fork.record()
        # the mean gradient, one flat buffer (one all-reduce across GPUs);
        # each group starts on a 16-byte boundary
        self.grads_flat, self.grads = _flat_views(shapes, device)
        self.losses = None
        self.cam_stats = None

    def fit_pairs(self, cams, params: dict) -> int:
        """Sizes every lane's pair list for these cameras (one synchronizing
        binning per camera); returns the largest K."""
        need = 0
        lane = self.lanes[0]
        n = int(params["means"].shape[0])
        for c in cams:
            gs_project(c, params, lane.proj)
            try:
                k = gs_bin_and_sort(c, n, lane.proj, lane.bins, sync=True)
            except GSError as e:
                if e.code != GS_ERR_CAPACITY:
                    raise
                k = e.n_pairs
            need = max(need, k)
        if need > self.lanes[0].bins.max_pairs:
            for ln in self.lanes:
                ln.regrow(int(math.ceil(need * 1.25)) + 1024)
        return need

    def step(self, cams, params: dict, targets, check: bool = False, adam: bool = True, stream=None,
             group=None):
        """One step over the cameras (targets [B, H, W, C]); updates params in
        place (adam=True) and returns the per-camera losses (a device tensor).
        self.grads receives the mean gradient.  check=True synchronizes and
        raises GSError(GS_ERR_CAPACITY) if a camera overflowed its pair list
        (its image was then background only; Adam has already run).

        With a torch.distributed process group of several ranks (data
        parallel: every rank its own B cameras, the same parameters), the
        ranks' mean gradients are summed by one all-reduce and Adam applies
        their mean, so every rank takes the same step."""
        B = len(cams)
        if self.losses is None or self.losses.numel() != B:
            self.losses = torch.zeros(B, dtype=torch.float32, device=self.device)
            self.cam_stats = torch.zeros((B, 2), dtype=torch.int64, device=self.device)
        world = _world(group)
        if world > 1 and adam:
            data_parallel_step(
                lambda: gs_train_step(cams, params, targets, self.lanes, self.fork, None, None, None, None,
                                      self.losses, self.cam_stats, self.grads, stream),
                lambda scale: gs_adam_step(params, [self.grads], self.m, self.v, self.cfg, self.step_count,
                                           grad_scale=scale, stream=stream),
                self.grads_flat, group)
        else:
            gs_train_step(cams, params, targets, self.lanes, self.fork, self.m if adam else None,
                          self.v if adam else None, self.cfg if adam else None,
                          self.step_count if adam else None, self.losses, self.cam_stats, self.grads, stream)
        if check:
            st = self.cam_stats.cpu()
            bad = [b for b in range(B) if int(st[b, 0]) != 0]
            if bad:
                err = GSError(int(st[bad[0], 0]), f"gs_train_step (cameras {bad})")
                err.n_pairs = int(st[:, 1].max())
                raise err
        return self.losses


def _flat_views(shapes: dict, device):
    """One float32 buffer holding an array per group, each starting on a
    16-byte boundary; returns (buffer, {group: view})."""
    offs, off = {}, 0
    for k in PARAM_KEYS:
        offs[k] = off
        off += (math.prod(shapes[k]) + 3) // 4 * 4
    flat = torch.zeros(max(off, 4), dtype=torch.float32, device=device)
    return flat, {k: flat[offs[k]:offs[k] + math.prod(shapes[k])].view(shapes[k]) for k in PARAM_KEYS}


def _world(group) -> int:
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized():
        return 1
    return dist.get_world_size(group)


def data_parallel_step(local_step, adam_step, grads_flat, group=None) -> None:
    """Data-parallel training step: local_step() writes this rank's mean
    gradient into grads_flat; one all-reduce sums the ranks' gradients; then
    adam_step(1 / world) applies their mean.  Every rank makes the same
    collective call in the same order."""
    import torch.distributed as dist
    local_step()
    dist.all_reduce(grads_flat, op=dist.ReduceOp.SUM, group=group)
    adam_step(1.0 / dist.get_world_size(group))
