"""Convenience layer over the C-ABI calls: buffer reuse, pair-list regrowth,
and a torch.autograd.Function.  Every step still runs in libgs.so.
"""
from __future__ import annotations

import math

import torch

from . import (GS_ERR_CAPACITY, Bins, GSError, Projected, channels, gs_bin_and_sort, gs_project, gs_render_bwd,
               gs_render_fwd)


class Rasterizer:
    """Owns the device buffers of one image size and up to n Gaussians.

    The pair list starts at ``max_pairs`` (default 16 per Gaussian) and is
    regrown by 25 % over the reported need when a frame overflows it
    ("SplatRs: We Gave the Model 4x More Pixels and It Got Worse", Lesson 2:
    a full-resolution 400k scene needs more than 16.7M pairs).
    """

    def __init__(self, n: int, width: int, height: int, max_pairs: int | None = None, device="cuda"):
        self.n, self.width, self.height = int(n), int(width), int(height)
        self.device = device
        self.proj = Projected(self.n, device)
        self.bins = Bins(self.n, int(max_pairs) if max_pairs else max(1024, 16 * self.n), width, height, device)
        P = self.width * self.height
        self.image = torch.empty((self.height, self.width, 3), dtype=torch.float32, device=device)
        self.T_final = torch.empty((self.height, self.width), dtype=torch.float32, device=device)
        self.last = torch.empty((self.height, self.width), dtype=torch.int32, device=device)
        self.grad2d = torch.empty((max(self.n, 1), 12), dtype=torch.float32, device=device)
        self.n_pairs = 0
        assert P > 0

    def _grow(self, need: int) -> None:
        self.bins = Bins(self.n, int(math.ceil(need * 1.25)) + 1024, self.width, self.height, self.device)

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
