"""Parity of the feature-channel calls (gs_render_features_fwd/bwd) with the
oracle ("Gaussian splatting in PyTorch", s5: channels of any kind blend
alike; s6: their backward).  Stage-fed like the colour tests: the oracle's
single-precision records, the GPU's own bins and forward state."""
import numpy as np
import pytest
import torch

import gaussian_splatting_differentiable_tile_b200 as G
import oracle as O
from oracle import features as OF

from gpu_common import IMG_TOL, ambiguous_pixels, cuda_params, grad_compare
from test_gpu_parity import SCENES, VARIANTS, _fwd_stage_fed

pytestmark = pytest.mark.gpu


def _features(n, F, seed=0):
    return np.ascontiguousarray(np.random.default_rng(seed).uniform(-1.0, 1.0, (n, F)), np.float32)


# F = 8 and 32: passes of eight channels; 4: one pass of four; 12: one of
# each
@pytest.mark.parametrize("scene,F,flags", [("ragged", 8, 0), ("student3k", 4, 0), ("ragged", 32, 0),
                                           ("student3k", 12, 0), ("ragged", 8, VARIANTS | G.GS_FLAG_TIGHT_TILES)])
def test_features_fwd_and_bwd_match_oracle(scene, F, flags):
    cam, params = SCENES[scene]()
    cam.flags = flags
    n = params["means"].shape[0]
    rec, proj, bins, K, image, T, last, ref = _fwd_stage_fed(cam, params)
    feats = _features(n, F)
    Fd = torch.from_numpy(feats).cuda()
    out = torch.full((cam.height, cam.width, F), float("nan"), device="cuda")
    G.gs_render_features_fwd(cam, n, proj, bins, Fd, out)
    torch.cuda.synchronize()
    ref_out = OF.render_features(rec, cam, feats.astype(np.float64))
    keep = ~ambiguous_pixels(ref, with_clamp=True)
    d = np.abs(out.cpu().numpy() - ref_out).max(axis=2)
    assert d[keep].max() <= IMG_TOL, d[keep].max()
    assert np.all(np.isfinite(out.cpu().numpy()))
    # backward: the colour share with dL/dimage = 0 is exactly zero, then the
    # features add theirs
    rng = np.random.default_rng(1)
    dl = np.where(keep[..., None], rng.normal(size=(cam.height, cam.width, F)), 0.0).astype(np.float32)
    P = cuda_params(params)
    grads = {k: torch.full_like(v, float("nan")) for k, v in P.items()}
    grad2d = torch.empty((n, 12), device="cuda")
    zero = torch.zeros((cam.height, cam.width, G.channels(cam)), device="cuda")
    Td, Ld = torch.from_numpy(T).cuda(), torch.from_numpy(last).cuda()
    G.gs_render_bwd(cam, n, P, proj, bins, Td, Ld, zero, grad2d, grads)
    dfeat = torch.full_like(Fd, float("nan"))
    G.gs_render_features_bwd(cam, n, P, proj, bins, Td, Ld, Fd, torch.from_numpy(dl).cuda(), grad2d, dfeat, grads)
    torch.cuda.synchronize()
    dfeat_ref, g2_ref, g2_abs = OF.render_features_bwd(rec, cam, feats.astype(np.float64), dl.astype(np.float64))
    dfeat_abs, _, _ = OF.render_features_bwd(rec, cam, np.abs(feats.astype(np.float64)),
                                             np.abs(dl.astype(np.float64)))
    grad_compare(dfeat.cpu().numpy(), dfeat_ref, dfeat_abs, "dL/dfeatures")
    pad = np.zeros((n, 3))
    nc = G.channels(cam)
    g2_full = np.hstack([g2_ref, pad] + ([np.zeros((n, 1))] if nc == 4 else []))
    g2a_full = np.hstack([g2_abs, pad] + ([np.zeros((n, 1))] if nc == 4 else []))
    raw_ref = O.project_bwd(params, cam, g2_full)
    bound = O.grad_bound(params, cam, g2a_full)
    got = {k: v.cpu().numpy() for k, v in grads.items()}
    for k in G.PARAM_KEYS:
        grad_compare(got[k], raw_ref[k], bound[k], k)
    assert np.all(got["colors"] == 0.0)


def test_features_argument_errors():
    cam, params = SCENES["tiny"]()
    n = params["means"].shape[0]
    rec, proj, bins, K, image, T, last, ref = _fwd_stage_fed(cam, params)
    out = torch.empty((cam.height, cam.width, 6), device="cuda")
    with pytest.raises(G.GSError) as ei:
        G.gs_render_features_fwd(cam, n, proj, bins, torch.zeros((n, 6), device="cuda"), out)
    assert ei.value.code == G.GS_ERR_INVALID_ARG
    buf = torch.zeros(n * 4 + 1, device="cuda")
    out4 = torch.empty((cam.height, cam.width, 4), device="cuda")
    with pytest.raises(G.GSError) as ei:
        G.gs_render_features_fwd(cam, n, proj, bins, buf[1:].view(n, 4), out4)
    assert ei.value.code == G.GS_ERR_ALIGNMENT
