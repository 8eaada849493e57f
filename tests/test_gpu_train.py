"""Parity of the training calls (gs_adam_step, gs_train_step) with the
oracle's training step ("Gaussian splatting in PyTorch" s7; "The backward
pass I deleted trained the model the Nano runs", "Training a smaller scene").

Adam runs in single precision against the oracle's double precision: the
moments agree to a few float roundings, the parameter step to 1e-5 of the
learning rate where the gradient's sign is certain.  The multi-camera step
is compared on a scene whose every blend and binning decision sits outside
the stated margins for every camera, with targets at least 0.01 from the
oracle's render, so both sides take the same decisions; the gradient then
follows the tolerances of the single-camera tests.
"""
import math

import numpy as np
import pytest
import torch

import gaussian_splatting_differentiable_tile_b200 as G
import oracle as O
from oracle import train as OT
from scenes import Camera, make_scene, tiny_camera

from gpu_common import GRAD_ABS, GRAD_REL, ambiguous_gaussians, ambiguous_pixels, cuda_params, grad_compare

pytestmark = pytest.mark.gpu

LR = {"means": 1e-3, "log_scales": 5e-3, "quats": 1e-3, "opacity_logits": 2.5e-2, "colors": 2.5e-3}
KEYS = G.PARAM_KEYS


def _np(d):
    return {k: v.detach().cpu().numpy().astype(np.float64) for k, v in d.items()}


def _rand_set(rng, n, scale=1.0, positive=False):
    shapes = {"means": (n, 3), "log_scales": (n, 3), "quats": (n, 4), "opacity_logits": (n,), "colors": (n, 3)}
    out = {}
    for k, sh in shapes.items():
        a = rng.normal(scale=scale, size=sh)
        out[k] = np.abs(a) if positive else a
    return {k: np.ascontiguousarray(v, np.float32) for k, v in out.items()}


# -------------------------------------------------------------------- Adam
@pytest.mark.parametrize("n", [1, 1001, 4096])
def test_adam_step_matches_oracle(n):
    """Three gradient slots summed and scaled, moments from earlier steps,
    step 5; n = 1001 leaves a scalar tail after the float4 body."""
    rng = np.random.default_rng(n)
    p0, m0 = _rand_set(rng, n), _rand_set(rng, n, 1e-3)
    v0 = _rand_set(rng, n, 1e-6, positive=True)
    slots = [_rand_set(rng, n, 10.0 ** rng.integers(-5, 0)) for _ in range(3)]
    P, M, V = cuda_params(p0), cuda_params(m0), cuda_params(v0)
    S = [cuda_params(s) for s in slots]
    out = {k: torch.empty_like(v) for k, v in P.items()}
    step = torch.tensor([4], dtype=torch.int64, device="cuda")
    cfg = G.adam_config(LR, 0.9, 0.999, 1e-8)
    G.gs_adam_step(P, S, M, V, cfg, step, grad_scale=1.0 / 3.0, grad_out=out)
    torch.cuda.synchronize()
    assert int(step.item()) == 5
    g = {k: sum(s[k].astype(np.float64) for s in slots) / 3.0 for k in KEYS}
    rp, rm, rv = OT.adam_step(p0, g, m0, v0, LR, 5)
    got_p, got_m, got_v, got_g = _np(P), _np(M), _np(V), _np(out)
    for k in KEYS:
        mag = sum(np.abs(sl[k].astype(np.float64)) for sl in slots) / 3.0
        assert np.all(np.abs(got_g[k] - g[k]) <= 3e-7 * mag), k
        np.testing.assert_allclose(got_m[k], rm[k], rtol=0, atol=2e-7 * (np.abs(m0[k]) + np.abs(g[k])).max())
        assert np.all(np.abs(got_v[k] - rv[k]) <= 3e-7 * (np.abs(v0[k]) + g[k] ** 2) + 1e-37)
        step_ref = rp[k] - p0[k]
        tol = 1e-5 * LR[k] + 2e-6 * np.abs(step_ref) + 1.2e-7 * np.abs(p0[k])
        assert np.all(np.abs((got_p[k] - p0[k]) - step_ref) <= tol), k


def test_adam_step_unaligned_groups_take_the_scalar_path():
    """Views one float into a buffer: every group except the quaternions
    (which must stay 16-byte aligned) runs the scalar loop."""
    n = 37
    rng = np.random.default_rng(1)
    p0, g0 = _rand_set(rng, n), _rand_set(rng, n, 1e-2)
    z = {k: np.zeros_like(v) for k, v in p0.items()}

    def shifted(d):
        out = {}
        for k, v in d.items():
            if k == "quats":
                out[k] = torch.from_numpy(v).cuda()
            else:
                buf = torch.empty(v.size + 1, dtype=torch.float32, device="cuda")
                out[k] = buf[1:].view(v.shape)
                out[k].copy_(torch.from_numpy(v))
        return out
    P, S, M, V = shifted(p0), shifted(g0), shifted(z), shifted(z)
    step = torch.zeros(1, dtype=torch.int64, device="cuda")
    G.gs_adam_step(P, [S], M, V, G.adam_config(LR), step)
    torch.cuda.synchronize()
    rp, _, _ = OT.adam_step(p0, g0, z, z, LR, 1)
    got = _np(P)
    for k in KEYS:
        assert np.all(np.abs((got[k] - p0[k]) - (rp[k] - p0[k])) <= 1e-5 * LR[k] + 1.2e-7 * np.abs(p0[k])), k


def test_adam_step_in_a_graph_advances_the_device_counter():
    """Captured once and replayed: the step count lives on the device, so
    each replay applies the next bias correction (constant gradient: every
    step has the size lr g / (|g| + eps))."""
    n = 64
    rng = np.random.default_rng(2)
    p0, g0 = _rand_set(rng, n), _rand_set(rng, n, 0.1)
    P = cuda_params(p0)
    S = cuda_params(g0)
    M = {k: torch.zeros_like(v) for k, v in P.items()}
    V = {k: torch.zeros_like(v) for k, v in P.items()}
    step = torch.zeros(1, dtype=torch.int64, device="cuda")
    cfg = G.adam_config(LR, 0.8, 0.95, 1e-6)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        G.gs_adam_step(P, [S], M, V, cfg, step, stream=s)  # warm-up outside the capture: step 1
        s.synchronize()
        with torch.cuda.graph(graph, stream=s):
            G.gs_adam_step(P, [S], M, V, cfg, step, stream=s)
    for _ in range(4):
        graph.replay()
    torch.cuda.synchronize()
    assert int(step.item()) == 5
    got = _np(P)
    for k in KEYS:
        expect = p0[k] - 5 * LR[k] * g0[k] / (np.abs(g0[k]) + 1e-6)
        assert np.all(np.abs(got[k] - expect) <= 1e-5 * LR[k] * 5 + 5e-7 * np.abs(p0[k])), k


def test_adam_step_argument_errors():
    P = cuda_params(_rand_set(np.random.default_rng(0), 4))
    step = torch.zeros(1, dtype=torch.int64, device="cuda")
    with pytest.raises(G.GSError) as ei:
        G.gs_adam_step(P, [], P, P, G.adam_config(LR), step)
    assert ei.value.code == G.GS_ERR_INVALID_ARG
    bad = dict(LR, colors=-1.0)
    with pytest.raises(G.GSError) as ei:
        G.gs_adam_step(P, [P], P, P, G.adam_config(bad), step)
    assert ei.value.code == G.GS_ERR_INVALID_ARG
    with pytest.raises(G.GSError) as ei:
        G.gs_adam_step(P, [P], P, P, G.adam_config(LR, beta1=1.0), step)
    assert ei.value.code == G.GS_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert int(step.item()) == 0  # nothing launched


# ----------------------------------------------------------- training step
def _turned(cam, deg):
    """The camera turned about the world y axis through the origin."""
    a = math.radians(deg)
    Ry = np.array([[math.cos(a), 0, math.sin(a)], [0, 1, 0], [-math.sin(a), 0, math.cos(a)]])
    V = np.array(cam.viewmat, np.float64).copy()
    V[:3, :3] = V[:3, :3] @ Ry
    return Camera(V.astype(np.float32), cam.fx, cam.fy, cam.cx, cam.cy, cam.width, cam.height, cam.near_z,
                  cam.bg)


def _clean_scene(n=240, seed0=100, flags=0):
    """Three 200 x 150 cameras (13 x 10 tiles, ragged last column and row)
    and the first seeded scene with no decision inside its margin for any of
    them."""
    base = tiny_camera(200, 150, 180.0, distance=3.0, bg=(0.1, 0.2, 0.3))
    cams = [base, _turned(base, 10.0), _turned(base, -14.0)]
    for c in cams:
        c.flags = flags
    for seed in range(seed0, seed0 + 100):
        params = make_scene("tiny", n=n, seed=seed)
        ok = True
        for c in cams:
            p = O.project(params, c)
            if ambiguous_gaussians(p).any() or ambiguous_pixels(O.render(p, c), with_clamp=True).any():
                ok = False
                break
        if ok:
            return cams, params
    raise RuntimeError("no clean scene")


def _targets_away_from(params, cams, seed=3):
    """Seeded U(0, 1) targets with every value moved at least 0.01 from the
    oracle's render, so that no sign of image - target is in doubt."""
    rng = np.random.default_rng(seed)
    out = []
    for c in cams:
        img = O.render(O.project(params, c), c)["image"]
        t = rng.uniform(0.0, 1.0, img.shape)
        near = np.abs(t - img) < 0.01
        t = np.where(near, img + np.where(t >= img, 0.01, -0.01) * 1.5, t)
        out.append(t)
    return out


def _step_bound(params, cams, targets):
    """Per-element scale of the mean gradient's rounding (the oracle's
    sum of absolute terms, averaged like the gradient)."""
    tot = None
    for c, tg in zip(cams, targets):
        p = O.project(params, c)
        img = O.render(p, c)["image"]
        _, dl = OT.l1_loss_grad(img, tg)
        _, g2_abs = O.render_bwd(p, c, dl)
        b = O.grad_bound(params, c, g2_abs)
        tot = b if tot is None else {k: tot[k] + b[k] for k in KEYS}
    return {k: v / len(cams) for k, v in tot.items()}


@pytest.mark.parametrize("lanes", [1, 2, 3])
def test_train_step_matches_oracle(lanes):
    cams, params = _clean_scene()
    targets = _targets_away_from(params, cams)
    n = params["means"].shape[0]
    tr = G.Trainer(n, 200, 150, lanes=lanes, lr=LR)
    P = cuda_params(params)
    T = torch.from_numpy(np.ascontiguousarray(np.stack(targets), np.float32)).cuda()
    losses = tr.step(cams, P, T, check=True).cpu().numpy()
    assert int(tr.step_count.item()) == 1
    tg32 = [t.astype(np.float32).astype(np.float64) for t in targets]
    ref = OT.train_step(params, cams, tg32, {k: np.zeros_like(v, np.float64) for k, v in params.items()},
                        {k: np.zeros_like(v, np.float64) for k, v in params.items()}, LR, 1)
    np.testing.assert_allclose(losses, ref["losses"], rtol=1e-5)
    bound = _step_bound(params, cams, tg32)
    grads = _np(tr.grads)
    for k in KEYS:
        grad_compare(grads[k], ref["grads"][k], bound[k], k)
    # Adam's first step is lr g / (|g| + eps): where the gradient's sign is
    # certain the step agrees to 1e-5 lr; elsewhere it is at most lr
    got = _np(P)
    n_sure = n_all = 0
    for k in KEYS:
        g = ref["grads"][k]
        unc = GRAD_ABS + GRAD_REL * np.maximum(np.abs(g), bound[k])
        sure = np.abs(g) > 10 * unc
        d_gpu = got[k] - params[k]
        d_ref = ref["params"][k] - params[k]
        assert np.all(np.abs(d_gpu - d_ref)[sure] <= 1e-5 * LR[k] + 1.2e-7 * np.abs(params[k][sure])), k
        assert np.all(np.abs(d_gpu) <= LR[k] * (1 + 1e-5) + 1.2e-7 * np.abs(params[k])), k
        n_sure += int(sure.sum())
        n_all += sure.size
    assert n_sure > 0.3 * n_all, (n_sure, n_all)


def test_train_step_depth_channel_and_gradient_only():
    """With GS_FLAG_DEPTH the targets carry a fourth channel; cfg None
    leaves the parameters alone and only writes the mean gradient."""
    cams, params = _clean_scene(flags=G.GS_FLAG_DEPTH)
    targets = _targets_away_from(params, cams)  # the depth channel too, like the colours
    n = params["means"].shape[0]
    tr = G.Trainer(n, 200, 150, lanes=2, channels=4, lr=LR)
    P = cuda_params(params)
    T = torch.from_numpy(np.ascontiguousarray(np.stack(targets), np.float32)).cuda()
    losses = tr.step(cams, P, T, check=True, adam=False).cpu().numpy()
    assert int(tr.step_count.item()) == 0
    got_p = _np(P)
    for k in KEYS:
        np.testing.assert_array_equal(got_p[k], params[k].astype(np.float64))
    tg32 = [t.astype(np.float32).astype(np.float64) for t in targets]
    ref = OT.train_step(params, cams, tg32, None, None, LR, 1, adam=False)
    np.testing.assert_allclose(losses, ref["losses"], rtol=1e-5)
    bound = _step_bound(params, cams, tg32)
    grads = _np(tr.grads)
    for k in KEYS:
        grad_compare(grads[k], ref["grads"][k], bound[k], k)


def test_train_step_reports_an_overflowed_pair_list():
    cams, params = _clean_scene()
    n = params["means"].shape[0]
    tr = G.Trainer(n, 200, 150, lanes=2, max_pairs=64, lr=LR)
    P = cuda_params(params)
    T = torch.zeros((3, 150, 200, 3), dtype=torch.float32, device="cuda")
    with pytest.raises(G.GSError) as ei:
        tr.step(cams, P, T, check=True)
    assert ei.value.code == G.GS_ERR_CAPACITY
    st = tr.cam_stats.cpu().numpy()
    assert np.all(st[:, 0] == G.GS_ERR_CAPACITY) and np.all(st[:, 1] > 64)
    # regrown from the reported need, the step succeeds
    need = tr.fit_pairs(cams, cuda_params(params))
    assert need == int(st[:, 1].max()) or need > 64
    tr.step(cams, cuda_params(params), T, check=True)


def test_train_step_argument_errors():
    cams, params = _clean_scene()
    n = params["means"].shape[0]
    tr = G.Trainer(n, 200, 150, lanes=1, lr=LR)
    P = cuda_params(params)
    T = torch.zeros((3, 150, 200, 3), dtype=torch.float32, device="cuda")
    odd = tiny_camera(64, 64, 60.0)
    with pytest.raises(G.GSError) as ei:
        tr.step(cams[:2] + [odd], P, T[:3])
    assert ei.value.code == G.GS_ERR_INVALID_ARG
    assert int(tr.step_count.item()) == 0


def test_training_equivalence_over_ten_steps():
    """"Throughput: the tile rasterizer" gates the tiled trainer on its PSNR
    divergence from the naive one over a run.  Here a student (the clean
    scene perturbed) is fitted to the teacher's renders from three cameras
    for ten Adam steps on each side: the per-step mean L1 losses agree to
    1e-4 relative and the final PSNR of the two students against the
    targets to 0.01 dB.  Single-precision gradients differ from the oracle's
    by about 1e-6 relative; Adam turns that into the same relative change of
    each step except where a gradient is near zero, where a step of up to lr
    may take either sign."""
    cams, teacher = _clean_scene()
    targets = [O.render(O.project(teacher, c), c)["image"].astype(np.float32) for c in cams]
    rng = np.random.default_rng(4)
    student = {k: np.ascontiguousarray(v + rng.normal(scale=0.03, size=v.shape), np.float32)
               for k, v in teacher.items()}
    n = student["means"].shape[0]
    lr = {"means": 2e-3, "log_scales": 1e-2, "quats": 5e-3, "opacity_logits": 2.5e-2, "colors": 1e-2}
    tr = G.Trainer(n, 200, 150, lanes=3, lr=lr)
    P = cuda_params(student)
    T = torch.from_numpy(np.ascontiguousarray(np.stack(targets))).cuda()
    ref_p = {k: v.astype(np.float64) for k, v in student.items()}
    m = {k: np.zeros_like(v) for k, v in ref_p.items()}
    v = {k: np.zeros_like(x) for k, x in ref_p.items()}
    tg64 = [t.astype(np.float64) for t in targets]
    gpu_l, ref_l = [], []
    for t in range(1, 11):
        gpu_l.append(float(tr.step(cams, P, T).mean().item()))
        out = OT.train_step(ref_p, cams, tg64, m, v, lr, t)
        ref_l.append(float(np.mean(out["losses"])))
        ref_p, m, v = out["params"], out["m"], out["v"]
    np.testing.assert_allclose(gpu_l, ref_l, rtol=1e-4)
    assert ref_l[-1] < ref_l[0]
    gp = _np(P)
    ps_gpu = np.mean([OT.psnr(O.render(O.project(gp, c), c)["image"], tg) for c, tg in zip(cams, tg64)])
    ps_ref = np.mean([OT.psnr(O.render(O.project(ref_p, c), c)["image"], tg) for c, tg in zip(cams, tg64)])
    assert abs(ps_gpu - ps_ref) <= 0.01, (ps_gpu, ps_ref)
