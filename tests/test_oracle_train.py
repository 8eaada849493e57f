"""Pins of the oracle's training step ("Gaussian splatting in PyTorch", s7:
render, L1 against the target, backward, Adam over the raw parameters with a
learning rate per group; "The backward pass I deleted trained the model the
Nano runs", "Training a smaller scene": one student fitted from several
cameras).

Adam is pinned against torch.optim.Adam in float64 (the library routine the
page uses) and against closed forms that hold for any correct Adam; the
multi-camera step against finite differences of the mean loss and against
the single-camera step."""
import math

import numpy as np
import pytest

import oracle as O
from oracle import train as OT
from scenes import Camera

from test_oracle_gradients import _clean, _scene

LR = {"means": 1e-3, "log_scales": 5e-3, "quats": 1e-3, "opacity_logits": 2.5e-2, "colors": 2.5e-3}


def _rand_params(rng, n):
    return {"means": rng.normal(size=(n, 3)), "log_scales": rng.normal(size=(n, 3)),
            "quats": rng.normal(size=(n, 4)), "opacity_logits": rng.normal(size=n),
            "colors": rng.uniform(size=(n, 3))}


def _zeros_like(p):
    return {k: np.zeros_like(v) for k, v in p.items()}


def test_l1_closed_form():
    img = np.array([[[0.2], [0.5]], [[0.7], [0.7]]])
    tgt = np.array([[[0.1], [0.5]], [[0.9], [0.6]]])
    loss, g = OT.l1_loss_grad(img, tgt)
    assert abs(loss - 0.1) < 1e-15
    np.testing.assert_array_equal(g.ravel(), [0.25, 0.0, -0.25, 0.25])  # sign(0) = 0


def test_adam_matches_torch_float64():
    """Five steps with a learning rate per group, random gradients, against
    torch.optim.Adam (the page's optimiser) in float64."""
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(3)
    p0 = _rand_params(rng, 7)
    tp = {k: torch.tensor(v, dtype=torch.float64, requires_grad=True) for k, v in p0.items()}
    opt = torch.optim.Adam([{"params": [tp[k]], "lr": LR[k]} for k in OT.PARAM_KEYS], betas=(0.9, 0.999),
                           eps=1e-8)
    p, m, v = p0, _zeros_like(p0), _zeros_like(p0)
    for t in range(1, 6):
        g = {k: rng.normal(scale=10.0 ** rng.integers(-6, 2), size=x.shape) for k, x in p0.items()}
        for k in OT.PARAM_KEYS:
            tp[k].grad = torch.tensor(g[k], dtype=torch.float64)
        opt.step()
        p, m, v = OT.adam_step(p, g, m, v, LR, t)
        for k in OT.PARAM_KEYS:
            np.testing.assert_allclose(p[k], tp[k].detach().numpy(), rtol=1e-13, atol=1e-15)
            st = opt.state[tp[k]]
            np.testing.assert_allclose(m[k], st["exp_avg"].numpy(), rtol=1e-13, atol=1e-300)
            np.testing.assert_allclose(v[k], st["exp_avg_sq"].numpy(), rtol=1e-13, atol=1e-300)


def test_adam_first_step_is_lr_sized():
    """s7: an Adam step changes each raw value by about lr whatever the
    gradient's size: at t = 1, m_hat = g and v_hat = g^2 exactly, so the
    step is lr g / (|g| + eps).  In log space that is the same relative
    change exp(-+lr) of a 1 mm and a 1 m scale."""
    p = {k: np.zeros(2) for k in OT.PARAM_KEYS}
    p["log_scales"] = np.log(np.array([0.001, 1.0]))
    g = {k: np.array([1e-3, -50.0]) for k in OT.PARAM_KEYS}
    g["log_scales"] = np.array([-2e-4, -7.0])  # both shrink-gradients negative: scales grow
    out, _, _ = OT.adam_step(p, g, _zeros_like(p), _zeros_like(p), LR, 1)
    for k in OT.PARAM_KEYS:
        np.testing.assert_allclose(out[k] - p[k], -LR[k] * g[k] / (np.abs(g[k]) + 1e-8), rtol=1e-12)
    ratio = np.exp(out["log_scales"]) / np.exp(p["log_scales"])
    np.testing.assert_allclose(ratio, math.exp(LR["log_scales"]), rtol=1e-4)


def test_adam_bias_correction_constant_gradient():
    """Under a constant gradient the bias-corrected moments equal g and g^2
    at every step, so every step has the same size; a missing or wrong
    correction makes the early steps differ."""
    rng = np.random.default_rng(5)
    p0 = _rand_params(rng, 3)
    g = {k: rng.normal(size=v.shape) for k, v in p0.items()}
    p, m, v = p0, _zeros_like(p0), _zeros_like(p0)
    for t in range(1, 12):
        q, m, v = OT.adam_step(p, g, m, v, LR, t, beta1=0.8, beta2=0.95, eps=1e-6)
        for k in OT.PARAM_KEYS:
            np.testing.assert_allclose(q[k] - p[k], -LR[k] * g[k] / (np.abs(g[k]) + 1e-6), rtol=1e-9, atol=1e-15)
        p = q


def _second_camera(cam, angle_deg=12.0):
    """The first camera turned about the world y axis through the origin."""
    a = math.radians(angle_deg)
    Ry = np.array([[math.cos(a), 0, math.sin(a)], [0, 1, 0], [-math.sin(a), 0, math.cos(a)]])
    V = np.array(cam.viewmat, np.float64).copy()
    V[:3, :3] = V[:3, :3] @ Ry
    return Camera(V.astype(np.float32), cam.fx, cam.fy, cam.cx, cam.cy, cam.width, cam.height, cam.near_z,
                  cam.bg)


def _two_camera_scene(seed0=40):
    for seed in range(seed0, seed0 + 300):
        cam, params = _scene(seed, n=6, bg=(0.2, 0.3, 0.1))
        cam2 = _second_camera(cam)
        if _clean(cam, params) and _clean(cam2, params):
            return [cam, cam2], params
    raise RuntimeError("no clean two-camera scene")


def _targets(cams, seed=7):
    rng = np.random.default_rng(seed)
    return [rng.uniform(0, 1, (c.height, c.width, 3)) for c in cams]


def test_train_step_of_identical_cameras_equals_one_camera():
    cams, params = _two_camera_scene()
    tg = _targets(cams[:1])[0]
    one = OT.train_step(params, cams[:1], [tg], None, None, LR, 1, adam=False)
    three = OT.train_step(params, [cams[0]] * 3, [tg] * 3, None, None, LR, 1, adam=False)
    assert three["losses"] == [one["losses"][0]] * 3
    for k in OT.PARAM_KEYS:
        np.testing.assert_allclose(three["grads"][k], one["grads"][k], rtol=1e-14, atol=1e-18)


def test_train_step_gradient_matches_finite_differences():
    """The step's gradient is that of the mean of the cameras' L1 losses:
    central differences of that mean through the whole oracle (projection,
    blend, L1) on every raw parameter of two Gaussians.  The scene keeps
    every decision at least 1e-4 from its threshold and every value at least
    0.01 from its target, so a step of 1e-6 flips nothing."""
    cams, params = _two_camera_scene()
    rng = np.random.default_rng(8)
    targets = []
    for c in cams:  # every value at least 0.01 above or below the render
        img = O.render(O.project(params, c), c, nthreads=2)["image"]
        targets.append(img + rng.choice([-1.0, 1.0], img.shape) * rng.uniform(0.01, 0.3, img.shape))
    out = OT.train_step(params, cams, targets, None, None, LR, 1, adam=False)

    def mean_loss(p):
        return np.mean([OT.l1_loss_grad(O.render(O.project(p, c), c, nthreads=2)["image"], tg)[0]
                        for c, tg in zip(cams, targets)])

    h = 1e-6
    checked = 0
    for k in OT.PARAM_KEYS:
        for idx in np.ndindex(params[k].shape):
            if idx[0] not in (0, 3):
                continue
            pp = {q: v.copy() for q, v in params.items()}
            pm = {q: v.copy() for q, v in params.items()}
            pp[k][idx] += h
            pm[k][idx] -= h
            fd = (mean_loss(pp) - mean_loss(pm)) / (2 * h)
            an = out["grads"][k][idx]
            assert abs(fd - an) <= 1e-9 + 1e-4 * abs(an), (k, idx, fd, an)
            checked += 1
    assert checked == 2 * 14


def test_distillation_steps_reduce_the_loss():
    """"Training a smaller scene": a student started from a perturbed copy of
    the teacher, fitted to the teacher's renders from two cameras, gets
    closer to them (mean L1 falls over ten Adam steps)."""
    cams, teacher = _two_camera_scene()
    targets = [O.render(O.project(teacher, c), c, nthreads=2)["image"] for c in cams]
    rng = np.random.default_rng(11)
    student = {k: v + rng.normal(scale=0.05, size=v.shape) for k, v in teacher.items()}
    lr = {"means": 2e-3, "log_scales": 1e-2, "quats": 1e-2, "opacity_logits": 5e-2, "colors": 1e-2}
    m, v = _zeros_like(student), _zeros_like(student)
    losses = []
    for t in range(1, 11):
        out = OT.train_step(student, cams, targets, m, v, lr, t)
        losses.append(np.mean(out["losses"]))
        student, m, v = out["params"], out["m"], out["v"]
    assert losses[-1] < 0.7 * losses[0], losses


def test_psnr_closed_form():
    a = np.zeros((4, 4, 3))
    b = np.full((4, 4, 3), 0.1)
    assert abs(OT.psnr(a, b) - 20.0) < 1e-12
    assert OT.psnr(a, a) == float("inf")
