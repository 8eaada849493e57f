"""Training step of the oracle: the L1 loss, Adam, and one step over several
cameras, in double precision.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Sources (by page title and section):
  [GSP]  "Gaussian splatting in PyTorch", s7 "Fitting splats with Adam": the
         loop render -> L1 against the target -> backward -> Adam step over
         the raw parameters, with a learning rate per parameter group
         (torch.optim.Adam).
  [DIST] "The backward pass I deleted trained the model the Nano runs",
         "Training a smaller scene": one student optimised against renders
         from sixty cameras, so that the result is a 3D model.
Adam itself is Kingma and Ba's algorithm (bias-corrected first and second
moment estimates), written here in its textbook form.
"""
from __future__ import annotations

import numpy as np

from . import oracle as _o

PARAM_KEYS = ("means", "log_scales", "quats", "opacity_logits", "colors")

__all__ = ["PARAM_KEYS", "l1_loss_grad", "adam_step", "camera_loss_grad", "train_step", "psnr"]


def l1_loss_grad(image, target):
    """[GSP] s7: loss = mean |image - target| over every value; its gradient
    is sign(image - target) / count, with sign(0) = 0 (the subgradient
    torch's abs uses)."""
    d = np.asarray(image, np.float64) - np.asarray(target, np.float64)
    return float(np.abs(d).mean()), np.sign(d) / d.size


def adam_step(params: dict, grads: dict, m: dict, v: dict, lr: dict, t: int, beta1: float = 0.9,
              beta2: float = 0.999, eps: float = 1e-8):
    """One Adam step (step number t >= 1) on every parameter group:
        m <- beta1 m + (1 - beta1) g
        v <- beta2 v + (1 - beta2) g^2
        m_hat = m / (1 - beta1^t),  v_hat = v / (1 - beta2^t)
        p <- p - lr m_hat / (sqrt(v_hat) + eps)
    lr maps each key of PARAM_KEYS to its learning rate.  Returns new
    (params, m, v) dicts; the inputs are not modified."""
    if t < 1:
        raise ValueError("t counts from 1")
    P, M, V = {}, {}, {}
    for k in PARAM_KEYS:
        g = np.asarray(grads[k], np.float64)
        mk = beta1 * np.asarray(m[k], np.float64) + (1.0 - beta1) * g
        vk = beta2 * np.asarray(v[k], np.float64) + (1.0 - beta2) * g * g
        m_hat = mk / (1.0 - beta1 ** t)
        v_hat = vk / (1.0 - beta2 ** t)
        P[k] = np.asarray(params[k], np.float64) - lr[k] * m_hat / (np.sqrt(v_hat) + eps)
        M[k], V[k] = mk, vk
    return P, M, V


def camera_loss_grad(params: dict, cam, target, nthreads: int | None = None) -> dict:
    """One camera's share of the step: project, render, L1 against the
    target, the blend's backward and the chain rule to the raw parameters."""
    p = _o.project(params, cam)
    r = _o.render(p, cam, nthreads=nthreads)
    loss, dl = l1_loss_grad(r["image"], target)
    g2, _ = _o.render_bwd(p, cam, dl, nthreads=nthreads)
    raw = _o.project_bwd(params, cam, g2)
    return {"loss": loss, "image": r["image"], "grads": raw, "proj": p, "render": r, "dl": dl}


def train_step(params: dict, cams, targets, m: dict, v: dict, lr: dict, t: int, beta1: float = 0.9,
               beta2: float = 0.999, eps: float = 1e-8, adam: bool = True, nthreads: int | None = None) -> dict:
    """One training step over the cameras: the loss is the mean of the
    cameras' L1 losses, so the gradient is the mean of their gradients;
    then one Adam step (skipped with adam=False).  Returns the new params,
    m, v, the mean gradient `grads`, the per-camera `losses` and `images`."""
    per = [camera_loss_grad(params, c, tg, nthreads) for c, tg in zip(cams, targets)]
    B = len(per)
    grads = {k: sum(q["grads"][k] for q in per) / B for k in PARAM_KEYS}
    out = {"grads": grads, "losses": [q["loss"] for q in per], "images": [q["image"] for q in per]}
    if adam:
        out["params"], out["m"], out["v"] = adam_step(params, grads, m, v, lr, t, beta1, beta2, eps)
    return out


def psnr(image, target, peak: float = 1.0) -> float:
    """Peak signal-to-noise ratio in dB: 10 log10(peak^2 / MSE)."""
    mse = float(np.mean((np.asarray(image, np.float64) - np.asarray(target, np.float64)) ** 2))
    return float("inf") if mse == 0.0 else 10.0 * np.log10(peak * peak / mse)
