"""Oracle for the fused optimiser step (TEST INFRASTRUCTURE: only tests/,
__graft_entry__.smoke() and bench.py's CPU leg may use it).

Plain float64 numpy, restating:
  * Adam (Kingma and Ba, "Adam: A Method for Stochastic Optimization", 2015,
    Algorithm 1): m <- b1 m + (1 - b1) g, v <- b2 v + (1 - b2) g^2,
    m_hat = m / (1 - b1^t), v_hat = v / (1 - b2^t),
    p <- p - lr m_hat / (sqrt(v_hat) + eps);
  * the per-parameter learning rates and the schedule of "4-3DGS训练与优化"
    section C.2: one learning rate per parameter group (position, scale,
    rotation, opacity, colour), the position and scale rates warmed up
    linearly over the first iterations (factor min(1, t / warmup));
  * the parametrisation the rasterizer's inputs come from: scales = exp(log
    scales), opacity = sigmoid(logit), so the gradients it returns (w.r.t.
    the activated values) are chained through those maps first; the
    quaternion is renormalised to unit length after its update (the
    section's note on the rotation group is read as keeping the parameter
    on the unit sphere between steps).
Parity pinned by tests/test_oracle_adam.py.
"""
from __future__ import annotations

from typing import Dict

import numpy as np

GROUPS = ("means", "log_scales", "quats", "logit_opacity", "colors")
GRAD_OF = {"means": "dL_dmeans", "log_scales": "dL_dscales", "quats": "dL_dquats",
           "logit_opacity": "dL_dopacity", "colors": "dL_dcolors"}
WARMED = ("means", "log_scales")


def sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def raw_gradients(params: Dict[str, np.ndarray], grads: Dict[str, np.ndarray]) -> Dict[str, np.ndarray]:
    """Gradients w.r.t. the raw parameters from those w.r.t. the activated
    values: d exp(x)/dx = exp(x), d sigmoid(x)/dx = sigmoid(x) (1 - sigmoid(x))."""
    p = {k: np.asarray(v, np.float64) for k, v in params.items()}
    g = {k: np.asarray(grads[GRAD_OF[k]], np.float64) for k in GROUPS}
    s = np.exp(p["log_scales"])
    o = sigmoid(p["logit_opacity"])
    g["log_scales"] = g["log_scales"] * s
    g["logit_opacity"] = g["logit_opacity"] * o * (1.0 - o)
    return g


def adam_step(params, grads, m, v, step: int, lr: Dict[str, float], beta1: float, beta2: float, eps: float,
              warmup: int):
    """One step; returns (params, m, v, scales, opacity) as new float64 arrays.
    ``m``/``v`` are dicts keyed like ``params``."""
    if step < 1:
        raise ValueError("steps count from 1")
    g = raw_gradients(params, grads)
    out_p, out_m, out_v = {}, {}, {}
    bc1 = 1.0 - beta1 ** step
    bc2 = 1.0 - beta2 ** step
    for k in GROUPS:
        p = np.asarray(params[k], np.float64)
        mk = beta1 * np.asarray(m[k], np.float64) + (1.0 - beta1) * g[k]
        vk = beta2 * np.asarray(v[k], np.float64) + (1.0 - beta2) * g[k] * g[k]
        m_hat = mk / bc1
        v_hat = vk / bc2
        rate = lr[k] * (min(1.0, step / warmup) if (k in WARMED and warmup > 0) else 1.0)
        p = p - rate * m_hat / (np.sqrt(v_hat) + eps)
        if k == "quats":
            n = np.linalg.norm(p, axis=1, keepdims=True)
            p = np.where(n > 0, p / np.where(n > 0, n, 1.0), p)
        out_p[k], out_m[k], out_v[k] = p, mk, vk
    return out_p, out_m, out_v, np.exp(out_p["log_scales"]), sigmoid(out_p["logit_opacity"])
