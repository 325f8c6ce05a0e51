"""Parity of the fused optimiser step (gs_adam_step) with its oracle, step by
step: each step's GPU state (fp32) is the oracle's input, so no drift
between fp32 and float64 accumulates across steps."""
import numpy as np
import pytest
import torch

from oracle import adam as A
from differentiable_gaussian_splatting_preprocess_b200 import binding as B

from _gpu_pipeline import rel_l2, to_np

pytestmark = pytest.mark.gpu

LR = dict(means=1.6e-4, log_scales=5e-3, quats=1e-3, logit_opacity=5e-2, colors=2.5e-3)


def _cfg(warmup):
    return B.GsAdamConfig(LR["means"], LR["log_scales"], LR["quats"], LR["logit_opacity"], LR["colors"],
                          0.9, 0.999, 1e-15, warmup)


def _split(flat, n, c):
    sizes = dict(means=(n, 3), log_scales=(n, 3), quats=(n, 4), logit_opacity=(n,), colors=(n, c))
    out, off = {}, 0
    for k in A.GROUPS:
        cnt = int(np.prod(sizes[k]))
        out[k] = flat[off:off + cnt].reshape(sizes[k]).astype(np.float64)
        off += cnt
    return out


@pytest.mark.parametrize("n,c,warmup", [(10_000, 3, 2), (3_001, 48, 0)])
def test_adam_steps_match_oracle(n, c, warmup):
    rng = np.random.default_rng(n + c)
    q = rng.normal(size=(n, 4))
    q /= np.linalg.norm(q, axis=1, keepdims=True)
    host = dict(means=rng.normal(size=(n, 3)), log_scales=rng.normal(-4, 0.5, size=(n, 3)), quats=q,
                logit_opacity=rng.normal(size=n), colors=rng.uniform(size=(n, c)))
    dev = {k: torch.from_numpy(v.astype(np.float32)).cuda() for k, v in host.items()}
    m = torch.zeros((11 + c) * n, device="cuda")
    v = torch.zeros_like(m)
    scales = torch.empty((n, 3), device="cuda")
    opacity = torch.empty(n, device="cuda")
    cfg = _cfg(warmup)
    for step in range(1, 4):
        g = dict(dL_dmeans=rng.normal(size=(n, 3)), dL_dscales=rng.normal(size=(n, 3)) * 50,
                 dL_dquats=rng.normal(size=(n, 4)), dL_dopacity=rng.normal(size=n),
                 dL_dcolors=rng.normal(size=(n, c)))
        g32 = {k: x.astype(np.float32) for k, x in g.items()}
        gd = {k: torch.from_numpy(x).cuda() for k, x in g32.items()}
        before = {k: to_np(t).astype(np.float64) for k, t in dev.items()}
        m0, v0 = _split(to_np(m), n, c), _split(to_np(v), n, c)
        B.gs_adam_step(cfg, step, dev, gd, m, v, scales, opacity)
        torch.cuda.synchronize()
        # the kernel receives the rates, betas and eps as fp32: the oracle gets those values
        f = lambda x: float(np.float32(x))  # noqa: E731
        op, om, ov, os_, oo = A.adam_step(before, g32, m0, v0, step, {k: f(x) for k, x in LR.items()}, f(0.9),
                                          f(0.999), f(1e-15), warmup)
        gm, gv = _split(to_np(m), n, c), _split(to_np(v), n, c)
        for k in A.GROUPS:
            after = to_np(dev[k]).astype(np.float64)
            # the fp32 result of p - delta: within a few ulps of the parameter,
            # plus a relative error of the update itself
            ulp = np.spacing(np.abs(op[k]).astype(np.float32)).astype(np.float64)
            bound = 8 * ulp + 1e-5 * np.abs(op[k] - before[k]) + 1e-30
            assert np.all(np.abs(after - op[k]) <= bound), (step, k, np.max(np.abs(after - op[k]) / bound))
            assert rel_l2(gm[k], om[k]) <= 1e-6, (step, k)
            assert rel_l2(gv[k], ov[k]) <= 1e-5, (step, k)
        np.testing.assert_allclose(np.linalg.norm(to_np(dev["quats"]), axis=1), 1.0, atol=1e-6)
        np.testing.assert_allclose(to_np(scales), os_, rtol=1e-5)
        np.testing.assert_allclose(to_np(opacity), oo, rtol=0, atol=1e-6)


def test_adam_rejects_bad_arguments():
    n = 8
    dev = dict(means=torch.zeros((n, 3), device="cuda"), log_scales=torch.zeros((n, 3), device="cuda"),
               quats=torch.zeros((n, 4), device="cuda"), logit_opacity=torch.zeros(n, device="cuda"),
               colors=torch.zeros((n, 3), device="cuda"))
    g = dict(dL_dmeans=dev["means"], dL_dscales=dev["log_scales"], dL_dquats=dev["quats"],
             dL_dopacity=dev["logit_opacity"], dL_dcolors=dev["colors"])
    m = torch.zeros(14 * n, device="cuda")
    with pytest.raises(B.GsError):
        B.gs_adam_step(_cfg(0), 0, dev, g, m, m.clone())
    bad = _cfg(0)
    bad.beta2 = 1.0
    with pytest.raises(B.GsError):
        B.gs_adam_step(bad, 1, dev, g, m, m.clone())
