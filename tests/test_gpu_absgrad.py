"""Parity of the absolute 2D gradient (absgrad, gsplat guide lmnt.cn/news/262699
§4.1) with the oracle: gs_raster_bwd with gs_grad2d.xy_abs set against the
oracle's per-pixel absolute sums (sums of non-negative terms, so the plain
gradient tolerance applies without a cancellation allowance); the other 2D
gradients unchanged by the option; the densification statistic on |xy_abs|."""
import numpy as np
import pytest
import torch

from gaussian_splatting_differentiable_02_b200 import pipeline as pl
from gaussian_splatting_differentiable_02_b200 import scenes

from _parity import BAND_ALPHA, BAND_T, CudaRun, check_grads

pytestmark = pytest.mark.gpu


def _absgrad(run, up):
    run.view.dL_dimage.copy_(torch.from_numpy(np.ascontiguousarray(up, np.float32)))
    g2 = pl.Grad2D(run.scene.n, absgrad=True)
    pl.raster_bwd(run.proj, run.view, g2, run.bg)
    torch.cuda.synchronize()
    return g2


@pytest.mark.parametrize("case", ["tiny", "anisotropic"])
def test_absgrad_matches_oracle(orc, case):
    if case == "tiny":
        wl = scenes.tiny()
        scene, cam, up = wl.scene, wl.cameras[0], wl.upstream[0]
    else:
        # needle-shaped splats: the factored evaluation path
        rng = np.random.default_rng(31)
        scene = scenes.random_scene(rng, 600, 2, mean_box=1.0, log_scale=(-4.5, -1.5))
        R, t = scenes.look_at((0.5, 0.2, -4.0))
        cam = scenes.camera(R, t, 120.0, 120.0, 50.0, 18.5, 100, 37)
        up = rng.standard_normal((37, 100, 3)).astype(np.float32)
    run = CudaRun(scene, cam)
    plain = run.backward(up)
    g2 = _absgrad(run, up)
    # the option leaves the ordinary gradients as they were (same arithmetic; the
    # order of the atomic adds of different warps may differ between launches)
    rows_abs = g2.as_rows()
    scale = np.abs(plain).max(axis=0)
    assert np.all(np.abs(rows_abs - plain) <= 1e-6 * scale + 1e-5 * np.abs(plain))
    ref = orc.project(scene, cam)
    want, want_abs, touched = orc.render_bwd(ref, cam, up.reshape(-1, 3).astype(np.float64), band_alpha=BAND_ALPHA,
                                             band_T=BAND_T)
    rows = np.nonzero(touched == 0)[0]
    assert len(rows) > 0.8 * scene.n
    got = g2.xy_abs.cpu().numpy()
    check_grads(got[:, 0], want_abs[:, 0], "abs du", rows=rows)
    check_grads(got[:, 1], want_abs[:, 1], "abs dv", rows=rows)
    assert np.all(got[:, 0] >= np.abs(plain[:, 0]) * (1 - 1e-5) - 1e-12)


def test_densify_statistic_uses_the_absolute_gradient(orc):
    wl = scenes.tiny()
    run = CudaRun(wl.scene, wl.cameras[0])
    g2 = _absgrad(run, wl.upstream[0])
    n = wl.scene.n
    grads = run.g.zeros_like()
    acc = torch.zeros((n,), device="cuda")
    cnt = torch.zeros((n,), device="cuda", dtype=torch.int32)
    pl.project_bwd(run.g, run.view, run.proj, g2, grads, acc, cnt)
    torch.cuda.synchronize()
    xa = g2.xy_abs.cpu().numpy().astype(np.float64)
    vis = run.proj.radius.cpu().numpy() > 0
    np.testing.assert_allclose(acc.cpu().numpy()[vis], np.hypot(xa[vis, 0], xa[vis, 1]), rtol=1e-6, atol=1e-12)
    assert np.all(acc.cpu().numpy()[~vis] == 0)
    assert np.array_equal(cnt.cpu().numpy(), vis.astype(np.int32))


def test_trainer_with_absgrad():
    rng = np.random.default_rng(32)
    scene = scenes.random_scene(rng, 500, 1, mean_box=1.0, log_scale=(-4.0, -2.5))
    R, t = scenes.look_at((0.0, 0.0, -4.0))
    cam = scenes.camera(R, t, 128.0, 128.0, 64.0, 64.0, 128, 128)
    target = torch.from_numpy(rng.random((128, 128, 3)).astype(np.float32)).cuda()
    lrs = {"means": 1.6e-4, "log_scales": 5e-3, "quats": 1e-3, "opacity_logits": 5e-2, "sh": 2.5e-3}
    runs = []
    for absgrad in (False, True):
        tr = pl.Trainer(pl.Gaussians.from_scene(scene), [pl.View(scene.n, cam)], [target], dict(lrs), densify=True,
                        absgrad=absgrad)
        tr.step()
        torch.cuda.synchronize()
        runs.append((tr.gauss.to_numpy(), tr.densify_accum.cpu().numpy(), tr.densify_count.cpu().numpy()))
    (pa, da, ca), (pb, db, cb) = runs
    for k in pa:
        # the option changes only the statistic (up to the order of atomic adds, which
        # can flip Adam's first step for a gradient that is a near-zero cancellation)
        close = np.abs(pa[k] - pb[k]) <= 1e-6 + 1e-5 * np.abs(pa[k])
        assert close.mean() >= 0.999, (k, float(close.mean()))
    assert np.array_equal(ca, cb)
    assert np.all(db >= da * (1 - 1e-5)) and np.any(db > 1.01 * da)
