"""Pins of the oracle's absolute-gradient sums (gsplat's absgrad, gsplat guide
lmnt.cn/news/262699 §4.1): for every Gaussian and every 2D-gradient slot, the sum
over pixels of the absolute value of that pixel's contribution.  Pinned by brute
force (one reverse pass per pixel, absolute values summed here), by the single-pixel
case (the sum of absolute values of one term is its absolute value) and by the
triangle inequality."""
import numpy as np

from gaussian_splatting_differentiable_02_b200 import scenes


def _case():
    rng = np.random.default_rng(21)
    scene = scenes.random_scene(rng, 150, 1, mean_box=1.0, log_scale=(-3.5, -2.0))
    R, t = scenes.look_at((0.3, -0.2, -4.0))
    cam = scenes.camera(R, t, 48.0, 48.0, 24.0, 20.0, 48, 40)
    return scene, cam


def test_absgrad_is_the_sum_of_per_pixel_absolute_contributions(orc):
    scene, cam = _case()
    p = orc.project(scene, cam)
    rng = np.random.default_rng(22)
    up = rng.standard_normal((48 * 40, 3))
    g2, g2a, _ = orc.render_bwd(p, cam, up)
    brute = np.zeros_like(g2a)
    for pix in range(48 * 40):
        gp, gpa, _ = orc.render_bwd(p, cam, up[pix:pix + 1], pix=np.array([pix]))
        # one pixel: the sum of |term| is |term|
        np.testing.assert_array_equal(gpa, np.abs(gp))
        brute += np.abs(gp)
    np.testing.assert_allclose(g2a, brute, rtol=1e-12, atol=1e-300)
    assert np.all(g2a >= np.abs(g2) * (1 - 1e-12))
    # some Gaussians collect terms of both signs (absgrad strictly larger)
    assert np.sum(g2a[:, 0] > 1.001 * np.abs(g2[:, 0])) > 10
