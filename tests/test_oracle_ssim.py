"""Pins of the oracle's structural similarity (orc_ssim) and the L1 + D-SSIM loss:
the window and zero padding against scipy (a Gaussian window from
scipy.signal.windows and scipy.ndimage.correlate with constant padding), closed
forms for constant images (interior and border, where only part of the window
lies inside the image), identities (ssim(x, x) = 1, symmetry), and central
finite differences of the gradient."""
import numpy as np
import pytest
from scipy import ndimage
from scipy.signal import windows

import oracle

C1, C2 = 0.01 ** 2, 0.03 ** 2


def _window2d():
    g = windows.gaussian(11, std=1.5)
    g = g / g.sum()
    return np.outer(g, g), g


def test_map_matches_scipy_windowed_moments():
    rng = np.random.default_rng(0)
    x = rng.random((23, 31, 3))
    y = np.clip(x + 0.2 * rng.standard_normal(x.shape), 0, 1)
    _, smap, _ = oracle.ssim(x, y, want_map=True)
    w2, _ = _window2d()
    for c in range(3):
        f = lambda a: ndimage.correlate(a, w2, mode="constant", cval=0.0)  # noqa: E731
        mx, my = f(x[..., c]), f(y[..., c])
        vx, vy, cxy = f(x[..., c] ** 2) - mx ** 2, f(y[..., c] ** 2) - my ** 2, f(x[..., c] * y[..., c]) - mx * my
        S = (2 * mx * my + C1) * (2 * cxy + C2) / ((mx ** 2 + my ** 2 + C1) * (vx + vy + C2))
        np.testing.assert_allclose(smap[..., c], S, rtol=1e-12, atol=1e-13)


def test_constant_images_closed_form_inside_and_at_the_border():
    """x = a, y = b everywhere: with W(p) the window weight that falls inside the
    image, mx = a W, var x = a^2 W (1 - W), cov = a b W (1 - W), so
    S = (2 a b W^2 + C1)(2 a b W (1 - W) + C2) / ((a^2 + b^2) W^2 + C1)((a^2 + b^2) W (1 - W) + C2);
    W = 1 in the interior."""
    H, Wd, a, b = 16, 13, 0.7, 0.3
    x = np.full((H, Wd, 1), a)
    y = np.full((H, Wd, 1), b)
    _, smap, _ = oracle.ssim(x, y, want_map=True)
    _, g = _window2d()
    cum = lambda n, p: sum(g[k + 5] for k in range(-5, 6) if 0 <= p + k < n)  # noqa: E731
    for py in range(H):
        for px in range(Wd):
            Wp = cum(H, py) * cum(Wd, px)
            want = ((2 * a * b * Wp * Wp + C1) * (2 * a * b * Wp * (1 - Wp) + C2) /
                    (((a * a + b * b) * Wp * Wp + C1) * ((a * a + b * b) * Wp * (1 - Wp) + C2)))
            assert abs(smap[py, px, 0] - want) < 1e-12, (py, px)
    # interior: W = 1
    assert abs(smap[8, 6, 0] - (2 * a * b + C1) / (a * a + b * b + C1)) < 1e-12


def test_identity_and_symmetry():
    rng = np.random.default_rng(1)
    x = rng.random((19, 14, 3))
    y = rng.random((19, 14, 3))
    s_xx, _, g_xx = oracle.ssim(x, x, want_grad=True)
    assert abs(s_xx - 1.0) < 1e-14
    assert np.max(np.abs(g_xx)) < 1e-14   # x = y maximises ssim
    assert abs(oracle.ssim(x, y)[0] - oracle.ssim(y, x)[0]) < 1e-14
    assert oracle.ssim(x, y)[0] < 0.5


@pytest.mark.parametrize("shape", [(12, 9, 3), (7, 16, 1)])
def test_gradient_by_central_differences(shape):
    rng = np.random.default_rng(2)
    x = rng.random(shape)
    y = np.clip(x + 0.3 * rng.standard_normal(shape), 0, 1)
    _, _, g = oracle.ssim(x, y, want_grad=True)
    h = 1e-6
    for idx in [(0, 0, 0), (shape[0] - 1, shape[1] - 1, shape[2] - 1), (3, 4, 0), (5, 2, shape[2] - 1)]:
        xp, xm = x.copy(), x.copy()
        xp[idx] += h
        xm[idx] -= h
        fd = (oracle.ssim(xp, y)[0] - oracle.ssim(xm, y)[0]) / (2 * h)
        assert abs(fd - g[idx]) <= 1e-7 * max(1e-3, abs(g[idx])) + 1e-11, (idx, fd, g[idx])


def test_l1_dssim_combination():
    rng = np.random.default_rng(3)
    x = rng.random((10, 12, 3))
    y = rng.random((10, 12, 3))
    loss, g = oracle.l1_dssim(x, y, 1.0, 0.2)
    s, _, gs = oracle.ssim(x, y, want_grad=True)
    assert abs(loss - (np.abs(x - y).mean() + 0.2 * (1 - s))) < 1e-14
    np.testing.assert_allclose(g, np.sign(x - y) / x.size - 0.2 * gs, rtol=0, atol=1e-16)
    loss0, g0 = oracle.l1_dssim(x, x)
    assert abs(loss0) < 1e-14 and np.max(np.abs(g0)) < 1e-14
