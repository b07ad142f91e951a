"""Pins of the CPU oracle against things other than itself: closed forms, a
library routine (scipy's spherical harmonics, scipy's quaternion rotation,
numpy linear algebra), brute force, invariants and central finite differences.
Each test is chosen so that a plausible slip in the oracle (a dropped term, a
wrong sign, a swapped index, a transposed matrix) fails at least one of them.
"""
import math

import numpy as np
import pytest
import scipy.special as sps
from scipy.spatial.transform import Rotation

from gaussian_splatting_differentiable_02_b200 import scenes

C0 = 1.0 / (2.0 * math.sqrt(math.pi))


def one_scene(means, quats, log_scales, logits, sh, deg):
    n = len(means)
    return scenes.Scene(np.asarray(means, np.float32).reshape(n, 3), np.asarray(quats, np.float32).reshape(n, 4),
                        np.asarray(log_scales, np.float32).reshape(n, 3), np.asarray(logits, np.float32).reshape(n),
                        np.asarray(sh, np.float32).reshape(n, (deg + 1) ** 2, 3), deg)


# ---------------------------------------------------------------- spherical harmonics

def fib_sphere(n):
    i = np.arange(n) + 0.5
    z = 1.0 - 2.0 * i / n
    phi = math.pi * (1.0 + math.sqrt(5.0)) * i
    r = np.sqrt(1.0 - z * z)
    return np.stack([r * np.cos(phi), r * np.sin(phi), z], axis=1)


def test_sh_matches_scipy_real_form(orc):
    """Real SH with Condon-Shortley phase, index l^2+l+m: sqrt2*Re(Y_l^m) for m>0,
    sqrt2*Im(Y_l^|m|) for m<0, Y_l^0 for m=0, with scipy's complex Y_l^m."""
    d = fib_sphere(200)
    Y = orc.sh_basis(d, 3)
    theta = np.arccos(np.clip(d[:, 2], -1, 1))
    phi = np.arctan2(d[:, 1], d[:, 0])
    for l in range(4):
        for m in range(-l, l + 1):
            ref = sps.sph_harm_y(l, abs(m), theta, phi)
            if m > 0:
                r = math.sqrt(2.0) * ref.real
            elif m < 0:
                r = math.sqrt(2.0) * ref.imag
            else:
                r = ref.real
            np.testing.assert_allclose(Y[:, l * l + l + m], r, atol=1e-12, err_msg=f"l={l} m={m}")


def test_sh_orthonormal_by_quadrature(orc):
    d = fib_sphere(20000)
    Y = orc.sh_basis(d, 3)
    G = Y.T @ Y * (4.0 * math.pi / len(d))
    np.testing.assert_allclose(G, np.eye(16), atol=2e-3)


def test_sh_degree1_signs(orc):
    """The colour convention: Y_1 = (-c y, c z, -c x) with c = sqrt(3/(4 pi))."""
    c = math.sqrt(3.0 / (4.0 * math.pi))
    Y = orc.sh_basis(np.array([[0.6, 0.0, 0.8], [0.0, 1.0, 0.0]]), 1)
    np.testing.assert_allclose(Y[0], [C0, 0.0, c * 0.8, -c * 0.6], atol=1e-15)
    np.testing.assert_allclose(Y[1], [C0, -c, 0.0, 0.0], atol=1e-15)


# ---------------------------------------------------------------- projection

def tiny_cam(W=128, H=128, f=128.0):
    return scenes.tiny().cameras[0] if (W, H, f) == (128, 128, 128.0) else None


def test_projection_isotropic_on_axis_closed_form(orc):
    """Identity rotation, equal scales s, mean on the optical axis at depth z:
    Sigma' = (f s / z)^2 I + eps I, conic = I / that, radius = ceil(3 sqrt(a + sqrt(0.1)))."""
    cam = scenes.tiny().cameras[0]        # eye (0,0,-4) looking at the origin, f = 128, c = 64
    s = 0.05
    sc = one_scene([[0, 0, 1.0]], [[1, 0, 0, 0]], [[math.log(s)] * 3], [0.3], [[[0.2, 0.4, 0.6]]], 0)
    p = orc.project(sc, cam, quantize=False)
    z = 5.0
    a = (128.0 * np.float32(s) / z) ** 2 + 0.3
    assert p["radius"][0] == math.ceil(3 * math.sqrt(a + math.sqrt(0.1)))
    np.testing.assert_allclose(p["depth"][0], z, rtol=1e-15)
    np.testing.assert_allclose(p["xy"][0], [64.0, 64.0], atol=1e-12)
    np.testing.assert_allclose(p["conic"][0], [1 / a, 0.0, 1 / a], rtol=1e-6, atol=1e-15)
    np.testing.assert_allclose(p["opacity"][0], sps.expit(float(np.float32(0.3))), rtol=1e-15)
    np.testing.assert_allclose(p["rgb"][0], C0 * np.float32([0.2, 0.4, 0.6]).astype(np.float64) + 0.5, rtol=1e-15)


def _numpy_projection(mu, q_wxyz, log_s, cam):
    """Independent restatement with scipy's quaternion rotation, numpy products,
    a finite-difference Jacobian of the pinhole map and numpy's inverse."""
    R = np.asarray(cam["R"], np.float64)
    t = np.asarray(cam["t"], np.float64)
    fx, fy, cx, cy = cam["fx"], cam["fy"], cam["cx"], cam["cy"]
    Rq = Rotation.from_quat([q_wxyz[1], q_wxyz[2], q_wxyz[3], q_wxyz[0]]).as_matrix()
    S = np.diag(np.exp(np.asarray(log_s, np.float64)))
    Sig = Rq @ S @ S.T @ Rq.T
    p = R @ np.asarray(mu, np.float64) + t
    limx = 1.3 * 0.5 * cam["width"] / fx
    limy = 1.3 * 0.5 * cam["height"] / fy
    pj = p.copy()
    pj[0] = np.clip(p[0] / p[2], -limx, limx) * p[2]
    pj[1] = np.clip(p[1] / p[2], -limy, limy) * p[2]

    def pin(x):
        return np.array([fx * x[0] / x[2], fy * x[1] / x[2]])
    J = np.zeros((2, 3))
    h = 1e-6
    for k in range(3):
        e = np.zeros(3)
        e[k] = h * max(1.0, abs(pj[k]))
        J[:, k] = (pin(pj + e) - pin(pj - e)) / (2 * e[k])
    S2 = J @ R @ Sig @ R.T @ J.T + cam["eps2d"] * np.eye(2)
    Q = np.linalg.inv(S2)
    uv = pin(p) + np.array([cx, cy])
    return uv, p[2], np.array([Q[0, 0], Q[0, 1], Q[1, 1]])


@pytest.mark.parametrize("offscreen", [False, True])
def test_projection_anisotropic_matches_numpy(orc, offscreen):
    rng = np.random.default_rng(5)
    cam = scenes.box100k(poses=3).cameras[1]
    n = 50
    sc = scenes.random_scene(rng, n, 2, mean_box=1.5, log_scale=(-3.5, -1.5))
    if offscreen:   # large Gaussians pushed sideways: the Jacobian clamp is active, footprints still on screen
        R = np.asarray(cam["R"], np.float64)
        sc.means[:] = (sc.means + 5.5 * R[0]).astype(np.float32)
        sc.log_scales[:] = rng.uniform(-1.0, 0.0, sc.log_scales.shape).astype(np.float32)
    p = orc.project(sc, cam, quantize=False)
    checked = clamped = 0
    for i in range(n):
        uv, z, con = _numpy_projection(sc.means[i], sc.quats[i], sc.log_scales[i], cam)
        if p["radius"][i] == 0:
            continue
        checked += 1
        np.testing.assert_allclose(p["xy"][i], uv, rtol=1e-12)
        np.testing.assert_allclose(p["depth"][i], z, rtol=1e-12)
        np.testing.assert_allclose(p["conic"][i], con, rtol=1e-6, atol=1e-9 * np.abs(con).max())
        if offscreen:
            clamped += abs(uv[0] - cam["cx"]) > 1.3 * 0.5 * cam["width"]
    assert checked > 5
    if offscreen:
        assert clamped > 5


def test_rect_covers_three_sigma_pixels(orc):
    """Invariant: every pixel inside the 3-sigma ellipse (d^T Sigma'^-1 d <= 9)
    lies in a tile of the Gaussian's rectangle."""
    rng = np.random.default_rng(7)
    cam = scenes.tiny().cameras[0]
    sc = scenes.random_scene(rng, 60, 0, mean_box=1.2, log_scale=(-3.5, -1.0))
    p = orc.project(sc, cam, quantize=False)
    ys, xs = np.mgrid[0:128, 0:128]
    px, py = xs + 0.5, ys + 0.5
    for i in np.nonzero(p["radius"])[0]:
        A, B, Cc = p["conic"][i]
        dx, dy = p["xy"][i, 0] - px, p["xy"][i, 1] - py
        inside = (A * dx * dx + 2 * B * dx * dy + Cc * dy * dy) <= 9.0
        tx, ty = xs[inside] // 16, ys[inside] // 16
        r = p["rect"][i]
        assert np.all((tx >= r[0]) & (tx < r[2]) & (ty >= r[1]) & (ty < r[3])), i
        assert p["tiles_touched"][i] == (r[2] - r[0]) * (r[3] - r[1])


def test_culling(orc):
    cam = scenes.tiny().cameras[0]
    nan = float("nan")
    sc = one_scene([[0, 0, -3.9], [0, 0, -5.0], [nan, 0, 0], [0, 0, 0], [0, 0, 0], [50, 0, 0]],
                   [[1, 0, 0, 0], [1, 0, 0, 0], [1, 0, 0, 0], [0, 0, 0, 0], [1, 0, 0, 0], [1, 0, 0, 0]],
                   [[-3] * 3] * 6, [0, 0, 0, 0, float("inf"), 0], [[[0.5] * 3]] * 6, 0)
    p = orc.project(sc, cam)
    # 0: z = 0.1 <= near; 1: behind; 2: NaN mean; 3: zero quaternion; 4: inf logit; 5: far off-screen
    assert list(p["radius"]) == [0, 0, 0, 0, 0, 0]
    assert list(p["tiles_touched"]) == [0] * 6


# ---------------------------------------------------------------- keys

def test_keys_brute_force_tiny(orc):
    wl = scenes.tiny()
    cam = wl.cameras[0]
    p = orc.project(wl.scene, cam)
    keys, vals, ranges = orc.keys(p, cam)
    TX = 8
    inst = []
    for i in range(wl.scene.n):
        if p["radius"][i] == 0:
            continue
        zb = int(np.float32(p["depth"][i]).view(np.uint32))
        x0, y0, x1, y1 = p["rect"][i]
        for ty in range(y0, y1):
            for tx in range(x0, x1):
                inst.append((((ty * TX + tx) << 32) | zb, i))
    inst.sort()
    assert len(inst) == len(keys) > 1000
    assert [k for k, _ in inst] == [int(k) for k in keys]
    assert [v for _, v in inst] == [int(v) for v in vals]
    for t in range(64):
        members = [j for j, (k, _) in enumerate(inst) if k >> 32 == t]
        exp = (members[0], members[-1] + 1) if members else (0, 0)
        assert tuple(ranges[t]) == exp


# ---------------------------------------------------------------- compositing

def test_single_centred_gaussian_gives_colour_times_opacity(orc):
    """(u, v) = (63.5, 63.5) is pixel (63, 63)'s centre: image = rgb * min(0.99, o) there."""
    cam = scenes.tiny().cameras[0]
    for logit in (0.7, 8.0):            # o = 0.668 and o = 0.99966 (clamped to 0.99)
        sc = one_scene([[1 / 64, 1 / 64, 0.0]], [[1, 0, 0, 0]], [[-3.0] * 3], [logit], [[[0.3, -0.2, 1.1]]], 0)
        p = orc.project(sc, cam)
        assert tuple(p["xy"][0]) == (63.5, 63.5)
        img, fT, nc, amb = orc.render(p, cam, pix=[63 * 128 + 63])
        o = float(np.float32(sps.expit(float(np.float32(logit)))))
        rgb = np.float32(C0 * np.float32([0.3, -0.2, 1.1]).astype(np.float64) + 0.5).astype(np.float64)
        a = min(0.99, o)
        np.testing.assert_allclose(img[0], rgb * a, rtol=1e-7)
        np.testing.assert_allclose(fT[0], 1 - a, rtol=1e-12)
        assert nc[0] == 1 and amb[0] == 0


def test_weights_telescope(orc):
    """With every colour 1 and a black background the image is sum_i a_i T_i = 1 - T_final <= 1."""
    wl = scenes.tiny()
    sc = wl.scene
    sc = one_scene(sc.means, sc.quats, sc.log_scales, sc.opacity_logits, np.full((sc.n, 1, 3), 0.5 / C0), 0)
    cam = wl.cameras[0]
    p = orc.project(sc, cam)
    assert np.all(p["rgb"][p["radius"] > 0] == 1.0)
    img, fT, nc, amb = orc.render(p, cam)
    np.testing.assert_allclose(img[:, 0] + fT, 1.0, atol=1e-12)
    assert np.all(img <= 1.0 + 1e-12) and np.all(fT >= 1e-4 * (1 - 1e-9))
    assert nc.max() > 5


def test_equal_depth_orders_by_gid(orc):
    cam = scenes.tiny().cameras[0]
    m = [1 / 64, 1 / 64, 0.0]
    sc = one_scene([m, m], [[1, 0, 0, 0]] * 2, [[-3.0] * 3] * 2, [0.0, 0.0],
                   [[[0.5 / C0, -0.5 / C0, -0.5 / C0]], [[-0.5 / C0, 0.5 / C0, -0.5 / C0]]], 0)
    p = orc.project(sc, cam)
    img, fT, nc, amb = orc.render(p, cam, pix=[63 * 128 + 63])
    a = 0.5
    np.testing.assert_allclose(img[0], [a, a * (1 - a), 0.0], atol=1e-12)   # red (gid 0) in front
    assert nc[0] == 2


def test_skip_below_one_over_255(orc):
    cam = scenes.tiny().cameras[0]
    for factor, contributes in ((1 - 1e-3, False), (1 + 1e-3, True)):
        o = factor / 255.0
        sc = one_scene([[1 / 64, 1 / 64, 0.0]], [[1, 0, 0, 0]], [[-3.0] * 3], [math.log(o / (1 - o))],
                       [[[0.5 / C0] * 3]], 0)
        p = orc.project(sc, cam)
        img, fT, nc, amb = orc.render(p, cam, pix=[63 * 128 + 63])
        assert (nc[0] == 1) == contributes and amb[0] == 0
        assert (img[0, 0] > 0) == contributes


def test_opaque_stack_stops(orc):
    """Five Gaussians of alpha 0.95 at one pixel centre: T = 1, .05, .0025, 1.25e-4;
    the 4th would leave 6.25e-6 < 1e-4, so it and the 5th are not blended."""
    cam = scenes.tiny().cameras[0]
    n = 5
    means = [[(1 / 64) * (4 + k) / 4, (1 / 64) * (4 + k) / 4, float(k)] for k in range(n)]   # same pixel, deeper
    o = 0.95
    cols = [0.2, 0.4, 0.6, 0.8, 1.0]
    sc = one_scene(means, [[1, 0, 0, 0]] * n, [[-3.0] * 3] * n, [math.log(o / (1 - o))] * n,
                   [[[(c - 0.5) / C0] * 3] for c in cols], 0)
    p = orc.project(sc, cam)
    np.testing.assert_allclose(p["xy"], 63.5, atol=1e-4)
    img, fT, nc, amb = orc.render(p, cam, pix=[63 * 128 + 63])
    assert nc[0] == 3 and amb[0] == 0
    on = p["opacity"][0]
    G = [math.exp(-0.5 * (p["conic"][k, 0] * (p["xy"][k, 0] - 63.5) ** 2 + p["conic"][k, 2] *
                          (p["xy"][k, 1] - 63.5) ** 2 + 2 * p["conic"][k, 1] * (p["xy"][k, 0] - 63.5) *
                          (p["xy"][k, 1] - 63.5))) for k in range(3)]
    al = [on * g for g in G]
    T, C = 1.0, 0.0
    for k in range(3):
        C += p["rgb"][k, 0] * al[k] * T
        T *= 1 - al[k]
    np.testing.assert_allclose(img[0, 0], C, rtol=1e-12)
    np.testing.assert_allclose(fT[0], T, rtol=1e-12)


# ---------------------------------------------------------------- gradients

def _fd_scene(seed, deg):
    """Few large Gaussians inside a single 16x16-tile image: every alpha stays well
    above 1/255, below the 0.99 clamp, and T well above 1e-4, so the image is
    smooth in every parameter (one of them sits off-screen with its Jacobian clamped)."""
    rng = np.random.default_rng(seed)
    R, t = scenes.look_at((0.0, 0.0, -4.0))
    cam = scenes.camera(R, t, 20.0, 20.0, 8.0, 8.0, 16, 16)
    n = 4
    nc = (deg + 1) ** 2
    means = np.array([[0.3, -0.2, 0.1], [-0.4, 0.3, 0.5], [0.1, 0.5, -0.3], [-5.5, 0.1, 0.4]], np.float32)
    quats = rng.standard_normal((n, 4)).astype(np.float32)
    log_scales = rng.uniform(0.3, 0.9, (n, 3)).astype(np.float32)
    log_scales[3] = [1.8, 1.6, 1.7]
    logits = rng.uniform(-1.5, 0.8, n).astype(np.float32)
    sh = np.zeros((n, nc, 3), np.float32)
    sh[:, 0, :] = rng.uniform(0.5, 1.5, (n, 3))
    if nc > 1:
        sh[:, 1:, :] = 0.1 * rng.standard_normal((n, nc - 1, 3))
    return scenes.Scene(means, quats, log_scales, logits, sh, deg), cam


@pytest.mark.parametrize("deg", [0, 3])
def test_backward_matches_central_differences(orc, deg):
    sc, cam = _fd_scene(11, deg)
    bg = (0.2, 0.1, 0.3)
    p = orc.project(sc, cam, quantize=False)
    assert np.all(p["radius"] > 0)
    rng = np.random.default_rng(3)
    g = rng.standard_normal((256, 3))
    img, fT, nc, amb = orc.render(p, cam, bg=bg, band_alpha=1e-2, band_T=1e-2)
    assert not amb.any()
    g2, g2a, touched = orc.render_bwd(p, cam, g, bg=bg, band_alpha=1e-2, band_T=1e-2)
    grads = orc.project_bwd(sc, cam, g2)

    def loss(s):
        q = orc.project(s, cam, quantize=False)
        im, *_ = orc.render(q, cam, bg=bg)
        return float((im * g).sum())

    names = ["means", "quats", "log_scales", "opacity_logits", "sh"]
    worst = 0.0
    for name in names:
        arr = getattr(sc, name)
        an = grads[name].reshape(arr.shape)
        for idx in np.ndindex(arr.shape):
            x0 = float(arr[idx])
            h = 1e-4 * max(1.0, abs(x0))
            sp = scenes.Scene(*(getattr(sc, k).astype(np.float64).copy() for k in names), deg)
            getattr(sp, name)[idx] = x0 + h
            lp = loss(sp)
            getattr(sp, name)[idx] = x0 - h
            lm = loss(sp)
            fd = (lp - lm) / (2 * h)
            err = abs(fd - an[idx]) / max(abs(fd), 1e-2)
            worst = max(worst, err)
            assert err < 1e-3, (name, idx, fd, an[idx])
    assert worst < 1e-3


def test_project_bwd_matches_central_differences_of_projection(orc):
    """The dual-number Jacobian against finite differences of each projected output."""
    rng = np.random.default_rng(2)
    cam = scenes.box100k(poses=2).cameras[0]
    sc = scenes.random_scene(rng, 6, 3, mean_box=1.0, log_scale=(-3.0, -1.5))
    p = orc.project(sc, cam, quantize=False)
    vis = np.nonzero(p["radius"])[0]
    assert len(vis) >= 4
    names = ["means", "quats", "log_scales", "opacity_logits", "sh"]
    for q in range(9):
        g2 = np.zeros((sc.n, 9))
        g2[:, q] = 1.0
        grads = orc.project_bwd(sc, cam, g2)
        for name in names:
            arr = getattr(sc, name)
            for i in vis:
                for j in np.ndindex(arr.shape[1:]):
                    idx = (i,) + j
                    x0 = float(arr[idx])
                    h = 1e-5 * max(1.0, abs(x0))
                    outs = []
                    for s in (+1, -1):
                        sp = scenes.Scene(*(getattr(sc, k).astype(np.float64).copy() for k in names), 3)
                        getattr(sp, name)[idx] = x0 + s * h
                        pp = orc.project(sp, cam, quantize=False, idx=[i])
                        v = np.concatenate([pp["xy"][0], pp["conic"][0], [pp["opacity"][0]], pp["rgb"][0]])
                        outs.append(v[q])
                    fd = (outs[0] - outs[1]) / (2 * h)
                    an = grads[name].reshape((sc.n,) + arr.shape[1:])[idx]
                    scale = max(abs(fd), 1e-6 * (1 + abs(v[q])))
                    assert abs(fd - an) <= 1e-4 * scale + 1e-9, (q, name, idx, fd, an)


def test_densify_statistic(orc):
    sc, cam = _fd_scene(4, 0)
    g2 = np.zeros((sc.n, 9))
    g2[:, 0] = [3.0, 0.0, -1.0, 2.0]
    g2[:, 1] = [4.0, 1.0, 0.0, 0.0]
    out = orc.project_bwd(sc, cam, g2, densify=True)
    np.testing.assert_allclose(out["densify_accum"], [5.0, 1.0, 1.0, 2.0])
    assert list(out["densify_count"]) == [1, 1, 1, 1]


# ---------------------------------------------------------------- Adam and L1

def test_adam_closed_forms(orc):
    rng = np.random.default_rng(0)
    p0 = rng.standard_normal(1000).astype(np.float32)
    g = (rng.standard_normal(1000) * 10.0 ** rng.uniform(-6, 2, 1000)).astype(np.float32)
    lr, b1, b2, eps = 1e-3, 0.9, 0.99, 1e-15
    m = np.zeros_like(p0)
    v = np.zeros_like(p0)
    p = p0
    for step in (1, 2, 3):     # a constant gradient moves every step by lr * sign(g)
        p, m, v = orc.adam(p, g, m, v, lr, b1, b2, eps, step)
        assert np.all(np.abs(p - (p0 - step * lr * np.sign(g))) <= 2e-6 + 1e-6 * np.abs(p0))
    # then a zero gradient after one step: move by lr * (b1/(1+b1)) / sqrt(b2/(1+b2)) * sign(g)
    p1, m1, v1 = orc.adam(p0, g, np.zeros_like(p0), np.zeros_like(p0), lr, b1, b2, eps, 1)
    p2, _, _ = orc.adam(p1, np.zeros_like(g), m1, v1, lr, b1, b2, eps, 2)
    step2 = lr * (b1 / (1 + b1)) / math.sqrt(b2 / (1 + b2))
    assert np.all(np.abs(p2 - (p1 - step2 * np.sign(g))) <= 2e-6 + 1e-6 * np.abs(p0))


def test_l1_worked_example(orc):
    img = np.array([0.5, 0.2, 0.9, 0.0], np.float32)
    tgt = np.array([0.1, 0.2, 1.0, 0.25], np.float32)
    loss, g = orc.l1(img, tgt)
    np.testing.assert_allclose(loss, (0.4 + 0.0 + 0.1 + 0.25) / 4, rtol=1e-6)
    assert list(g) == [0.25, 0.0, -0.25, -0.25]


def test_clamped_alpha_has_no_opacity_or_shape_gradient(orc):
    """At a pixel where o*G exceeds 0.99 the blended alpha is the constant 0.99:
    finite differences in the opacity logit and the mean are zero there, while the
    colour still receives alpha*T*g."""
    R, t = scenes.look_at((0.0, 0.0, -4.0))
    cam = scenes.camera(R, t, 20.0, 20.0, 8.0, 8.0, 16, 16)
    sc = one_scene([[0.0, 0.0, 0.0]], [[1, 0, 0, 0]], [[0.5] * 3], [8.0], [[[0.5 / C0, 0.0, 0.0]]], 0)
    p = orc.project(sc, cam, quantize=False)
    pix = [7 * 16 + 7]          # centre (7.5, 7.5) is 0.5 px from the mean at (8, 8)
    g = np.array([[1.0, 2.0, 3.0]])
    g2, _, _ = orc.render_bwd(p, cam, g, pix=pix)
    assert np.all(g2[0, :6] == 0.0)
    np.testing.assert_allclose(g2[0, 6:], 0.99 * np.array([1.0, 2.0, 3.0]), rtol=1e-12)
    grads = orc.project_bwd(sc, cam, g2)
    for name in ("means", "opacity_logits", "log_scales"):
        assert np.all(grads[name] == 0.0)


def _hand_projection(rows):
    """A projection dict built by hand: rows of (u, v, depth, isotropic conic c, opacity)."""
    n = len(rows)
    a = np.asarray(rows, np.float64)
    return {"xy": a[:, 0:2].copy(), "depth": a[:, 2].copy(),
            "conic": np.stack([a[:, 3], np.zeros(n), a[:, 3]], 1), "opacity": a[:, 4].copy(),
            "rgb": np.full((n, 3), 0.5), "radius": np.full(n, 3, np.int32),
            "rect": np.tile(np.array([0, 0, 1, 1], np.int32), (n, 1)),
            "tiles_touched": np.ones(n, np.uint32)}


def test_straddle_marks_only_the_gaussians_the_decision_can_change(orc):
    """The reverse pass excludes from comparison (touched) only the Gaussians whose gradient
    a straddling decision can change: after a skip/stop straddle every Gaussian that can
    blend at that pixel, not the far ones that merely share its tile; after a clamp
    straddle only the clamped entry (alpha is continuous across the clamp)."""
    cam = scenes.camera(np.eye(3), np.zeros(3), 16.0, 16.0, 8.0, 8.0, 16, 16)
    d = math.sqrt(2.0 * math.log(255.0 / 1.2))          # alpha = 1.2 / 255 at pixel (4, 4)
    rows = [(4.5, 4.5, 1.0, 1.0, 0.5),                   # C: blended at (4, 4)
            (4.5 + d, 4.5, 2.0, 1.0, 1.0),               # A: alpha 1.2/255 at (4, 4), inside a 0.5 band
            (14.5, 14.5, 3.0, 1.0, 0.9),                 # B: alpha ~ 1e-44 at (4, 4); 0.0017 at (12, 12)
            (12.5, 12.5, 4.0, 1.0, 0.99 * 1.001),        # D: clamped at (12, 12), inside a 0.01 band
            (12.5, 12.5, 5.0, 1.0, 0.3)]                 # E: blended at (12, 12) behind D
    p = _hand_projection(rows)
    up = np.array([[1.0, -0.5, 0.25]])
    _, amb = orc.render(p, cam, pix=np.array([4 * 16 + 4]), band_alpha=0.5, band_T=1e-4)[2:]
    assert amb[0] & 1
    _, _, touched = orc.render_bwd(p, cam, up, pix=np.array([4 * 16 + 4]), band_alpha=0.5, band_T=1e-4)
    assert list(touched) == [1, 1, 0, 0, 0]
    _, amb = orc.render(p, cam, pix=np.array([12 * 16 + 12]), band_alpha=0.01, band_T=1e-4)[2:]
    assert amb[0] == 2
    _, _, touched = orc.render_bwd(p, cam, up, pix=np.array([12 * 16 + 12]), band_alpha=0.01, band_T=1e-4)
    assert list(touched) == [0, 0, 0, 1, 0]


def _alt(p, i, scale):
    q = {k: v.copy() for k, v in p.items()}
    q["opacity"][i] *= scale
    return q


def test_straddle_allowance_is_the_difference_of_the_two_decisions(orc):
    """The straddle output of the reverse pass is, per Gaussian and component, the
    difference between the terms with a straddling decision taken each way.  Pinned
    against two renders whose opacity is nudged to either side of the threshold (far
    outside the band, so neither straddles): the skip test at 1/255, the stop test at
    T(1 - alpha) = 1e-4 and the 0.99 clamp."""
    cam = scenes.camera(np.eye(3), np.zeros(3), 16.0, 16.0, 8.0, 8.0, 16, 16)
    pix = np.array([4 * 16 + 4])
    up = np.array([[1.0, -0.5, 0.25]])
    band = dict(band_alpha=1e-5, band_T=1e-4)
    tiny = dict(band_alpha=1e-12, band_T=1e-12)
    # skip straddle: E's alpha at the pixel is (1/255)(1 + 2e-6)
    d = math.sqrt(2.0 * math.log(255.0 / (1.0 + 2e-6)))
    p = _hand_projection([(4.5, 4.5, 1.0, 1.0, 0.5),          # C in front, blended
                          (4.5 + d, 4.5, 2.0, 1.0, 1.0),      # E straddles the skip test
                          (4.5, 5.5, 3.0, 0.5, 0.3)])         # D behind, blended
    p["rgb"] = np.array([[0.9, 0.2, 0.1], [0.1, 0.8, 0.3], [0.3, 0.3, 0.9]])
    _, _, _, st = orc.render_bwd(p, cam, up, pix=pix, straddle=True, **band)
    hi = orc.render_bwd(_alt(p, 1, 1 + 2e-4), cam, up, pix=pix, **tiny)[0]
    lo = orc.render_bwd(_alt(p, 1, 1 - 2e-4), cam, up, pix=pix, **tiny)[0]
    want = np.abs(hi - lo)
    # E's own terms appear or vanish; D behind sees its T change; C in front (at its own
    # centre, so no position or shape terms) sees only the colour behind it change
    assert st[1].max() > 0 and st[2][6:].min() > 0 and st[0][5] > 0
    np.testing.assert_allclose(st, want, rtol=1e-3, atol=1e-15)

    # stop straddle: 13 entries of alpha 0.5, then one whose T(1 - alpha) is 1e-4 (1 + 3e-5)
    T13 = 0.5 ** 13
    ak = 1.0 - 1e-4 * (1.0 + 3e-5) / T13
    rows = [(4.5, 4.5, 1.0 + j, 0.5, 0.5) for j in range(13)] + [(4.5, 4.5, 20.0, 0.5, ak), (4.5, 4.5, 21.0, 0.5, 0.4)]
    p = _hand_projection(rows)
    p["rgb"] = np.linspace(0.1, 0.9, 3 * len(rows)).reshape(-1, 3)
    _, _, _, st = orc.render_bwd(p, cam, up, pix=pix, straddle=True, **band)
    hi = orc.render_bwd(_alt(p, 13, 1 + 1e-3), cam, up, pix=pix, **tiny)[0]   # stops there
    lo = orc.render_bwd(_alt(p, 13, 1 - 1e-3), cam, up, pix=pix, **tiny)[0]   # blends it
    want = np.abs(hi - lo)
    assert st[13].max() > 0 and np.all(st[14] == 0)
    np.testing.assert_allclose(st, want, rtol=1e-2, atol=1e-15)

    # clamp straddle: a single entry with o e^-sigma = 0.99 (1 + 2e-6) at the pixel
    p = _hand_projection([(4.5, 4.5, 1.0, 0.5, 0.99 * (1 + 2e-6))])
    _, _, _, st = orc.render_bwd(p, cam, up, pix=pix, straddle=True, **band)
    hi = orc.render_bwd(_alt(p, 0, 1 + 1e-3), cam, up, pix=pix, **tiny)[0]   # clamped
    lo = orc.render_bwd(_alt(p, 0, 1 - 1e-3), cam, up, pix=pix, **tiny)[0]   # not clamped
    assert np.all(st[0, 6:] == 0)        # the clamp does not change alpha, only its derivatives
    np.testing.assert_allclose(st[0, :6], np.abs(hi - lo)[0, :6], rtol=5e-3, atol=1e-15)

    # no straddle: nothing
    p = _hand_projection([(4.5, 4.5, 1.0, 1.0, 0.5)])
    _, _, _, st = orc.render_bwd(p, cam, up, pix=pix, straddle=True, **band)
    assert not st.any()
