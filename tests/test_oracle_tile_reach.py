"""Pins of the oracle's tile-reach bound (the smallest sigma of a Gaussian's
footprint over a tile's box of pixel centres), on which the culled binning's
parity rests: closed forms, brute force over the box, and the class rule on
hand-made instances."""
import numpy as np
import pytest

import oracle as orc


def _brute_min(u, v, A, B, C, tx, ty, widen=0.0, n=801):
    """Minimum of sigma over an n x n grid of the box plus a dense sampling of its four edges."""
    x0, x1 = 16 * tx + 0.5 - widen, 16 * tx + 15.5 + widen
    y0, y1 = 16 * ty + 0.5 - widen, 16 * ty + 15.5 + widen
    xs = np.linspace(x0, x1, n)
    ys = np.linspace(y0, y1, n)
    X, Y = np.meshgrid(xs, ys)
    dx, dy = X - u, Y - v
    grid = 0.5 * (A * dx * dx + C * dy * dy) + B * dx * dy
    e = np.linspace(0.0, 1.0, 200001)
    ex = x0 + (x1 - x0) * e
    ey = y0 + (y1 - y0) * e
    edges = []
    for xe in (x0, x1):
        ddx, ddy = xe - u, ey - v
        edges.append(0.5 * (A * ddx * ddx + C * ddy * ddy) + B * ddx * ddy)
    for ye in (y0, y1):
        ddx, ddy = ex - u, ye - v
        edges.append(0.5 * (A * ddx * ddx + C * ddy * ddy) + B * ddx * ddy)
    return min(grid.min(), min(x.min() for x in edges))


def _random_conic(rng):
    """Inverse of R diag(s1^2, s2^2) R^T with scales from 0.3 to 40 px and any angle."""
    s = np.exp(rng.uniform(np.log(0.3), np.log(40.0), 2))
    t = rng.uniform(0, np.pi)
    R = np.array([[np.cos(t), -np.sin(t)], [np.sin(t), np.cos(t)]])
    inv = R @ np.diag(1.0 / s ** 2) @ R.T
    return inv[0, 0], inv[0, 1], inv[1, 1]


def test_isotropic_closed_form():
    """A = C = a, B = 0: sigma = a/2 |d|^2, so the minimum is a/2 times the squared
    distance from the mean to the box."""
    rng = np.random.default_rng(0)
    for _ in range(200):
        a = np.exp(rng.uniform(-6, 2))
        u, v = rng.uniform(-40, 80, 2)
        tx, ty = 1, 2
        x0, x1, y0, y1 = 16.5, 31.5, 32.5, 47.5
        ddx = max(x0 - u, 0.0, u - x1)
        ddy = max(y0 - v, 0.0, v - y1)
        want = 0.5 * a * (ddx * ddx + ddy * ddy)
        got = orc.tile_min_sigma([[u, v]], [[a, 0.0, a]], [tx], [ty])[0]
        assert abs(got - want) <= 1e-12 * max(1.0, want)


def test_mean_inside_the_box_is_zero_and_outside_positive():
    got = orc.tile_min_sigma([[20.0, 40.0], [20.0, 60.0]], [[0.5, 0.2, 0.3]] * 2, [1, 1], [2, 2])
    assert got[0] == 0.0 and got[1] > 0.0


def test_anisotropic_against_brute_force():
    """Random rotated ellipses (scales 0.3..40 px) and means inside, beside and far
    from the box: the closed minimum is never above the sampled minimum and within the
    sampling resolution of it."""
    rng = np.random.default_rng(1)
    for k in range(150):
        A, B, C = _random_conic(rng)
        u, v = rng.uniform(-30, 80, 2)
        widen = [0.0, 4.0 / 1024][k % 2]
        got = orc.tile_min_sigma([[u, v]], [[A, B, C]], [1], [2], widen)[0]
        brute = _brute_min(u, v, A, B, C, 1, 2, widen)
        assert got <= brute + 1e-12 * max(1.0, brute)
        # the edge sampling step is 15/200000 px: sigma moves by at most |grad| * step there
        grad = np.hypot(A, C) * 200.0 + abs(B) * 200.0
        assert brute - got <= grad * 15.0 / 200000 + 1e-12, (k, got, brute)


def test_widening_grows_the_box():
    rng = np.random.default_rng(2)
    for _ in range(100):
        A, B, C = _random_conic(rng)
        u, v = rng.uniform(-30, 80, 2)
        a = orc.tile_min_sigma([[u, v]], [[A, B, C]], [1], [2], 0.0)[0]
        b = orc.tile_min_sigma([[u, v]], [[A, B, C]], [1], [2], 0.01)[0]
        assert b <= a


def test_not_positive_definite_is_nan():
    got = orc.tile_min_sigma([[0.0, 0.0]] * 3, [[1.0, 2.0, 1.0], [-1.0, 0.0, 1.0], [1.0, 0.0, 0.0]], [1] * 3, [1] * 3)
    assert np.all(np.isnan(got))


def test_classes_on_hand_made_instances():
    """A unit-opacity round splat of sigma_px = 2 (A = C = 1/4): ln(255) = 5.54, so the
    footprint reaches sqrt(2 ln 255 / A) = 6.66 px from the mean.  Tile (0, 0)'s box of
    centres is [0.5, 15.5]^2; a mean at x = 15.5 + d, y = 8 is d px from it."""
    r = np.sqrt(2.0 * np.log(255.0) / 0.25)
    tiles_x = 4
    rows = []
    for d in (r - 0.01, r + 0.001, r + 0.1):
        rows.append((15.5 + d, 8.0))
    proj = {"xy": np.array(rows), "conic": np.array([[0.25, 0.0, 0.25]] * 3), "opacity": np.ones(3)}
    keys = np.zeros(3, np.uint64)   # tile 0 for every instance
    vals = np.arange(3, dtype=np.uint32)
    keep, drop = orc.tile_reach_classes(proj, keys, vals, tiles_x)
    assert list(keep) == [True, False, False]
    # r + 0.001 lies inside the band a culled binning may keep; r + 0.1 does not
    assert list(drop) == [False, False, True]
    # an opacity of 1/255 reaches only the mean's own point, 0 none
    proj["opacity"] = np.array([1.0 / 255.0, 0.0, 1.0])
    proj["xy"] = np.array([[8.0, 8.0], [8.0, 8.0], [60.0, 8.0]])
    keep, drop = orc.tile_reach_classes(proj, keys, vals, tiles_x)
    assert keep[0] and not drop[0]
    assert drop[1] and not keep[1]
    assert drop[2] and not keep[2]
    # a form that is not positive definite keeps its tile
    proj["conic"] = np.array([[1.0, 2.0, 1.0], [0.25, 0.0, 0.25], [0.25, 0.0, 0.25]])
    proj["opacity"] = np.ones(3)
    keep, drop = orc.tile_reach_classes(proj, keys, vals, tiles_x)
    assert keep[0] and not drop[0]


def test_culled_list_checks_accept_valid_and_reject_broken_lists():
    """The parity helper of the culled binning, on the oracle's own list of the tiny
    workload: the list without its must-go instances passes; one without a must-stay
    instance, one with a must-go instance, or one out of order fails; the n_contrib
    move into the shorter list lands on the same instances."""
    import sys, os
    sys.path.insert(0, os.path.dirname(__file__))
    from _parity import _ranges_of, check_culled_binning, culled_n_contrib
    from gaussian_splatting_differentiable_02_b200 import scenes
    wl = scenes.tiny()
    cam = wl.cameras[0]
    ref = orc.project(wl.scene, cam)
    keys, vals, ranges = orc.keys(ref, cam)
    tx, ty = orc.tiles(cam)
    keep, drop = orc.tile_reach_classes(ref, keys, vals, tx)
    assert keep.sum() > 0 and drop.sum() > 0 and not (keep & drop).any()
    sel = ~drop
    gk, gv = keys[sel], vals[sel]
    touched = np.bincount(gv.astype(np.int64), minlength=wl.scene.n)
    pos = check_culled_binning(gk, gv, _ranges_of(gk, tx * ty), ref, keys, vals, tx, ty, touched)
    assert np.array_equal(np.nonzero(pos >= 0)[0], np.nonzero(sel)[0])
    img, T, nc, amb = orc.render(ref, cam)
    mapped = culled_n_contrib(nc, None, cam["width"], tx, ranges, pos, _ranges_of(gk, tx * ty))
    assert (mapped >= 0).all() and (mapped <= nc).all() and (mapped[nc > 0] > 0).all()
    # the mapped position holds the same Gaussian as the oracle's last blended entry
    W = cam["width"]
    p = np.nonzero(nc > 0)[0]
    t = (p // W // 16) * tx + (p % W) // 16
    gr = _ranges_of(gk, tx * ty)
    assert np.array_equal(gv[gr[t, 0] + mapped[p] - 1], vals[ranges[t, 0].astype(np.int64) + nc[p] - 1])
    # broken lists
    must = np.nonzero(keep)[0]
    sel2 = sel.copy()
    sel2[must[len(must) // 2]] = False
    with pytest.raises(AssertionError):
        check_culled_binning(keys[sel2], vals[sel2], _ranges_of(keys[sel2], tx * ty), ref, keys, vals, tx, ty)
    sel3 = sel.copy()
    sel3[np.nonzero(drop)[0][0]] = True
    with pytest.raises(AssertionError):
        check_culled_binning(keys[sel3], vals[sel3], _ranges_of(keys[sel3], tx * ty), ref, keys, vals, tx, ty)
    swapped_k, swapped_v = gk.copy(), gv.copy()
    swapped_k[[3, 4]] = swapped_k[[4, 3]]
    swapped_v[[3, 4]] = swapped_v[[4, 3]]
    with pytest.raises(AssertionError):
        check_culled_binning(swapped_k, swapped_v, _ranges_of(gk, tx * ty), ref, keys, vals, tx, ty)


def test_every_blending_pixel_lies_in_a_must_keep_instance():
    """Against the compositing rule itself: for every instance of the tiny workload's
    rectangle binning and every pixel centre of its tile, alpha = o e^-sigma >= 1/255
    there implies the instance is one the culled binning must keep; and an instance the
    rule lets go has alpha below 1/255 at all of its tile's pixel centres."""
    from gaussian_splatting_differentiable_02_b200 import scenes
    wl = scenes.tiny()
    cam = wl.cameras[0]
    ref = orc.project(wl.scene, cam)
    keys, vals, _ = orc.keys(ref, cam)
    tx, _ = orc.tiles(cam)
    keep, drop = orc.tile_reach_classes(ref, keys, vals, tx)
    gid = vals.astype(np.int64)
    tile = (keys >> np.uint64(32)).astype(np.int64)
    u, v = ref["xy"][gid].T
    A, B, C = ref["conic"][gid].T
    o = ref["opacity"][gid]
    px = 16.0 * (tile % tx)[:, None] + np.arange(16)[None, :] + 0.5        # [K, 16]
    py = 16.0 * (tile // tx)[:, None] + np.arange(16)[None, :] + 0.5
    dx = px[:, None, :] - u[:, None, None]                                  # [K, 16 rows, 16 cols]
    dy = py[:, :, None] - v[:, None, None]
    sig = 0.5 * (A[:, None, None] * dx * dx + C[:, None, None] * dy * dy) + B[:, None, None] * dx * dy
    alpha_max = (o[:, None, None] * np.exp(-sig)).reshape(len(gid), -1).max(axis=1)
    blends = alpha_max >= 1.0 / 255.0
    assert blends.sum() > 1000
    assert keep[blends].all()
    assert (alpha_max[drop] < 1.0 / 255.0).all()
    # the culling is worth having: many instances reach no pixel
    assert (~blends).sum() > 0.2 * len(gid)
