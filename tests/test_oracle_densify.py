"""Pins of the oracle's adaptive density control (orc_densify) against hand-built
cases whose decisions are fixed by construction, scipy's quaternion rotation, the
sample covariance of many split draws, and layout invariants.

Rule pinned here (gsplat guide, lmnt.cn/news/262699, §4.1, densify_and_prune with
a gradient threshold, a minimum opacity, an extent and a maximum screen size):
prune unless opacity >= min_opacity or when the largest radius seen exceeds the
screen limit; densify when count > 0 and accum / count >= the threshold, cloning
Gaussians whose largest scale is <= the scale threshold and splitting the rest
into two children drawn from the Gaussian with scales divided by 1.6."""
import math

import numpy as np
import pytest
from scipy.spatial.transform import Rotation

import oracle
from gaussian_splatting_differentiable_02_b200 import scenes

PRUNE, KEEP, CLONE, SPLIT = 0, 1, 2, 3


def _scene(n, sh_degree=1, seed=0):
    rng = np.random.default_rng(seed)
    return scenes.random_scene(rng, n, sh_degree)


def test_hand_built_decisions_and_layout():
    sc = _scene(8)
    sc.log_scales[:] = math.log(0.01)          # small: clone when densified
    sc.log_scales[5] = [math.log(0.2), math.log(0.01), math.log(0.01)]  # one large axis: split
    sc.opacity_logits[:] = 0.0                 # opacity 0.5
    sc.opacity_logits[0] = -10.0               # opacity 4.5e-5
    accum = np.array([1.0, 1.0, 1.0, 4e-4, 0.5, 1.0, 1.0, 1.0])
    count = np.array([1, 1, 0, 4, 2, 1, 1, 1], np.int32)
    radius = np.array([0, 100, 0, 0, 0, 0, 38, 39], np.int32)
    noise = np.zeros((8, 2, 3))
    r = oracle.densify(sc, accum, count, radius, noise, grad_threshold=0.25, scale_threshold=0.05,
                       min_opacity=0.005, max_screen_radius=38)
    # 0: opacity below the minimum, whatever its gradient; 1: screen radius 100 > 38;
    # 2: never visible (count 0); 3: mean 1e-4 below the threshold; 4: mean exactly
    # the threshold (0.5 / 2 = 0.25) and small -> clone; 5: large -> split;
    # 6: radius equal to the limit is kept, densified, small -> clone; 7: radius 39 > 38
    assert r["decision"].tolist() == [PRUNE, PRUNE, KEEP, KEEP, CLONE, SPLIT, CLONE, PRUNE]
    assert r["n_out"] == 8
    assert r["source"].tolist() == [2, 3, 4, 4, 5, 5, 6, 6]
    assert r["fresh"].tolist() == [False, False, False, True, True, True, False, True]
    # no screen test when the limit is 0
    r0 = oracle.densify(sc, accum, count, radius, noise, 0.25, 0.05, 0.005, 0)
    assert r0["decision"].tolist() == [PRUNE, CLONE, KEEP, KEEP, CLONE, SPLIT, CLONE, CLONE]


def test_opacity_bound_is_inclusive_and_nan_is_pruned():
    sc = _scene(3)
    sc.opacity_logits[:] = [0.0, -1e-6, np.nan]   # opacity 0.5 exactly, just below, NaN
    z = np.zeros(3)
    r = oracle.densify(sc, z, z.astype(np.int32), z.astype(np.int32), np.zeros((3, 2, 3)), 1.0, 1.0, 0.5, 0)
    assert r["decision"].tolist() == [KEEP, PRUNE, PRUNE]


def test_clone_is_an_exact_copy_and_kept_rows_are_unchanged():
    sc = _scene(200, sh_degree=3, seed=3)
    rng = np.random.default_rng(4)
    accum = rng.uniform(0, 1, 200)
    count = rng.integers(0, 3, 200).astype(np.int32)
    r = oracle.densify(sc, accum, count, np.zeros(200, np.int32), rng.standard_normal((200, 2, 3)),
                       0.3, 0.05, 0.005, 0)
    for key in ("means", "quats", "log_scales", "opacity_logits", "sh"):
        src = np.asarray(getattr(sc, key), np.float64)
        for k in range(r["n_out"]):
            i = r["source"][k]
            d = r["decision"][i]
            if d in (KEEP, CLONE):
                np.testing.assert_array_equal(r[key][k], src[i])
            elif key in ("quats", "opacity_logits", "sh"):
                np.testing.assert_array_equal(r[key][k], src[i])
    dec = r["decision"]
    assert r["n_out"] == np.sum(dec == KEEP) + 2 * np.sum(dec == CLONE) + 2 * np.sum(dec == SPLIT)
    assert np.all(np.diff(r["source"]) >= 0)
    assert {CLONE, SPLIT, KEEP} <= set(dec.tolist())


def test_split_children_against_scipy_rotation():
    sc = _scene(1)
    sc.quats[0] = 2.0 * np.array([0.3, -0.5, 0.7, 0.2]) / np.linalg.norm([0.3, -0.5, 0.7, 0.2])  # not unit
    sc.log_scales[0] = np.log([0.3, 0.05, 0.1])
    sc.means[0] = [0.25, -0.5, 1.0]
    noise = np.array([[[0.5, -1.0, 2.0], [-1.5, 0.25, 0.75]]])
    r = oracle.densify(sc, np.ones(1), np.ones(1, np.int32), np.zeros(1, np.int32), noise, 0.5, 0.01, 0.0, 0,
                       quantize=False)
    assert r["decision"].tolist() == [SPLIT] and r["fresh"].tolist() == [True, True]
    w, x, y, z = sc.quats[0].astype(np.float64)
    rot = Rotation.from_quat([x, y, z, w])         # scipy is scalar-last and normalises
    s = np.exp(sc.log_scales[0].astype(np.float64))
    for j in range(2):
        want = sc.means[0].astype(np.float64) + rot.apply(s * noise[0, j])
        np.testing.assert_allclose(r["means"][j], want, rtol=0, atol=1e-14)
        # scale divided by 1.6
        np.testing.assert_allclose(np.exp(r["log_scales"][j]) * 1.6, s, rtol=1e-14)


def test_split_children_sample_the_gaussian():
    """Children of one Gaussian over many N(0, I) draws have the Gaussian's mean and
    covariance R diag(s^2) R^T (scipy rotation matrix), within sampling error."""
    m = 20000
    sc = _scene(m)
    q = np.array([0.8, 0.1, -0.4, 0.3])
    sc.quats[:] = q
    sc.log_scales[:] = np.log([0.2, 0.05, 0.1])
    sc.means[:] = [1.0, 2.0, -1.0]
    sc.opacity_logits[:] = 0.0
    noise = np.random.default_rng(7).standard_normal((m, 2, 3))
    r = oracle.densify(sc, np.ones(m), np.ones(m, np.int32), np.zeros(m, np.int32), noise, 0.5, 0.01, 0.0, 0,
                       quantize=False)
    kids = r["means"]
    assert kids.shape == (2 * m, 3)
    Rm = Rotation.from_quat([q[1], q[2], q[3], q[0]]).as_matrix()
    cov = Rm @ np.diag(np.array([0.2, 0.05, 0.1]) ** 2) @ Rm.T
    emp = np.cov((kids - [1.0, 2.0, -1.0]).T, bias=True)
    # standard error of a covariance entry ~ sqrt((s_ii s_jj + s_ij^2) / N)
    se = np.sqrt((np.outer(np.diag(cov), np.diag(cov)) + cov ** 2) / (2 * m))
    assert np.all(np.abs(emp - cov) < 5 * se + 1e-12)
    np.testing.assert_allclose(kids.mean(0), [1.0, 2.0, -1.0], atol=5 * 0.2 / math.sqrt(2 * m))


def test_moments_carry_over():
    sc = _scene(50, seed=9)
    rng = np.random.default_rng(10)
    accum = rng.uniform(0, 1, 50)
    count = np.ones(50, np.int32)
    m = {"means": rng.standard_normal((50, 3)), "quats": rng.standard_normal((50, 4)),
         "log_scales": rng.standard_normal((50, 3)), "opacity_logits": rng.standard_normal(50),
         "sh": rng.standard_normal((50, 4, 3))}
    r = oracle.densify(sc, accum, count, np.zeros(50, np.int32), rng.standard_normal((50, 2, 3)), 0.5, 0.02, 0.005,
                       0, moments=[m])
    (mm,) = r["moments"]
    for key in m:
        for k in range(r["n_out"]):
            if r["fresh"][k]:
                assert np.all(mm[key][k] == 0)
            else:
                np.testing.assert_array_equal(mm[key][k], m[key][r["source"][k]])


@pytest.mark.parametrize("n", [0, 1])
def test_degenerate_sizes(n):
    sc = _scene(max(n, 1))
    if n == 0:
        sc = sc.subset(np.arange(0))
    r = oracle.densify(sc, np.ones(n), np.ones(n, np.int32), np.zeros(n, np.int32), np.zeros((n, 2, 3)),
                       0.5, 1.0, 0.0, 0)
    assert r["n_out"] == (0 if n == 0 else 2)
