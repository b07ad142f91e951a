"""Parity of the culled binning (gs_camera.tile_cull: a Gaussian binned only into
the tiles of its rectangle where its alpha can reach 1/255) against the oracle and
against the rectangle binning on the GPU:

  * the projection is the rectangle run's, bit for bit (the flag is the binning's);
  * the culled list is the oracle's rectangle list minus some instances, in the same
    order, keeping every instance the oracle's tile-reach bound says must stay and
    none it says must go; its ranges are its own;
  * image and final_T equal the rectangle run's bit for bit, and the oracle's within
    the image tolerance; n_contrib equals the oracle's (and the rectangle run's)
    moved into the shorter lists;
  * the 2D gradients match the oracle's;
  * at full size (a 1080p view of the 1M mixture, a 4K view of the 3M city) the whole
    list and every pixel;
  * the Trainer with and without culling gives the same losses and updates.
"""
import numpy as np
import pytest
import torch

from gaussian_splatting_differentiable_02_b200 import pipeline as pl
from gaussian_splatting_differentiable_02_b200 import scenes

from _parity import (BAND_ALPHA, BAND_T, CudaRun, check_culled_binning, check_grads, check_images,
                     check_projection, culled_n_contrib)

pytestmark = pytest.mark.gpu

LRS = {"means": 1.6e-4, "log_scales": 5e-3, "quats": 1e-3, "opacity_logits": 5e-2, "sh": 2.5e-3}


def _check_pair(orc, scene, cam, bg=(0.0, 0.0, 0.0), max_amb_frac=1e-3, backward=True):
    a = CudaRun(scene, cam, bg=bg)                   # rectangles
    b = CudaRun(scene, cam, bg=bg, tile_cull=True)   # culled
    ref = orc.project(scene, cam)
    pa, pb = a.projection(), b.projection()
    check_projection(pb, ref)
    for k in ("xy", "depth", "conic", "opacity", "rgb", "radius", "rect", "tiles_touched"):
        assert np.array_equal(pa[k], pb[k]), k
    keys, vals, ranges = orc.keys(ref, cam)
    tx, ty = orc.tiles(cam)
    ak, av, ar = a.sorted_instances()
    assert np.array_equal(ak, keys) and np.array_equal(av, vals) and np.array_equal(ar, ranges)
    gk, gv, gr = b.sorted_instances()
    pos = check_culled_binning(gk, gv, gr, ref, keys, vals, tx, ty)
    W = cam["width"]
    ia, Ta, na = a.images()
    ib, Tb, nb = b.images()
    assert np.array_equal(ia, ib) and np.array_equal(Ta, Tb)
    assert np.array_equal(culled_n_contrib(na, None, W, tx, ranges, pos, gr), nb)
    img, T, nc, amb = orc.render(ref, cam, bg=bg, band_alpha=BAND_ALPHA, band_T=BAND_T)
    check_images(ib, Tb, nb, img, T, culled_n_contrib(nc, None, W, tx, ranges, pos, gr), amb,
                 max_amb_frac=max_amb_frac)
    if backward:
        rng = np.random.default_rng(7)
        up = rng.standard_normal((cam["height"], W, 3)).astype(np.float32)
        g2_gpu = b.backward(up)
        g2, g2a, touched = orc.render_bwd(ref, cam, up.reshape(-1, 3).astype(np.float64), bg=bg,
                                          band_alpha=BAND_ALPHA, band_T=BAND_T)
        rows = np.nonzero(touched == 0)[0]
        for q, name in enumerate(["du", "dv", "dA", "dB", "dC", "do", "dr", "dg", "db"]):
            check_grads(g2_gpu[:, q], g2[:, q], name, rows=rows, ref_abs=g2a[:, q], max_bad_frac=0.002)
    return len(keys), len(gk)


def test_tiny_workload(orc):
    wl = scenes.tiny()
    K_rect, K_cull = _check_pair(orc, wl.scene, wl.cameras[0])
    assert 0 < K_cull < K_rect


def test_ragged_image_sh_degrees_and_a_background(orc):
    rng = np.random.default_rng(3)
    for deg in (1, 3):
        scene = scenes.random_scene(rng, 700, deg, log_scale=(-3.5, -1.5))
        R, t = scenes.look_at((0.3, -0.2, -4.0))
        cam = scenes.camera(R, t, 90.0, 90.0, 50.0, 18.5, 100, 37)     # 7 x 3 tiles, both edges ragged
        _check_pair(orc, scene, cam, bg=(0.0, 0.3, 0.7))


def test_low_opacities_reach_few_or_no_tiles(orc):
    """Opacity logits ~ N(-5, 1) (opacities around 0.007, most between 9e-4 and 0.05):
    those below about 1/255 get no instance at all."""
    rng = np.random.default_rng(8)
    scene = scenes.random_scene(rng, 1500, 0, log_scale=(-3.0, -1.5), logit=(-5.0, 1.0))
    cam = scenes.tiny().cameras[0]
    b = CudaRun(scene, cam, tile_cull=True)
    p = b.projection()
    vis = p["radius"] > 0
    faint = vis & (p["opacity"] < 1.0 / 255 * 0.999)
    assert faint.sum() > 100
    gk, gv, gr = b.sorted_instances()
    assert not np.isin(np.nonzero(faint)[0], gv.astype(np.int64)).any()
    _check_pair(orc, scene, cam)


def test_needles(orc):
    """Long thin Gaussians (scales e^-1.5 by e^-7) seen at 480x270: footprints far from
    their rectangles' shape, conics with condition numbers up to about 1e4."""
    rng = np.random.default_rng(9)
    n = 1200
    scene = scenes.random_scene(rng, n, 1, log_scale=(-7.0, -6.5))
    scene.log_scales[:, 0] = rng.uniform(-2.0, -1.0, n).astype(np.float32)
    R, t = scenes.look_at((0.5, -0.4, -4.0))
    cam = scenes.camera(R, t, 400.0, 400.0, 240.0, 135.0, 480, 270)
    K_rect, K_cull = _check_pair(orc, scene, cam, max_amb_frac=2e-3)
    assert K_cull < 0.8 * K_rect


def test_full_size_view_of_the_1m_mixture(orc):
    """One 1920x1080 view of the 1M mixture: the whole culled list against the oracle's
    rectangle list and tile-reach bound, and every pixel against the rectangle run."""
    wl = scenes.multiview1m()
    cam = wl.cameras[5]
    scene = wl.scene
    a = CudaRun(scene, cam, capacity=12_000_000)
    ia, Ta, na = a.images()
    ak, av, ar = a.sorted_instances()
    ak, av, ar = ak.copy(), av.copy(), ar.copy()
    del a
    torch.cuda.empty_cache()
    b = CudaRun(scene, cam, capacity=12_000_000, tile_cull=True)
    ref = orc.project(scene, cam)
    pb = b.projection()
    check_projection(pb, ref)
    keys, vals, ranges = orc.keys(ref, cam)
    assert np.array_equal(ak, keys) and np.array_equal(av, vals) and np.array_equal(ar, ranges)
    tx, ty = orc.tiles(cam)
    gk, gv, gr = b.sorted_instances()
    pos = check_culled_binning(gk, gv, gr, ref, keys, vals, tx, ty)
    assert len(gk) < 0.6 * len(keys)
    ib, Tb, nb = b.images()
    assert np.array_equal(ia, ib) and np.array_equal(Ta, Tb)
    assert np.array_equal(culled_n_contrib(na, None, cam["width"], tx, ranges, pos, gr), nb)


def test_full_size_4k_view_of_the_3m_city(orc):
    """One 3840x2160 view of the 3M city (15 tile bits, two tile passes): the whole
    culled list against the oracle's rectangle list and tile-reach bound, and every
    pixel against the rectangle run."""
    wl = scenes.city3m(poses=1)
    cam = wl.cameras[0]
    scene = wl.scene
    a = CudaRun(scene, cam, capacity=40_000_000)
    ia, Ta, na = a.images()
    ak, av, ar = (x.copy() for x in a.sorted_instances())
    del a
    torch.cuda.empty_cache()
    b = CudaRun(scene, cam, capacity=40_000_000, tile_cull=True)
    ref = orc.project(scene, cam)
    keys, vals, ranges = orc.keys(ref, cam)
    assert np.array_equal(ak, keys) and np.array_equal(av, vals) and np.array_equal(ar, ranges)
    del ak, av, ar
    tx, ty = orc.tiles(cam)
    gk, gv, gr = b.sorted_instances()
    pos = check_culled_binning(gk, gv, gr, ref, keys, vals, tx, ty)
    assert len(gk) < 0.8 * len(keys)
    ib, Tb, nb = b.images()
    assert np.array_equal(ia, ib) and np.array_equal(Ta, Tb)
    assert np.array_equal(culled_n_contrib(na, None, cam["width"], tx, ranges, pos, gr), nb)


def _cams(n_views, seed=0):
    rng = np.random.default_rng(seed)
    cams = []
    for _ in range(n_views):
        eye = rng.standard_normal(3)
        eye = 4.0 * eye / np.linalg.norm(eye)
        R, t = scenes.look_at(eye)
        cams.append(scenes.camera(R, t, 128.0, 128.0, 64.0, 64.0, 128, 128))
    return cams


@pytest.mark.parametrize("packed", [False, True])
def test_trainer_with_and_without_culling(packed):
    """Five views with densification statistics: the first step gives the same loss,
    visibility counts and images, with fewer instances; three steps give the same
    parameters up to the order of the atomic adds."""
    rng = np.random.default_rng(13)
    scene = scenes.random_scene(rng, 600, 1, mean_box=1.0, log_scale=(-3.5, -2.0))
    cams = _cams(5, 8)
    targets = [torch.from_numpy(rng.random((128, 128, 3)).astype(np.float32)).cuda() for _ in cams]
    out = []
    for cull in (False, True):
        g = pl.Gaussians.from_scene(scene)
        tr = pl.Trainer(g, [pl.View(scene.n, c) for c in cams], targets, dict(LRS), densify=True, packed=packed,
                        tile_cull=cull)
        tr.step()
        torch.cuda.synchronize()
        first = (tr.loss.item(), tr.densify_count.cpu().numpy(), tr.kcount.cpu().numpy().copy(),
                 [vw.image.cpu().numpy() for vw in tr.views])
        tr.step()
        tr.step()
        torch.cuda.synchronize()
        out.append((tr.gauss.to_numpy(), first))
    (a, (la, ca, ka, ima)), (b, (lb, cb, kb, imb)) = out
    assert abs(la - lb) <= 1e-12 * abs(la)
    assert np.array_equal(ca, cb)
    assert np.all(kb < ka)
    assert all(np.array_equal(x, y) for x, y in zip(ima, imb))
    for k in pl.PARAM_NAMES:
        close = np.abs(a[k] - b[k]) <= 1e-6 + 1e-5 * np.abs(a[k])
        assert close.mean() >= 0.999, (k, float(close.mean()))
