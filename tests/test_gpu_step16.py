"""Parity of the benchmarked training step at its full size: one Trainer.step() of the
1M-Gaussian 64-cluster mixture seen from its 16 poses at 1920x1080, in the
configuration the benchmark times (every view projected, one batched depth order of
the 16 views, binning from that order with two tile passes on a high-priority stream,
compositing on three streams, L1 loss, the fused 16-view backward through the
projection with the densification statistics and Adam on all five groups), against
the oracle:

  * every view's projection (features <= 1 ulp, integers exact), and its complete
    sorted instance list and tile ranges: the binning the benchmark runs is the
    culled one (each Gaussian only in the tiles its footprint reaches), checked as
    the oracle's rectangle list less instances the oracle's tile-reach bound lets
    go, keeping all it must keep, in the same order, with its own ranges;
  * per view, image, final T and n_contrib (moved into the culled lists) on every
    pixel of a set of tiles (the heaviest, ragged edges, random tiles, and the tiles
    of the sampled Gaussians below), and dL/dimage of the L1 loss there;
  * per view, the 2D gradients (full L1 upstream) of every Gaussian whose tile
    rectangle lies inside the rendered tiles, so the oracle sees all of its pixels;
  * for a sample of Gaussians covered that way in every view: the densification
    statistics and the parameters and Adam moments after the step, against the sum
    over views of the oracle's chain of its own 2D gradients followed by the
    oracle's Adam; the tolerance is the spec one plus what the measured 2D
    differences move each gradient through the chain (|J| |d2D|).

A second test runs the fused 16-view backward with Adam at the same size on seeded
2D gradients and checks 3000 sampled Gaussians against the oracle's chain and Adam.
"""
import numpy as np
import pytest
import torch

from gaussian_splatting_differentiable_02_b200 import pipeline as pl
from gaussian_splatting_differentiable_02_b200 import scenes

from _parity import (AMB_FRAC_LONG_LISTS, BAND_ALPHA, BAND_T, G_ATOL, G_RTOL, SUM_BOUND, check_culled_binning,
                     check_grads, check_images, check_projection, culled_n_contrib)

pytestmark = pytest.mark.gpu

NAMES = pl.PARAM_NAMES
EPS32 = float(np.finfo(np.float32).eps)


@pytest.fixture(scope="module")
def stepped():
    wl = scenes.multiview1m(views=16)
    n = wl.scene.n
    gauss = pl.Gaussians.from_scene(wl.scene)
    views = [pl.View(n, c) for c in wl.cameras]
    targets = [torch.from_numpy(t).cuda() for t in wl.targets]
    # the benchmark's Trainer: densify statistics, 3 streams, batched depth order, one view group
    tr = pl.Trainer(gauss, views, targets, dict(wl.adam_lr), densify=True, streams=3, batched_sort=True, groups=1)
    tr.step()
    torch.cuda.synchronize()
    assert tr.step_count == 1 and tr.depth_orders is not None
    yield wl, tr
    del tr
    torch.cuda.empty_cache()


def _gpu_projection(tr, k):
    p = tr.projs[k]
    return {"xy": p.xy.cpu().numpy(), "depth": p.depth.cpu().numpy(),
            "conic": p.conic_opacity[:, :3].cpu().numpy(), "opacity": p.conic_opacity[:, 3].cpu().numpy(),
            "rgb": p.rgb[:, :3].cpu().numpy(), "radius": tr.radii[k].cpu().numpy(),
            "rect": p.rect.cpu().numpy().astype(np.int32) & 0xffff,
            "tiles_touched": p.tiles_touched.cpu().numpy().astype(np.uint32)}


def _tile_pixels(tiles, tx, W, H):
    pix = []
    for t in sorted(tiles):
        x0, y0 = (t % tx) * 16, (t // tx) * 16
        ys = np.arange(y0, min(y0 + 16, H))
        xs = np.arange(x0, min(x0 + 16, W))
        pix.append((ys[:, None] * W + xs[None, :]).reshape(-1))
    return np.concatenate(pix).astype(np.int64)


def _rect_tiles(rect, tx):
    return [y * tx + x for y in range(rect[1], rect[3]) for x in range(rect[0], rect[2])]


def _natural(g: pl.Gaussians, idx, deg):
    """Rows idx of GPU parameter-shaped arrays in the oracle's natural layout."""
    ti = torch.from_numpy(np.asarray(idx, np.int64)).cuda()
    return {"means": g.means[ti, :3].cpu().numpy(), "quats": g.quats[ti].cpu().numpy(),
            "log_scales": g.log_scales[ti, :3].cpu().numpy(), "opacity_logits": g.opacity_logits[ti].cpu().numpy(),
            "sh": pl.planes_to_sh(g.sh[:, ti].cpu().numpy(), deg)}


def _scene_natural(scene, idx):
    return {"means": scene.means[idx], "quats": scene.quats[idx], "log_scales": scene.log_scales[idx],
            "opacity_logits": scene.opacity_logits[idx], "sh": scene.sh[idx]}


def test_benchmarked_step_matches_oracle(orc, stepped):
    wl, tr = stepped
    scene, cams = wl.scene, wl.cameras
    n, deg, nv = scene.n, scene.sh_degree, len(cams)
    W, H = cams[0]["width"], cams[0]["height"]
    tx, ty = (W + 15) // 16, (H + 15) // 16
    rng = np.random.default_rng(0)
    counts = tr.kcount.cpu().numpy()

    # ---- pass 1: projection and the complete sorted lists of every view, bit-exact
    rects, visible, lengths = [], [], []
    moved = []   # culled binning: per view, the oracle's list index -> the GPU list index, and both ranges
    for k, cam in enumerate(cams):
        ref = orc.project(scene, cam)
        check_projection(_gpu_projection(tr, k), ref)
        keys, vals, ranges = orc.keys(ref, cam)
        K = int(counts[k])
        view = tr.views[k]
        gk = view.keys[:K].cpu().numpy().view(np.uint64)
        gv = view.vals[:K].cpu().numpy().view(np.uint32)
        gr = view.ranges.cpu().numpy().view(np.uint32)
        if tr.tile_cull:
            # the oracle's rectangle list less what the tile-reach bound lets go, in order
            pos = check_culled_binning(gk, gv, gr, ref, keys, vals, tx, ty)
            assert K < 0.6 * len(keys), (k, K, len(keys))
            moved.append((pos.astype(np.int32), ranges.astype(np.int64), gr.astype(np.int64)))
        else:
            assert K == len(keys), (k, K, len(keys))
            assert np.array_equal(gk, keys), k
            assert np.array_equal(gv, vals), k
            assert np.array_equal(gr, ranges), k
        rects.append(ref["rect"].copy())
        visible.append(ref["radius"] > 0)
        lengths.append((ranges[:, 1].astype(np.int64) - ranges[:, 0]))
        del keys, vals, ref

    # ---- the Gaussians whose update is checked: from a random pool of Gaussians visible in
    # at least half of the views, the ones whose tiles in all views hold the shortest lists
    # (cheap for the oracle), plus random ones
    seen = np.sum(visible, axis=0)
    pool = rng.choice(np.nonzero(seen >= nv // 2)[0], 4000, replace=False)
    cost = np.zeros(len(pool))
    for k in range(nv):
        for j, i in enumerate(pool):
            if visible[k][i]:
                cost[j] += lengths[k][_rect_tiles(rects[k][i], tx)].sum()
    order = np.argsort(cost)
    sample = np.sort(np.concatenate([pool[order[:64]], rng.choice(pool[order[64:]], 32, replace=False)]))

    # ---- pass 2: per view, images, dL/dimage and 2D gradients on a set of tiles
    per_view = []
    n_amb_total = n_px_total = 0
    sign_amb_total = 0
    n_allow_total = n_elem_total = 0
    for k, cam in enumerate(cams):
        view = tr.views[k]
        lens = lengths[k]
        tiles = set(int(t) for t in np.argsort(-lens)[:4])
        tiles |= {tx * ty - 1, (ty - 1) * tx, tx - 1, tx * (ty // 2) + tx - 1}
        tiles |= set(int(t) for t in rng.choice(tx * ty, 8, replace=False))
        for i in sample:
            if visible[k][i]:
                tiles |= set(_rect_tiles(rects[k][i], tx))
        pix = _tile_pixels(tiles, tx, W, H)
        ref = orc.project(scene, cam)
        img, T, nc, amb = orc.render(ref, cam, pix=pix, band_alpha=BAND_ALPHA, band_T=BAND_T)
        gi = view.image.cpu().numpy().reshape(-1, 3)[pix]
        gT = view.final_T.cpu().numpy().reshape(-1)[pix]
        gn = view.n_contrib.cpu().numpy().reshape(-1)[pix]
        if tr.tile_cull:   # n_contrib counts positions in the culled lists
            pos, rr, gr = moved[k]
            nc = culled_n_contrib(nc, pix, W, tx, rr, pos, gr)
        err, namb = check_images(gi, gT, gn, img, T, nc, amb, max_amb_frac=AMB_FRAC_LONG_LISTS)
        n_amb_total += namb
        n_px_total += len(pix)

        # L1 upstream from the oracle's own image: sign(image - target) / (3 H W), sign(0) = 0
        tgt = wl.targets[k].reshape(-1, 3)[pix]
        _, g_sub = orc.l1(img.astype(np.float32), tgt)
        up = np.sign(g_sub.astype(np.float64)) / (3.0 * W * H)
        # a pixel whose image lies within the image tolerance of its target may take the
        # other sign on the GPU: its dL/dimage is not compared, and the Gaussians that take
        # a term there are left out of the gradient comparisons below
        sign_flip = np.any(np.abs(img - tgt.astype(np.float64)) <= 1e-5, axis=1)
        gd = view.dL_dimage.cpu().numpy().reshape(-1, 3)[pix]
        cmp = ~sign_flip & (amb == 0)
        assert np.array_equal(gd[cmp], up[cmp].astype(np.float32)), k
        sign_amb_total += int(sign_flip.sum())

        g2, g2a, _, straddle = orc.render_bwd(ref, cam, up, pix=pix, band_alpha=BAND_ALPHA, band_T=BAND_T,
                                              straddle=True)
        # what a straddling decision the GPU may take the other way moves (the oracle's
        # difference of the two results), plus, at a pixel whose sign of (image - target)
        # is not decided, the terms of a reversed upstream on that channel
        allow = straddle.copy()
        if sign_flip.any():
            flip_up = np.where(np.abs(img - tgt.astype(np.float64))[sign_flip] <= 1e-5, 2.0 / (3.0 * W * H), 0.0)
            _, ga, _ = orc.render_bwd(ref, cam, flip_up, pix=pix[sign_flip])
            allow += ga
        # Gaussians whose whole tile rectangle was rendered: their oracle 2D gradient is complete
        # (a summed-area table of the tiles not rendered, queried over every rectangle)
        vis = visible[k]
        notin = np.ones((ty, tx), np.int64)
        tl = np.array(sorted(tiles))
        notin[tl // tx, tl % tx] = 0
        sat = np.zeros((ty + 1, tx + 1), np.int64)
        sat[1:, 1:] = notin.cumsum(0).cumsum(1)
        rc = rects[k].astype(np.int64)
        x0, y0, x1, y1 = rc[:, 0], rc[:, 1], rc[:, 2], rc[:, 3]
        missing = sat[y1, x1] - sat[y0, x1] - sat[y1, x0] + sat[y0, x0]
        inside = vis & (missing == 0)
        rows = np.nonzero(inside)[0]
        assert len(rows) > 500, (k, len(rows))
        g2_gpu = tr.grad2ds[k].as_rows().astype(np.float64)
        # per element: the benchmark spec's tolerance (its absolute part scaled to this upstream,
        # 1 / (3 H W) per pixel instead of N(0, 1)), the float32 summation bound of a
        # cancelling sum, and the straddle allowance; no Gaussian is left out
        atol = G_ATOL / (3.0 * W * H)
        dd = np.abs(g2_gpu[rows] - g2[rows])
        bound = atol + G_RTOL * np.abs(g2[rows]) + SUM_BOUND * g2a[rows] + 1.01 * allow[rows]
        assert np.all(dd <= bound), (k, int((dd > bound).sum()), float(np.max(dd - bound)))
        strict = dd <= atol + G_RTOL * np.abs(g2[rows])
        n_allow = int((~strict).sum())
        print(f"view {k}: K={int(counts[k])}, {len(tiles)} tiles / {len(pix)} px, max img err {err:.2e}, "
              f"{namb} ambiguous px, {int(sign_flip.sum())} sign-ambiguous px, {len(rows)} Gaussians' 2D gradients, "
              f"{n_allow} of {dd.size} elements within the summation or straddle allowance only")
        n_allow_total += n_allow
        n_elem_total += dd.size

        # the sampled Gaussians' 2D gradients and the chain's columns in this view
        Jk = []
        for q in range(9):
            e = np.zeros((len(sample), 9))
            e[:, q] = 1.0
            Jk.append(orc.project_bwd(scene, cam, e, idx=sample))
        pb = orc.project_bwd(scene, cam, g2[sample], idx=sample, densify=True)
        per_view.append({"g2": g2[sample], "g2a": g2a[sample], "gpu": g2_gpu[sample], "vis": vis[sample], "J": Jk,
                         "pb": pb})
        del ref, g2, g2a

    assert n_amb_total <= AMB_FRAC_LONG_LISTS * n_px_total

    # at most 1% of the compared 2D gradient elements pass through an allowance only
    assert n_allow_total <= 0.01 * n_elem_total, (n_allow_total, n_elem_total)

    # ---- the update of the sampled Gaussians: sum over views of the oracle's chain, then Adam;
    # every sampled Gaussian is checked, the measured 2D differences (bounded above)
    # propagated through the chain into each tolerance
    m = len(sample)
    g_ref = {k: 0.0 for k in NAMES}
    prop = {k: 0.0 for k in NAMES}
    sumb = {k: 0.0 for k in NAMES}
    acc_ref = np.zeros(m)
    cnt_ref = np.zeros(m, np.int64)
    acc_tol = np.zeros(m)
    for pv in per_view:
        d = np.abs(pv["gpu"] - pv["g2"])
        for k in NAMES:
            g_ref[k] = g_ref[k] + np.asarray(pv["pb"][k], np.float64).reshape(m, -1)
            for q in range(9):
                col = np.abs(np.asarray(pv["J"][q][k], np.float64)).reshape(m, -1)
                prop[k] = prop[k] + col * d[:, q:q + 1]
                sumb[k] = sumb[k] + col * np.abs(pv["g2"][:, q:q + 1])
        acc_ref += pv["pb"]["densify_accum"]
        cnt_ref += pv["pb"]["densify_count"]
        acc_tol += np.hypot(d[:, 0], d[:, 1]) * pv["vis"]
    got_acc = tr.densify_accum[torch.from_numpy(sample).cuda()].cpu().numpy()
    got_cnt = tr.densify_count[torch.from_numpy(sample).cuda()].cpu().numpy()
    assert np.array_equal(got_cnt, cnt_ref)
    assert np.all(np.abs(got_acc - acc_ref) <= 1.01 * acc_tol + 1e-6 * acc_ref + 1e-30)

    after = _natural(tr.gauss, sample, deg)
    m1 = _natural(tr.m, sample, deg)
    v1 = _natural(tr.v, sample, deg)
    before = _scene_natural(scene, sample)
    b1, b2, eps = (float(np.float32(x)) for x in (*scenes.ADAM_BETAS, scenes.ADAM_EPS))
    for k in NAMES:
        gr = g_ref[k].reshape(m, -1)
        # spec tolerance on the gradient, plus what the 2D differences move it through the
        # chain, plus the float32 summation bound of the sum over views
        tol = G_RTOL * np.abs(gr) + 1.01 * prop[k].reshape(m, -1) + SUM_BOUND * sumb[k].reshape(m, -1) + 1e-30
        lr = float(np.float32(wl.adam_lr[k]))
        p0 = np.asarray(before[k], np.float32).reshape(m, -1)
        z = np.zeros_like(p0)
        p1r, m1r, v1r = orc.adam(p0, gr.astype(np.float32), z, z, lr, b1, b2, eps, 1)
        p1r, m1r, v1r = (x.reshape(m, -1).astype(np.float64) for x in (p1r, m1r, v1r))
        gm = np.asarray(m1[k], np.float64).reshape(m, -1)
        gv = np.asarray(v1[k], np.float64).reshape(m, -1)
        gp = np.asarray(after[k], np.float64).reshape(m, -1)
        ok_m = np.abs(gm - m1r) <= (1 - b1) * 1.0001 * tol + 2 * EPS32 * np.abs(m1r)
        ok_v = np.abs(gv - v1r) <= (1 - b2) * 1.0001 * (2 * np.abs(gr) * tol + tol ** 2) + 3 * EPS32 * np.abs(v1r)
        # the first step moves by lr sign(g); where the gradient is within its tolerance of 0 the
        # direction is not determined
        undecided = np.abs(gr) <= tol
        ok_p = np.abs(gp - p1r) <= EPS32 * np.maximum(np.abs(p0), np.abs(p1r)) + 1e-5 * lr + undecided * 2 * lr
        for nm, ok in (("m", ok_m), ("v", ok_v), ("param", ok_p)):
            bad = ~ok
            assert not bad.any(), (k, nm, int(bad.sum()), np.argwhere(bad)[:3])
    print(f"step: all {m} sampled Gaussians checked end to end; {n_amb_total} ambiguous of {n_px_total} rendered "
          f"px; {sign_amb_total} sign-ambiguous px; {n_allow_total} of {n_elem_total} 2D gradient elements within "
          f"an allowance only")


def test_fused_16_view_backward_with_adam_at_full_size(orc, stepped):
    """gs_project_bwd_views_adam over the 16 views of 1M Gaussians, the launch the step
    makes, fed seeded 2D gradients (every visible Gaussian of every view), from seeded
    Adam moments at step 3; 3000 sampled Gaussians against the sum over views of the
    oracle's chain, then the oracle's Adam."""
    wl, tr = stepped
    scene, cams = wl.scene, wl.cameras
    n, deg, nv = scene.n, scene.sh_degree, len(cams)
    rng = np.random.default_rng(5)
    g = pl.Gaussians.from_scene(scene)               # the parameters the step projected
    grad2ds = []
    rows_all = []
    for k in range(nv):
        rows = rng.standard_normal((n, 9)).astype(np.float32) * 1e-3
        rows_all.append(rows)
        gd = pl.Grad2D(n)
        gd.xy.copy_(torch.from_numpy(np.ascontiguousarray(rows[:, 0:2])))
        gd.conic_opacity.copy_(torch.from_numpy(np.ascontiguousarray(rows[:, 2:6])))
        rgb = np.zeros((n, 4), np.float32)
        rgb[:, :3] = rows[:, 6:9]
        gd.rgb.copy_(torch.from_numpy(rgb))
        grad2ds.append(gd)
    mom, vel = g.zeros_like(), g.zeros_like()
    for t in list(mom.tensors().values()) + list(vel.tensors().values()):
        t.copy_(torch.from_numpy((1e-4 * rng.random(tuple(t.shape))).astype(np.float32)))
    idx = np.sort(rng.choice(n, 3000, replace=False))
    m0, v0 = _natural(mom, idx, deg), _natural(vel, idx, deg)
    grads = g.zeros_like()
    acc = torch.zeros(n, device="cuda")
    cnt = torch.zeros(n, device="cuda", dtype=torch.int32)
    pl.project_bwd_views_adam(g, tr.views, tr.proj, tr.radii, grad2ds, mom, vel, tr.lrs, 3, grads, acc, cnt)
    torch.cuda.synchronize()
    want = {k: 0.0 for k in NAMES}
    sh_abs = 0.0
    acc_ref = np.zeros(len(idx))
    cnt_ref = np.zeros(len(idx), np.int64)
    for k, cam in enumerate(cams):
        r = rows_all[k][idx].astype(np.float64)
        o = orc.project_bwd(scene, cam, r, idx=idx, densify=True)
        for p in NAMES:
            want[p] = want[p] + np.asarray(o[p], np.float64).reshape(len(idx), -1)
        # an SH coefficient takes one term per view, Y_lm(dir) times its channel's colour
        # gradient, so the chain of |2D gradients| gives each term's magnitude: the float32
        # sum over views is checked against its summation bound where it cancels
        sh_abs = sh_abs + np.abs(np.asarray(orc.project_bwd(scene, cam, np.abs(r), idx=idx)["sh"],
                                            np.float64)).reshape(len(idx), -1)
        acc_ref += o["densify_accum"]
        cnt_ref += o["densify_count"]
    assert np.array_equal(cnt[torch.from_numpy(idx).cuda()].cpu().numpy(), cnt_ref)
    np.testing.assert_allclose(acc[torch.from_numpy(idx).cuda()].cpu().numpy(), acc_ref, rtol=1e-5, atol=1e-12)
    got_g = _natural(grads, idx, deg)
    for p in NAMES:
        check_grads(np.asarray(got_g[p]).reshape(len(idx), -1), want[p], f"fused16:{p}",
                    ref_abs=sh_abs if p == "sh" else None, max_bad_frac=0.01 if p == "sh" else 0.0)
    b1, b2, eps = (float(np.float32(x)) for x in (*scenes.ADAM_BETAS, scenes.ADAM_EPS))
    p1, mm, vv = _natural(g, idx, deg), _natural(mom, idx, deg), _natural(vel, idx, deg)
    before = _scene_natural(scene, idx)
    for p in NAMES:
        lr = float(np.float32(wl.adam_lr[p]))
        gr = np.asarray(got_g[p], np.float32).reshape(-1)    # Adam of the gradient the kernel summed
        pr, mr, vr = orc.adam(np.asarray(before[p], np.float32).reshape(-1), gr,
                              np.asarray(m0[p], np.float32).reshape(-1), np.asarray(v0[p], np.float32).reshape(-1),
                              lr, b1, b2, eps, 3)
        gm = np.asarray(mm[p], np.float64).reshape(-1)
        gv = np.asarray(vv[p], np.float64).reshape(-1)
        gp = np.asarray(p1[p], np.float64).reshape(-1)
        assert np.all(np.abs(gm - mr) <= 3 * EPS32 * (np.abs(mr) + 0.1 * np.abs(gr)) + 1e-20), p
        assert np.all(np.abs(gv - vr) <= 3 * EPS32 * (np.abs(vr) + 0.01 * gr.astype(np.float64) ** 2) + 1e-24), p
        upd = np.abs(pr.astype(np.float64) - np.asarray(before[p], np.float64).reshape(-1))
        bound = EPS32 * np.maximum(np.abs(pr), np.abs(gp)) + 1e-3 * upd + 1e-9
        assert np.all(np.abs(gp - pr) <= bound), (p, float(np.max(np.abs(gp - pr) - bound)))
