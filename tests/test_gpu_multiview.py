"""Parity of the multi-view backward through the projection (gs_project_bwd_views)
and of the fused Adam step (gs_project_bwd_views_adam) with the oracle: the sum
over views of the oracle's dual-number chain, then the oracle's Adam."""
import numpy as np
import pytest
import torch

from gaussian_splatting_differentiable_02_b200 import abi, scenes
from gaussian_splatting_differentiable_02_b200 import pipeline as pl

from _parity import check_grads

pytestmark = pytest.mark.gpu

NAMES = ("means", "quats", "log_scales", "opacity_logits", "sh")
LRS = {"means": 1.6e-4, "log_scales": 5e-3, "quats": 1e-3, "opacity_logits": 5e-2, "sh": 2.5e-3}


def _views(n_views, seed=0):
    rng = np.random.default_rng(seed)
    cams = []
    for k in range(n_views):
        eye = rng.standard_normal(3)
        eye = 4.0 * eye / np.linalg.norm(eye)
        R, t = scenes.look_at(eye)
        cams.append(scenes.camera(R, t, 128.0, 128.0, 64.0, 64.0, 128, 128))
    return cams


def _setup(orc, n_views=3, deg=2, seed=5):
    rng = np.random.default_rng(seed)
    scene = scenes.random_scene(rng, 800, deg, mean_box=1.0, log_scale=(-4.0, -2.0))
    cams = _views(n_views, seed)
    g = pl.Gaussians.from_scene(scene)
    proj = pl.Projected(scene.n)
    radii = torch.zeros((n_views, scene.n), dtype=torch.int32, device="cuda")
    views, g2s, g2_rows = [], [], []
    for k, cam in enumerate(cams):
        view = pl.View(scene.n, cam)
        pl.project(g, view, proj, radii[k])
        views.append(view)
        ref = orc.project(scene, cam)
        assert np.array_equal(radii[k].cpu().numpy(), ref["radius"])
        up = rng.standard_normal((128 * 128, 3))
        g2, _, _ = orc.render_bwd(ref, cam, up)
        rows = g2.astype(np.float32)
        g2_rows.append(rows)
        gd = pl.Grad2D(scene.n)
        gd.xy.copy_(torch.from_numpy(np.ascontiguousarray(rows[:, 0:2])))
        gd.conic_opacity.copy_(torch.from_numpy(np.ascontiguousarray(rows[:, 2:6])))
        rgb = np.zeros((scene.n, 4), np.float32)
        rgb[:, :3] = rows[:, 6:9]
        gd.rgb.copy_(torch.from_numpy(rgb))
        g2s.append(gd)
    torch.cuda.synchronize()
    want = {k: 0.0 for k in NAMES}
    acc = np.zeros(scene.n)
    cnt = np.zeros(scene.n, np.int64)
    for cam, rows in zip(cams, g2_rows):
        o = orc.project_bwd(scene, cam, rows.astype(np.float64), densify=True)
        for k in NAMES:
            want[k] = want[k] + o[k]
        acc += o["densify_accum"]
        cnt += o["densify_count"]
    return scene, cams, g, proj, radii, views, g2s, want, acc, cnt


def test_views_equal_sum_of_single_view_chains(orc):
    scene, cams, g, proj, radii, views, g2s, want, acc, cnt = _setup(orc)
    grads = g.zeros_like()
    da = torch.zeros(scene.n, device="cuda")
    dc = torch.zeros(scene.n, dtype=torch.int32, device="cuda")
    abi.gs_project_bwd_views(g.params(), [v.gcam for v in views], [proj.struct(radii[k]) for k in range(len(views))],
                             [x.struct() for x in g2s], grads.grads(), densify_accum=da.data_ptr(),
                             densify_count=dc.data_ptr(), stream=torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    got = grads.to_numpy()
    vis = np.nonzero(cnt > 0)[0]
    assert len(vis) > 500
    for k in NAMES:
        check_grads(got[k].reshape(scene.n, -1), np.asarray(want[k]).reshape(scene.n, -1), k, rows=vis)
    np.testing.assert_allclose(da.cpu().numpy(), acc, rtol=1e-5, atol=1e-9)
    assert np.array_equal(dc.cpu().numpy(), cnt)


@pytest.mark.parametrize("deg", [0, 3])
def test_fused_adam_matches_oracle_adam_of_summed_gradients(orc, deg):
    scene, cams, g, proj, radii, views, g2s, want, acc, cnt = _setup(orc, n_views=4, deg=deg, seed=9)
    rng = np.random.default_rng(3)
    m, v = g.zeros_like(), g.zeros_like()
    for t in list(m.tensors().values()) + list(v.tensors().values()):
        t.copy_(torch.from_numpy((0.01 * rng.random(tuple(t.shape))).astype(np.float32)))
    p0 = {k: getattr(g, k).cpu().numpy().copy() for k in NAMES}
    m0 = {k: getattr(m, k).cpu().numpy().copy() for k in NAMES}
    v0 = {k: getattr(v, k).cpu().numpy().copy() for k in NAMES}
    grads = g.zeros_like()
    step = 3
    b1, b2, eps = (float(np.float32(x)) for x in (0.9, 0.99, 1e-15))
    lrs = [float(np.float32(LRS[k])) for k in NAMES]
    abi.gs_project_bwd_views_adam(g.params(), [vw.gcam for vw in views],
                                  [proj.struct(radii[k]) for k in range(len(views))], [x.struct() for x in g2s],
                                  g.grads(), m.grads(), v.grads(), lrs, b1, b2, eps, step, grads=grads.grads(),
                                  stream=torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    # the summed gradient it applied
    got_g = grads.to_numpy()
    vis = np.nonzero(cnt > 0)[0]
    for k in NAMES:
        check_grads(got_g[k].reshape(scene.n, -1), np.asarray(want[k]).reshape(scene.n, -1), k, rows=vis)
    # Adam on the device layout: compare with the oracle's Adam of the reference gradient, rows where the
    # reference gradient is not a near-zero cancellation (there Adam's direction is not determined)
    eps32 = float(np.finfo(np.float32).eps)
    for gi, k in enumerate(NAMES):
        gref = np.zeros_like(p0[k])
        w = np.asarray(want[k])
        if k in ("means", "log_scales"):
            gref[:, :3] = w
        elif k == "sh":
            gref[:] = pl.sh_to_planes(w.astype(np.float32))
        else:
            gref[:] = w.reshape(gref.shape)
        p1, m1, v1 = orc.adam(p0[k], gref.astype(np.float32), m0[k], v0[k], lrs[gi], b1, b2, eps, step)
        gp, gm, gv = getattr(g, k).cpu().numpy(), getattr(m, k).cpu().numpy(), getattr(v, k).cpu().numpy()
        gerr = np.abs(getattr(grads, k).cpu().numpy() - gref)
        assert np.all(np.abs(gm - m1) <= 3 * eps32 * (np.abs(m1) + 0.1 * np.abs(gref)) + 0.1 * gerr + 1e-12), k
        assert np.all(np.abs(gv - v1) <= 3 * eps32 * (np.abs(v1) + 0.01 * gref ** 2) + 0.02 * gerr * np.abs(gref)
                      + 1e-12), k
        upd = np.abs(p1.astype(np.float64) - p0[k])
        bound = eps32 * np.maximum(np.abs(p1), np.abs(p0[k])) + 1e-3 * upd + 1e-9
        assert np.all(np.abs(gp - p1) <= bound), (k, float(np.max(np.abs(gp - p1) - bound)))


def test_bin_sort_async_matches_sync_and_reports_overflow(orc):
    wl = scenes.tiny()
    cam = wl.cameras[0]
    g = pl.Gaussians.from_scene(wl.scene)
    view = pl.View(wl.scene.n, cam)
    proj = pl.Projected(wl.scene.n)
    pl.project(g, view, proj)
    ref = orc.project(wl.scene, cam)
    keys, vals, ranges = orc.keys(ref, cam)
    K = len(keys)
    counter = torch.zeros(1, dtype=torch.int64, device="cuda")
    view._alloc(K + 100)
    pl.bin_sort_async(proj, view, counter)
    torch.cuda.synchronize()
    assert int(counter.item()) == K
    assert np.array_equal(view.keys[:K].cpu().numpy().view(np.uint64), keys)
    assert np.array_equal(view.vals[:K].cpu().numpy().view(np.uint32), vals)
    assert np.array_equal(view.ranges.cpu().numpy().view(np.uint32), ranges)
    # too small: K still reported, nothing emitted, every range empty
    view._alloc(64)
    view.keys.fill_(-7)
    pl.bin_sort_async(proj, view, counter)
    torch.cuda.synchronize()
    assert int(counter.item()) == K
    assert torch.all(view.ranges == 0)
    assert torch.all(view.keys == -7)


def test_trainer_fused_equals_unfused():
    """The fused multi-view step and the per-view step + gs_adam update the same
    parameters (both CUDA paths; a consistency check next to the oracle parity)."""
    rng = np.random.default_rng(12)
    scene = scenes.random_scene(rng, 600, 1, mean_box=1.0, log_scale=(-3.5, -2.0))
    cams = _views(3, 4)
    targets = [torch.from_numpy(rng.random((128, 128, 3)).astype(np.float32)).cuda() for _ in cams]
    out = []
    for fused in (True, False):
        g = pl.Gaussians.from_scene(scene)
        tr = pl.Trainer(g, [pl.View(scene.n, c) for c in cams], targets, dict(LRS), densify=True, fused=fused)
        tr.step()
        tr.step()
        torch.cuda.synchronize()
        out.append((g.to_numpy(), tr.densify_accum.cpu().numpy(), tr.densify_count.cpu().numpy(), tr.loss.item()))
    (a, da, ca, la), (b, db, cb, lb) = out
    assert np.array_equal(ca, cb)
    np.testing.assert_allclose(da, db, rtol=1e-5, atol=1e-9)
    assert abs(la - lb) <= 1e-9 * max(1.0, abs(la))
    for k in NAMES:
        # identical up to the rounding of the per-view float32 accumulation; Adam's first
        # steps move by about lr * sign(g), so an element whose gradient is a near-zero
        # cancellation may move the other way (at most 2 lr per step)
        d = np.abs(a[k] - b[k])
        close = d <= 1e-6 + 1e-6 * np.abs(a[k])
        assert close.mean() >= 0.999, (k, float(close.mean()))
        assert d.max() <= 4 * LRS[k] + 1e-6, (k, float(d.max()))


def test_sparse_adam_skips_gaussians_seen_in_no_view():
    """sparse_adam = 1: Gaussians visible in no view keep parameters and moments bit for
    bit; every other Gaussian gets exactly the dense update (same inputs, same arithmetic)."""
    rng = np.random.default_rng(41)
    scene = scenes.random_scene(rng, 700, 1, mean_box=1.0, log_scale=(-4.0, -2.0))
    scene.means[:120] += 40.0   # far outside every view
    cams = _views(3, 6)
    views = [pl.View(scene.n, c) for c in cams]
    g = pl.Gaussians.from_scene(scene)
    proj = pl.Projected(scene.n)
    radii = torch.zeros((len(cams), scene.n), dtype=torch.int32, device="cuda")
    g2s = []
    for k, vw in enumerate(views):
        pl.project(g, vw, proj, radii[k])
        pl.bin_sort(proj, vw, radii[k])
        pl.raster_fwd(proj, vw, radius=radii[k])
        vw.dL_dimage.copy_(torch.from_numpy(rng.standard_normal(tuple(vw.dL_dimage.shape)).astype(np.float32)))
        gd = pl.Grad2D(scene.n)
        pl.raster_bwd(proj, vw, gd, radius=radii[k])
        g2s.append(gd)
    torch.cuda.synchronize()
    vis = (radii.cpu().numpy() > 0).any(axis=0)
    assert not vis[:120].any() and vis.sum() > 400
    m0 = g.zeros_like()
    v0 = g.zeros_like()
    for t in list(m0.tensors().values()) + list(v0.tensors().values()):
        t.copy_(torch.from_numpy((0.01 * rng.random(tuple(t.shape))).astype(np.float32)))
    out = []
    for sparse in (False, True):
        gg = pl.Gaussians.from_scene(scene)
        m, v = gg.zeros_like(), gg.zeros_like()
        for a, b in zip(list(m.tensors().values()) + list(v.tensors().values()),
                        list(m0.tensors().values()) + list(v0.tensors().values())):
            a.copy_(b)
        pl.project_bwd_views_adam(gg, views, proj, radii, g2s, m, v, LRS, 2, sparse=sparse)
        torch.cuda.synchronize()
        out.append([{k: getattr(x, k).cpu().numpy() for k in NAMES} for x in (gg, m, v)])
    g_init = {k: getattr(g, k).cpu().numpy() for k in NAMES}
    init = [g_init, {k: getattr(m0, k).cpu().numpy() for k in NAMES}, {k: getattr(v0, k).cpu().numpy() for k in NAMES}]
    for dense, sparse, before in zip(out[0], out[1], init):
        for k in NAMES:
            d, s, b = dense[k], sparse[k], before[k]
            if k == "sh":   # [P][n][4]
                d, s, b = (np.moveaxis(x, 1, 0) for x in (d, s, b))
            assert np.array_equal(s[vis], d[vis]), k
            assert np.array_equal(s[~vis], b[~vis]), k
    # the dense step did move the unseen Gaussians' moments (they decay)
    assert not np.array_equal(out[0][1]["means"][~vis], init[1]["means"][~vis])


def test_trainer_stream_and_sort_configurations_agree():
    """Views on one stream with a sort per view, on two streams, and on three streams
    after batched depth sorts of all views at once, of two view groups and of one view
    per group: the first step (identical inputs) gives the same loss, counts and
    instance numbers; later steps agree up to the order of the atomic adds."""
    rng = np.random.default_rng(13)
    scene = scenes.random_scene(rng, 600, 1, mean_box=1.0, log_scale=(-3.5, -2.0))
    cams = _views(5, 8)
    targets = [torch.from_numpy(rng.random((128, 128, 3)).astype(np.float32)).cuda() for _ in cams]
    out = []
    for streams, batched, groups in ((1, False, 1), (2, False, 1), (3, True, 1), (3, True, 2), (2, True, 5)):
        g = pl.Gaussians.from_scene(scene)
        tr = pl.Trainer(g, [pl.View(scene.n, c) for c in cams], targets, dict(LRS), densify=True, streams=streams,
                        batched_sort=batched, groups=groups)
        tr.step()
        torch.cuda.synchronize()
        first = (tr.loss.item(), tr.densify_count.cpu().numpy(), tr.kcount.cpu().numpy(),
                 [vw.keys[:int(K)].cpu().numpy() for vw, K in zip(tr.views, tr.kcount.cpu().tolist())])
        tr.step()
        tr.step()
        torch.cuda.synchronize()
        out.append((tr.gauss.to_numpy(), first))
    (a, (la, ca, ka, keys_a)) = out[0]
    for b, (lb, cb, kb, keys_b) in out[1:]:
        assert np.array_equal(ca, cb) and np.array_equal(ka, kb)
        assert all(np.array_equal(x, y) for x, y in zip(keys_a, keys_b))
        assert abs(la - lb) <= 1e-9 * abs(la)
        for k in NAMES:
            close = np.abs(a[k] - b[k]) <= 1e-6 + 1e-5 * np.abs(a[k])
            assert close.mean() >= 0.999, (k, float(close.mean()))


def test_batched_depth_order_matches_the_per_view_sort(orc):
    """gs_depth_order_views + gs_bin_sort_ordered_async give, for every view, the keys,
    values and ranges of gs_bin_sort (bit for bit) and of the oracle."""
    rng = np.random.default_rng(14)
    scene = scenes.random_scene(rng, 3000, 1, mean_box=1.0, log_scale=(-4.0, -2.0))
    scene.means[:100] += 30.0   # some Gaussians culled in every view
    cams = _views(6, 9)
    g = pl.Gaussians.from_scene(scene)
    projs = [pl.Projected(scene.n) for _ in cams]
    views = [pl.View(scene.n, c, capacity=40 * scene.n) for c in cams]
    radii = torch.zeros((len(cams), scene.n), dtype=torch.int32, device="cuda")
    for k, vw in enumerate(views):
        pl.project(g, vw, projs[k], radii[k])
    d = pl.DepthOrder(scene.n, len(cams))
    pl.depth_order_views(projs, radii, d)
    counts = torch.zeros((len(cams),), dtype=torch.int64, device="cuda")
    for k, vw in enumerate(views):
        pl.bin_sort_ordered_async(projs[k], vw, d.order[k], counts[k:k + 1], radii[k])
    torch.cuda.synchronize()
    for k, (vw, cam) in enumerate(zip(views, cams)):
        K = int(counts[k].item())
        assert K <= vw.capacity
        ref = orc.project(scene, cam)
        keys, vals, ranges = orc.keys(ref, cam)
        assert K == len(keys)
        assert np.array_equal(vw.keys[:K].cpu().numpy().view(np.uint64), keys)
        assert np.array_equal(vw.vals[:K].cpu().numpy().view(np.uint32), vals)
        assert np.array_equal(vw.ranges.cpu().numpy().view(np.uint32), ranges)
        # the depth order itself: visible Gaussians by (depth bits, index), culled ones after
        order = d.order[k].cpu().numpy().view(np.uint32)
        r = radii[k].cpu().numpy()
        z = projs[k].depth.cpu().numpy().view(np.uint32).astype(np.uint64)
        keyz = np.where(r > 0, z, 0xFFFFFFFF)
        assert np.array_equal(order, np.lexsort((np.arange(scene.n), keyz)).astype(np.uint32))


@pytest.mark.parametrize("n_views,sparse", [(1, 0), (2, 1), (2, 0)])
def test_one_kernel_step_equals_two_launches(orc, n_views, sparse):
    """With one or two views and no gradient buffer the chain and the Adam step run in one
    kernel; with a buffer, as two launches (the chain writes the gradient, one Adam launch
    reads it).  Same inputs, same float32 gradient, same Adam arithmetic: parameters,
    moments and densification statistics identical bit for bit, and the buffer holds the
    gradient the multi-view chain gives (written over, not added to)."""
    scene, cams, g0, proj, radii, views, g2s, want, acc, cnt = _setup(orc, n_views=n_views, deg=3, seed=21)
    rng = np.random.default_rng(4)
    init = {k: (0.01 * rng.random(tuple(getattr(g0, k).shape))).astype(np.float32) for k in NAMES}
    lrs = [float(np.float32(LRS[k])) for k in NAMES]
    out = []
    for with_buffer in (False, True):
        g = g0.zeros_like()
        for k in NAMES:
            getattr(g, k).copy_(getattr(g0, k))
        m, v = g.zeros_like(), g.zeros_like()
        for k in NAMES:
            getattr(m, k).copy_(torch.from_numpy(init[k]))
            getattr(v, k).copy_(torch.from_numpy(init[k] * 0.5))
        grads = g.zeros_like()
        for t in grads.tensors().values():
            t.fill_(7.0)  # written over, so the fill must not survive
        da = torch.zeros(scene.n, device="cuda")
        dc = torch.zeros(scene.n, dtype=torch.int32, device="cuda")
        abi.gs_project_bwd_views_adam(g.params(), [vw.gcam for vw in views],
                                      [proj.struct(radii[k]) for k in range(n_views)], [x.struct() for x in g2s],
                                      g.grads(), m.grads(), v.grads(), lrs, 0.9, 0.99, 1e-15, 2,
                                      grads=grads.grads() if with_buffer else None, densify_accum=da.data_ptr(),
                                      densify_count=dc.data_ptr(), sparse_adam=sparse,
                                      stream=torch.cuda.current_stream().cuda_stream)
        torch.cuda.synchronize()
        out.append((g, m, v, grads, da.cpu().numpy(), dc.cpu().numpy()))
    (ga, ma, va, _, daa, dca), (gb, mb, vb, grads, dab, dcb) = out
    for k in NAMES:
        for x, y in ((ga, gb), (ma, mb), (va, vb)):
            assert torch.equal(getattr(x, k), getattr(y, k)), k
    assert np.array_equal(daa, dab) and np.array_equal(dca, dcb)
    # the buffer: the summed gradient, and the visible-view count in the means' w lane
    got = grads.to_numpy()
    vis = np.nonzero(cnt > 0)[0]
    for k in NAMES:
        check_grads(got[k].reshape(scene.n, -1), np.asarray(want[k]).reshape(scene.n, -1), k, rows=vis)
    assert np.array_equal(grads.means[:, 3].cpu().numpy(), cnt.astype(np.float32))


@pytest.mark.parametrize("packed", [False, True])
def test_graph_step_matches_eager(packed):
    """Trainer(graph=True) replays the views' part of the step from a CUDA graph: the same
    kernels on the same buffers as the eager step, so the same instance counts, the same
    first loss up to the order of its double-precision atomic sums, and parameters equal
    up to the order the gradient atomics happened to take.  The step is captured again
    after the instance buffers grow (the first step starts with small ones) and after
    densification reallocates everything."""
    rng = np.random.default_rng(17)
    scene = scenes.random_scene(rng, 600, 1, mean_box=1.0, log_scale=(-3.5, -2.0))
    cams = _views(3, 6)
    targets = [torch.from_numpy(rng.random((128, 128, 3)).astype(np.float32)).cuda() for _ in cams]
    out = []
    for graph in (False, True):
        g = pl.Gaussians.from_scene(scene)
        views = [pl.View(scene.n, c) for c in cams]
        for vw in views:
            vw._alloc(64)  # too small: the first step grows them
        tr = pl.Trainer(g, views, targets, dict(LRS), densify=True, packed=packed, graph=graph)
        losses, counts = [], []
        for it in range(4):
            tr.step()
            torch.cuda.synchronize()
            losses.append(tr.loss.item())
            counts.append(tr.kcount.cpu().numpy().copy())
            if it == 1:
                tr.densify_and_prune(max_screen_size=0.0)  # no screen-size pruning: most Gaussians stay
        out.append((tr.gauss.to_numpy(), losses, counts, tr.gauss.n))
    (a, la, ca, na), (b, lb, cb, nb) = out
    assert na == nb and na > 300
    assert abs(la[0] - lb[0]) <= 1e-9 * max(1.0, abs(la[0]))
    assert all(np.array_equal(x, y) for x, y in zip(ca[:2], cb[:2]))
    np.testing.assert_allclose(la, lb, rtol=1e-5)
    for k in NAMES:
        d = np.abs(a[k] - b[k])
        close = d <= 1e-6 + 1e-6 * np.abs(a[k])
        assert close.mean() >= 0.999, (k, float(close.mean()))
        assert d.max() <= 8 * LRS[k] + 1e-6, (k, float(d.max()))


@pytest.mark.parametrize("n_views", [1, 5, 16])
def test_views_binning_matches_per_view_binning(orc, n_views):
    """gs_bin_sort_ordered_views_async gives every view the keys, values, ranges and
    instance count of gs_bin_sort_ordered_async, bit for bit, with views of different
    capacities (one too small: its count is reported, nothing is emitted and its ranges
    are empty); one view against the oracle.  The tile orders (one launch for the group)
    are valid: a permutation of the tiles by non-increasing length bucket (the order
    inside a bucket is not specified)."""
    rng = np.random.default_rng(33)
    scene = scenes.random_scene(rng, 2500, 1, mean_box=1.0, log_scale=(-4.0, -2.0))
    scene.means[:50] += 30.0   # some Gaussians culled in every view
    cams = _views(n_views, 12)
    g = pl.Gaussians.from_scene(scene)
    projs = [pl.Projected(scene.n) for _ in cams]
    radii = torch.zeros((n_views, scene.n), dtype=torch.int32, device="cuda")
    caps = [40 * scene.n + 1000 * k for k in range(n_views)]  # view 1 gets 64 slots below: too small
    out = []
    for batched in (False, True):
        views = [pl.View(scene.n, c, capacity=caps[k]) for k, c in enumerate(cams)]
        if n_views > 1:
            views[1]._alloc(64)
        for vw in views:
            vw.keys.fill_(-3)
        for k, vw in enumerate(views):
            pl.project(g, vw, projs[k], radii[k])
        d = pl.DepthOrder(scene.n, n_views)
        pl.depth_order_views(projs, radii, d)
        counts = torch.full((n_views,), -1, dtype=torch.int64, device="cuda")
        if batched:
            pl.bin_sort_ordered_views_async(projs, views, d, counts, radii)
        else:
            for k, vw in enumerate(views):
                pl.bin_sort_ordered_async(projs[k], vw, d.order[k], counts[k:k + 1], radii[k])
        torch.cuda.synchronize()
        out.append(([vw.keys.cpu().numpy() for vw in views], [vw.vals.cpu().numpy() for vw in views],
                    [vw.ranges.cpu().numpy() for vw in views], [vw.order.cpu().numpy() for vw in views],
                    counts.cpu().numpy(), [vw.capacity for vw in views]))
    (ka, va, ra, oa, ca, cap), (kb, vb, rb, ob, cb, _) = out
    assert np.array_equal(ca, cb)
    for k in range(n_views):
        K = int(ca[k])
        assert np.array_equal(ra[k], rb[k])
        r = rb[k].view(np.uint32).reshape(-1, 2)
        bucket = 255 - np.minimum(255, np.floor(np.sqrt((r[:, 1] - r[:, 0]).astype(np.float32))).astype(np.int64))
        for o in (oa[k], ob[k]):
            o = o.view(np.uint32).astype(np.int64)
            assert np.array_equal(np.sort(o), np.arange(len(r)))
            assert np.all(np.diff(bucket[o]) >= 0)
        if K <= cap[k]:
            assert np.array_equal(ka[k][:K], kb[k][:K]) and np.array_equal(va[k][:K], vb[k][:K])
        else:
            assert not ra[k].any() and np.all(kb[k] == -3)
    ref = orc.project(scene, cams[0])
    keys, vals, ranges = orc.keys(ref, cams[0])
    assert int(cb[0]) == len(keys)
    assert np.array_equal(kb[0][:len(keys)].view(np.uint64), keys)
    assert np.array_equal(vb[0][:len(keys)].view(np.uint32), vals)
    assert np.array_equal(rb[0].view(np.uint32), ranges)
