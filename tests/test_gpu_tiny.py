"""Parity of the CUDA path with the oracle on the tiny workload (1,000 Gaussians,
128x128, SH degree 0, upstream dL/dimage ~ N(0,1)), every stage and every
output element, plus edge cases."""
import math

import numpy as np
import pytest
import torch

from gaussian_splatting_differentiable_02_b200 import abi, scenes
from gaussian_splatting_differentiable_02_b200 import pipeline as pl

from _parity import (BAND_ALPHA, BAND_T, G_ATOL, G_RTOL, CudaRun, chain_abs_bound, check_grads, check_images,
                     check_projection, grad_mismatch, ulp_diff)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tiny(orc):
    wl = scenes.tiny()
    cam = wl.cameras[0]
    run = CudaRun(wl.scene, cam)
    ref = orc.project(wl.scene, cam)
    return wl, cam, run, ref


def test_project(tiny):
    wl, cam, run, ref = tiny
    check_projection(run.projection(), ref)
    assert (ref["radius"] > 0).sum() > 900


def test_keys_sorted_order_and_ranges_bit_exact(orc, tiny):
    wl, cam, run, ref = tiny
    keys, vals, ranges = orc.keys(ref, cam)
    gk, gv, gr = run.sorted_instances()
    assert run.K == len(keys) > 0
    assert np.array_equal(gk, keys)
    assert np.array_equal(gv, vals)
    assert np.array_equal(gr, ranges)


def test_forward_image(orc, tiny):
    wl, cam, run, ref = tiny
    img, T, nc, amb = orc.render(ref, cam, band_alpha=BAND_ALPHA, band_T=BAND_T)
    gi, gT, gn = run.images()
    err, namb = check_images(gi, gT, gn, img, T, nc, amb)
    assert nc.max() > 3


def test_forward_is_deterministic(tiny):
    wl, cam, run, ref = tiny
    a = run.view.image.clone()
    pl.raster_fwd(run.proj, run.view)
    torch.cuda.synchronize()
    assert torch.equal(a, run.view.image)


def test_backward_grad2d(orc, tiny):
    wl, cam, run, ref = tiny
    g = wl.upstream[0]
    g2_gpu = run.backward(g)
    g2, g2a, touched = orc.render_bwd(ref, cam, g.reshape(-1, 3).astype(np.float64), band_alpha=BAND_ALPHA,
                                      band_T=BAND_T)
    rows = np.nonzero(touched == 0)[0]
    assert len(rows) > 900
    for q, name in enumerate(["du", "dv", "dA", "dB", "dC", "do", "dr", "dg", "db"]):
        check_grads(g2_gpu[:, q], g2[:, q], name, rows=rows, ref_abs=g2a[:, q], max_bad_frac=0.002)


def test_project_backward_from_reference_grad2d(orc, tiny):
    """GPU project_bwd fed the oracle's 2D gradients (rounded to float32) against the
    oracle's dual-number chain of the same float32 gradients."""
    wl, cam, run, ref = tiny
    g = wl.upstream[0]
    g2, _, _ = orc.render_bwd(ref, cam, g.reshape(-1, 3).astype(np.float64))
    g2f = g2.astype(np.float32)
    gpu = run.project_bwd(g2f, densify=True)
    want = orc.project_bwd(wl.scene, cam, g2f.astype(np.float64), densify=True)
    vis = np.nonzero(ref["radius"] > 0)[0]
    for k in ("means", "quats", "log_scales", "opacity_logits", "sh"):
        check_grads(gpu[k].reshape(wl.scene.n, -1), want[k].reshape(wl.scene.n, -1), k, rows=vis)
    np.testing.assert_allclose(gpu["densify_accum"], want["densify_accum"], rtol=1e-6, atol=1e-12)
    assert np.array_equal(gpu["densify_count"], want["densify_count"])


def test_end_to_end_parameter_gradients(orc, tiny):
    """Whole backward: CUDA raster_bwd -> CUDA project_bwd against oracle render_bwd -> oracle
    project_bwd, element by element.  The two sides start from different 2D gradients (each
    side's own, which agree element by element within their tolerance), so each parameter
    gradient may differ by what that 2D difference moves it through the chain, |J| |d2D|,
    plus the chain's own tolerance; nothing passes outside that bound."""
    wl, cam, run, ref = tiny
    g = wl.upstream[0]
    g2_gpu = run.backward(g)
    gpu = run.project_bwd(g2_gpu)
    g2, g2a, touched = orc.render_bwd(ref, cam, g.reshape(-1, 3).astype(np.float64), band_alpha=BAND_ALPHA,
                                      band_T=BAND_T)
    want = orc.project_bwd(wl.scene, cam, g2)
    prop = chain_abs_bound(orc, wl.scene, cam, g2_gpu.astype(np.float64) - g2)
    rows = np.nonzero((touched == 0) & (ref["radius"] > 0))[0]
    for k in ("means", "quats", "log_scales", "opacity_logits", "sh"):
        a = gpu[k].reshape(wl.scene.n, -1)[rows].astype(np.float64)
        b = want[k].reshape(wl.scene.n, -1)[rows]
        p = prop[k][rows]
        # the chain of fp32-accumulated 2D sums: report the norm-wise error too
        rel = np.linalg.norm(a - b) / np.linalg.norm(b)
        assert rel < 1e-5, (k, rel)
        d = np.abs(a - b)
        within_tol = d <= G_ATOL + G_RTOL * np.abs(b)
        bound = G_ATOL + G_RTOL * (np.abs(b) + p) + 1.01 * p
        assert np.all(d <= bound), (k, float(np.max(d - bound)))
        print(f"  {k}: {int((~within_tol).sum())} of {d.size} elements outside 1e-6 + 1e-4|ref|, all within the "
              f"propagated 2D difference")


def test_adam_matches_oracle(orc):
    """The ABI takes float32 hyper-parameters, so the oracle gets the same float32
    values.  Tolerance: a few float32 roundings of the terms of each update."""
    rng = np.random.default_rng(1)
    n = 4099                      # a ragged tail after the float4 body
    p = rng.standard_normal(n).astype(np.float32)
    m = (0.1 * rng.standard_normal(n)).astype(np.float32)
    v = (0.01 * rng.random(n)).astype(np.float32)
    gr = rng.standard_normal(n).astype(np.float32)
    lr, b1, b2, eps = (float(np.float32(x)) for x in (5e-2, 0.9, 0.99, 1e-15))
    tp, tg, tm, tv = (torch.from_numpy(x.copy()).cuda() for x in (p, gr, m, v))
    eps32 = float(np.finfo(np.float32).eps)
    for step in (1, 2, 7):
        # both sides start the step from the same float32 state
        for t, x in ((tp, p), (tm, m), (tv, v)):
            t.copy_(torch.from_numpy(x))
        abi.gs_adam(tp.data_ptr(), tg.data_ptr(), tm.data_ptr(), tv.data_ptr(), n, lr, b1, b2, eps, step,
                    torch.cuda.current_stream().cuda_stream)
        m_scale = np.abs(b1 * m.astype(np.float64)) + np.abs((1 - b1) * gr.astype(np.float64))
        v_scale = np.abs(b2 * v.astype(np.float64)) + np.abs((1 - b2) * gr.astype(np.float64) ** 2)
        p_old = p
        p, m, v = orc.adam(p, gr, m, v, lr, b1, b2, eps, step)
        torch.cuda.synchronize()
        assert np.all(np.abs(tm.cpu().numpy() - m) <= 3 * eps32 * m_scale)
        assert np.all(np.abs(tv.cpu().numpy() - v) <= 3 * eps32 * v_scale)
        update = np.abs(p.astype(np.float64) - p_old)
        # p_new = p_old - update rounds at the scale of the larger of the two; the
        # update m / sqrt(v) inherits the moments' relative errors plus a few
        # roundings of its own (sqrt, divide, scale)
        rel_upd = 3 * eps32 * m_scale / np.maximum(np.abs(m), 1e-30) + 1.5 * eps32 * v_scale / v + 8 * eps32
        scale = np.maximum(np.abs(p), np.abs(p_old))
        assert np.all(np.abs(tp.cpu().numpy() - p) <= eps32 * scale + rel_upd * update + 1e-12)


def test_l1_matches_oracle(orc):
    rng = np.random.default_rng(2)
    img = rng.random((37, 53, 3)).astype(np.float32)
    tgt = rng.random((37, 53, 3)).astype(np.float32)
    tgt[0, :5] = img[0, :5]       # sign(0) = 0
    ti, tt = torch.from_numpy(img).cuda(), torch.from_numpy(tgt).cuda()
    tg = torch.zeros_like(ti)
    loss = torch.zeros(1, dtype=torch.float64, device="cuda")
    abi.gs_l1_loss_grad(ti.data_ptr(), tt.data_ptr(), img.size, tg.data_ptr(), loss.data_ptr(),
                        torch.cuda.current_stream().cuda_stream)
    want_loss, want_g = orc.l1(img, tgt)
    assert np.array_equal(tg.cpu().numpy(), want_g)
    assert abs(loss.item() - want_loss) <= 1e-12


# ------------------------------------------------------------------ edge cases

def _run_and_compare(orc, scene, cam, bg=(0.0, 0.0, 0.0), max_amb_frac=1e-3):
    run = CudaRun(scene, cam, bg=bg)
    ref = orc.project(scene, cam)
    check_projection(run.projection(), ref)
    keys, vals, ranges = orc.keys(ref, cam)
    gk, gv, gr = run.sorted_instances()
    assert run.K == len(keys)
    assert np.array_equal(gk, keys) and np.array_equal(gv, vals) and np.array_equal(gr, ranges)
    img, T, nc, amb = orc.render(ref, cam, bg=bg, band_alpha=BAND_ALPHA, band_T=BAND_T)
    check_images(*run.images(), img, T, nc, amb, max_amb_frac=max_amb_frac)
    return run, ref


def test_empty_scene(orc):
    scene = scenes.random_scene(np.random.default_rng(0), 0, 0)
    cam = scenes.tiny().cameras[0]
    run = CudaRun(scene, cam, bg=(0.1, 0.2, 0.3))
    assert run.K == 0
    gi, gT, gn = run.images()
    assert np.all(gi == np.float32([0.1, 0.2, 0.3])) and np.all(gT == 1.0) and np.all(gn == 0)


def test_everything_behind_the_camera(orc):
    scene = scenes.random_scene(np.random.default_rng(1), 500, 0)
    scene.means[:, 2] -= 10.0          # camera at z = -4 looking +z
    cam = scenes.tiny().cameras[0]
    run, ref = _run_and_compare(orc, scene, cam, bg=(0.5, 0.5, 0.5))
    assert run.K == 0 and np.all(run.projection()["radius"] == 0)


def test_non_finite_parameters_are_culled(orc):
    rng = np.random.default_rng(2)
    scene = scenes.random_scene(rng, 300, 1)
    scene.means[0, 0] = np.nan
    scene.quats[1] = 0.0
    scene.log_scales[2, 1] = np.inf
    scene.opacity_logits[3] = np.nan
    scene.sh[4, 2, 1] = np.inf
    cam = scenes.tiny().cameras[0]
    run, ref = _run_and_compare(orc, scene, cam)
    assert np.all(run.projection()["radius"][:5] == 0)
    assert np.isfinite(run.images()[0]).all()


def test_ragged_image_and_multiple_sh_degrees(orc):
    rng = np.random.default_rng(3)
    for deg in (1, 2, 3):
        scene = scenes.random_scene(rng, 700, deg, log_scale=(-3.5, -1.5))
        R, t = scenes.look_at((0.3, -0.2, -4.0))
        cam = scenes.camera(R, t, 90.0, 90.0, 50.0, 18.5, 100, 37)     # 7 x 3 tiles, both edges ragged
        _run_and_compare(orc, scene, cam, bg=(0.0, 0.3, 0.7))


def test_capacity_overflow_reports_the_count(orc):
    wl = scenes.tiny()
    cam = wl.cameras[0]
    g = pl.Gaussians.from_scene(wl.scene)
    view = pl.View(wl.scene.n, cam, capacity=16)
    view._alloc(16)
    proj = pl.Projected(wl.scene.n)
    pl.project(g, view, proj)
    st, K = abi.gs_bin_sort(proj.struct(), view.n, view.gcam, view.workspace.data_ptr(), view.workspace.numel(),
                            view.keys.data_ptr(), view.vals.data_ptr(), view.capacity, view.ranges.data_ptr(),
                            torch.cuda.current_stream().cuda_stream, check=False)
    assert st == abi.GS_ERR_CAPACITY
    ref = orc.project(wl.scene, cam)
    assert K == int(ref["tiles_touched"].astype(np.int64).sum())
    assert pl.bin_sort(proj, view) == K       # the binding grows the buffers and retries


def test_opaque_stack_terminates_early(orc):
    """Many nearly opaque Gaussians on one spot: every pixel stops long before the list ends."""
    n = 600
    rng = np.random.default_rng(4)
    means = np.zeros((n, 3), np.float32)
    means[:, :2] = 0.02 * rng.standard_normal((n, 2))
    means[:, 2] = np.linspace(-1.0, 1.0, n)
    scene = scenes.Scene(means, np.tile(np.float32([1, 0, 0, 0]), (n, 1)),
                         np.full((n, 3), -1.0, np.float32), np.full(n, 4.0, np.float32),
                         rng.uniform(0, 1, (n, 1, 3)).astype(np.float32), 0)
    cam = scenes.tiny().cameras[0]
    # a stack of near-opaque splats puts many pixels' stopping decision near the
    # 1e-4 threshold: those pixels are counted and excluded, the rest compared
    run, ref = _run_and_compare(orc, scene, cam, max_amb_frac=0.01)
    gi, gT, gn = run.images()
    centre = 64 * 128 + 64
    assert 0 < gn[centre] < 10 and gT[centre] >= 1e-4


def test_needle_and_indefinite_conics(orc):
    """Conics written straight into the projected features (the rectangles and the
    sort stay those of the projection): needles with eigenvalue ratios up to 1e6 take
    the factored float32 evaluation, and conics that are indefinite in float32 (which
    the projection never writes) blend only where sigma >= 0, as the oracle's direct
    evaluation does."""
    wl = scenes.tiny()
    cam = wl.cameras[0]
    run = CudaRun(wl.scene, cam)
    p = run.projection()
    vis = np.argsort(-p["radius"])[:12]   # the largest footprints
    assert np.all(p["radius"][vis] > 4)
    con = run.proj.conic_opacity.cpu().numpy()
    rng = np.random.default_rng(5)
    for k, i in enumerate(vis[:12]):
        A = np.float32(rng.uniform(0.05, 0.5))
        ang = rng.uniform(0, np.pi)
        if k < 8:   # needle: eigenvalues A and A / kappa, rotated
            kappa = 10.0 ** rng.uniform(2, 6)
            l1, l2 = A, A / kappa
        else:       # indefinite
            l1, l2 = A, -A / 50
        c, s = np.cos(ang), np.sin(ang)
        con[i, 0] = l1 * c * c + l2 * s * s
        con[i, 1] = (l1 - l2) * c * s
        con[i, 2] = l1 * s * s + l2 * c * c
        con[i, 3] = 0.9
    run.proj.conic_opacity.copy_(torch.from_numpy(con))
    pl.raster_fwd(run.proj, run.view, run.bg)
    torch.cuda.synchronize()
    # the oracle composites exactly the features the kernels see
    ref = {k: np.asarray(v, np.float64) if v.dtype.kind == "f" else v for k, v in run.projection().items()}
    img, T, nc, amb = orc.render(ref, cam, band_alpha=BAND_ALPHA, band_T=BAND_T)
    gi, gT, gn = run.images()
    # an indefinite form is zero along two lines through the mean, where sigma changes
    # sign: the pixels near them are ambiguous by construction (excluded, counted)
    check_images(gi, gT, gn, img, T, nc, amb, max_amb_frac=0.08)
    # and the backward agrees on the same features
    up = wl.upstream[0]
    g2_gpu = run.backward(up)
    g2, g2a, touched = orc.render_bwd(ref, cam, up.reshape(-1, 3).astype(np.float64), band_alpha=BAND_ALPHA,
                                      band_T=BAND_T)
    rows = np.nonzero(touched == 0)[0]
    for q, name in enumerate(["du", "dv", "dA", "dB", "dC", "do", "dr", "dg", "db"]):
        check_grads(g2_gpu[:, q], g2[:, q], name, rows=rows, ref_abs=g2a[:, q], max_bad_frac=0.002)


@pytest.mark.parametrize("bg", [(0.2, 0.5, 0.8), (0.0, 0.0, 0.0)])
def test_backward_grad2d_with_a_background(orc, bg):
    """The reverse pass with a coloured background (its term of dL/dalpha, -T_final
    bg . g / (1 - alpha), formed per pixel) and with a black one (where the kernel
    leaves that term out), against the oracle's reverse pass with the same background."""
    wl = scenes.tiny()
    cam = wl.cameras[0]
    run = CudaRun(wl.scene, cam, bg=bg)
    ref = orc.project(wl.scene, cam)
    g = wl.upstream[0]
    g2_gpu = run.backward(g)
    g2, g2a, touched = orc.render_bwd(ref, cam, g.reshape(-1, 3).astype(np.float64), bg=bg, band_alpha=BAND_ALPHA,
                                      band_T=BAND_T)
    rows = np.nonzero(touched == 0)[0]
    assert len(rows) > 900
    for q, name in enumerate(["du", "dv", "dA", "dB", "dC", "do", "dr", "dg", "db"]):
        check_grads(g2_gpu[:, q], g2[:, q], name, rows=rows, ref_abs=g2a[:, q], max_bad_frac=0.002)


@pytest.mark.parametrize("size", [(100, 37), (1920, 1080)])   # the narrow-tile layout with ragged edges; the wide one
def test_forward_with_l1_equals_forward_then_l1(orc, size):
    """gs_raster_fwd_l1 (the L1 term in the forward kernel's epilogue) against
    gs_raster_fwd followed by gs_l1_loss_grad: image, final_T, n_contrib and
    dL/dimage bit-exact, the loss equal up to the order of its double sums, and
    both against the oracle's L1 of the rendered image."""
    W, H = size
    rng = np.random.default_rng(11)
    scene = scenes.random_scene(rng, 1500, 1, log_scale=(-3.5, -1.5))
    R, t = scenes.look_at((0.3, -0.2, -4.0))
    f = 0.9 * W
    cam = scenes.camera(R, t, f, f, 0.5 * W - 0.3, 0.5 * H + 0.2, W, H)
    bg = (0.1, 0.3, 0.6)
    run = CudaRun(scene, cam, bg=bg)     # runs gs_raster_fwd
    v = run.view
    img, T, nc = v.image.clone(), v.final_T.clone(), v.n_contrib.clone()
    target = torch.from_numpy(rng.random((H, W, 3), dtype=np.float32)).cuda()
    target.view(-1)[:64] = img.view(-1)[:64]      # sign(0) = 0
    loss_a = torch.zeros(1, dtype=torch.float64, device="cuda")
    pl.l1_loss_grad(v, target, loss_a)
    torch.cuda.synchronize()
    g_a = v.dL_dimage.clone()
    v.image.fill_(-1.0)
    v.final_T.fill_(-1.0)
    v.n_contrib.fill_(-1)
    v.dL_dimage.fill_(7.0)
    loss_b = torch.full((1,), 0.25, dtype=torch.float64, device="cuda")    # accumulates onto what is there
    pl.raster_fwd_l1(run.proj, v, target, loss_b, bg)
    torch.cuda.synchronize()
    assert torch.equal(v.image, img) and torch.equal(v.final_T, T) and torch.equal(v.n_contrib, nc)
    assert torch.equal(v.dL_dimage, g_a)
    assert abs((loss_b.item() - 0.25) - loss_a.item()) <= 1e-12 * loss_a.item()
    want_loss, want_g = orc.l1(img.cpu().numpy(), target.cpu().numpy())
    assert np.array_equal(g_a.cpu().numpy(), want_g)
    assert abs(loss_a.item() - want_loss) <= 1e-12 * want_loss
    assert (nc > 0).float().mean().item() > 0.05


@pytest.mark.parametrize("opaque", [False, True])
def test_counted_forward_visits(opaque):
    """gs_raster_fwd_counted: the same image, final_T and n_contrib as gs_raster_fwd,
    and its counters in their bounds: the pairs the per-pixel loop visits lie
    between sum(n_contrib) (a pixel visits at least up to its last blended entry) and
    the sum over pixels of their tile's list length (reached when no pixel stops);
    blended pairs <= visited pairs.  The opaque stack stops the pixels it covers
    after a few entries, so they visit less than their lists."""
    if opaque:
        n = 600
        rng = np.random.default_rng(4)
        means = np.zeros((n, 3), np.float32)
        means[:, :2] = 0.02 * rng.standard_normal((n, 2))
        means[:, 2] = np.linspace(-1.0, 1.0, n)
        scene = scenes.Scene(means, np.tile(np.float32([1, 0, 0, 0]), (n, 1)),
                             np.full((n, 3), -1.0, np.float32), np.full(n, 4.0, np.float32),
                             rng.uniform(0, 1, (n, 1, 3)).astype(np.float32), 0)
        cam = scenes.tiny().cameras[0]
    else:
        wl = scenes.tiny()
        scene, cam = wl.scene, wl.cameras[0]
    run = CudaRun(scene, cam)
    img, T, nc = (x.clone() for x in (run.view.image, run.view.final_T, run.view.n_contrib))
    counts = torch.zeros(5, device="cuda", dtype=torch.int64)
    pl.raster_fwd_counted(run.proj, run.view, counts)
    torch.cuda.synchronize()
    assert torch.equal(run.view.image, img) and torch.equal(run.view.final_T, T) and torch.equal(run.view.n_contrib, nc)
    evaluated, blended, staged, reached, visited = counts.cpu().tolist()
    W, H = cam["width"], cam["height"]
    r = run.view.ranges.cpu().numpy().astype(np.int64)
    lens = r[:, 1] - r[:, 0]
    ys, xs = np.mgrid[0:H, 0:W]
    tile = (ys // 16) * ((W + 15) // 16) + xs // 16
    list_pairs = int(lens[tile].sum())
    assert int(nc.sum().item()) <= visited <= list_pairs
    assert blended <= visited
    assert reached <= staged and blended <= evaluated
    if opaque:
        assert visited < list_pairs
    with pytest.raises(ValueError):
        pl.raster_fwd_counted(run.proj, run.view, torch.zeros(4, device="cuda", dtype=torch.int64))
