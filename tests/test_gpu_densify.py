"""Parity of adaptive density control (gs_densify_plan / gs_densify_apply) with the
oracle's orc_densify: decisions, output count and output order bit-exact, copied
parameters and moments bit-exact, split children (computed in double on both sides
and rounded once) within one float32 ulp; the largest-radius statistic of the
fused backward; edge cases; the Trainer's densify-then-train sequence."""
import numpy as np
import pytest
import torch

from gaussian_splatting_differentiable_02_b200 import abi, scenes
from gaussian_splatting_differentiable_02_b200 import pipeline as pl

pytestmark = pytest.mark.gpu

NAMES = ("means", "quats", "log_scales", "opacity_logits", "sh")
LRS = {"means": 1.6e-4, "log_scales": 5e-3, "quats": 1e-3, "opacity_logits": 5e-2, "sh": 2.5e-3}


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _random_like(rng, scene):
    """A parameter-shaped scene of N(0, 1) values (stand-in Adam moments)."""
    n, nc = scene.n, (scene.sh_degree + 1) ** 2
    f = np.float32
    return scenes.Scene(rng.standard_normal((n, 3)).astype(f), rng.standard_normal((n, 4)).astype(f),
                        rng.standard_normal((n, 3)).astype(f), rng.standard_normal(n).astype(f),
                        rng.standard_normal((n, nc, 3)).astype(f), scene.sh_degree)


def _natural(s):
    return {"means": s.means, "quats": s.quats, "log_scales": s.log_scales, "opacity_logits": s.opacity_logits,
            "sh": s.sh}


def _densify_and_compare(orc, scene, accum, count, max_radius, noise, cfg, moments=True, seed=0):
    rng = np.random.default_rng(seed)
    g = pl.Gaussians.from_scene(scene)
    msc = _random_like(rng, scene) if moments else None
    vsc = _random_like(rng, scene) if moments else None
    m = pl.Gaussians.from_scene(msc) if moments else None
    v = pl.Gaussians.from_scene(vsc) if moments else None
    out, om, ov, dec = pl.densify(g, _dev(accum), _dev(count), _dev(max_radius) if max_radius is not None else None,
                                  _dev(noise), cfg, m, v)
    torch.cuda.synchronize()
    n = scene.n
    want = orc.densify(scene, accum, count, max_radius if max_radius is not None else np.zeros(n, np.int32),
                       noise.reshape(n, 2, 3), cfg.grad_threshold, cfg.scale_threshold, cfg.min_opacity,
                       cfg.max_screen_radius if max_radius is not None else 0,
                       moments=[_natural(msc), _natural(vsc)] if moments else ())
    assert np.array_equal(dec.cpu().numpy(), want["decision"])
    assert out.n == want["n_out"]
    got = out.to_numpy()
    split = want["decision"][want["source"]] == abi.GS_DENSIFY_SPLIT
    for k in NAMES:
        a = np.asarray(got[k], np.float64)
        b = np.asarray(want[k], np.float64)
        if k in ("means", "log_scales"):
            assert np.array_equal(a[~split], b[~split]), k
            ulp = np.spacing(np.abs(b[split]).astype(np.float32)).astype(np.float64)
            assert np.all(np.abs(a[split] - b[split]) <= ulp), (k, float(np.max(np.abs(a[split] - b[split]))))
        else:
            assert np.array_equal(a, b), k
    if moments:
        for mine, ref in zip((om.to_numpy(), ov.to_numpy()), want["moments"]):
            for k in NAMES:
                assert np.array_equal(np.asarray(mine[k], np.float32), np.asarray(ref[k], np.float32)), k
    return want


def test_random_mixture_of_decisions(orc):
    rng = np.random.default_rng(1)
    n = 5000
    # largest scale around the 0.01 clone / split boundary, opacity around the 0.005 minimum
    scene = scenes.random_scene(rng, n, 3, log_scale=(-7.0, -4.0), logit=(-2.0, 3.0))
    accum = rng.uniform(0.0, 6e-4, n).astype(np.float32)
    count = rng.integers(0, 4, n).astype(np.int32)
    max_radius = rng.integers(0, 50, n).astype(np.int32)
    noise = rng.standard_normal((n, 6)).astype(np.float32)
    cfg = pl.densify_config(1920, 1080)   # 0.0002, 0.005, 0.01, 38 px
    want = _densify_and_compare(orc, scene, accum, count, max_radius, noise, cfg)
    counts = np.bincount(want["decision"], minlength=4)
    assert np.all(counts > 100), counts


@pytest.mark.parametrize("deg", [0, 1, 2])
def test_sh_degrees_and_no_moments(orc, deg):
    rng = np.random.default_rng(2 + deg)
    n = 1037   # ragged against the 256-thread blocks
    scene = scenes.random_scene(rng, n, deg, log_scale=(-5.5, -3.0), logit=(-3.0, 3.0))
    accum = rng.uniform(0.0, 4e-4, n).astype(np.float32)
    count = rng.integers(0, 3, n).astype(np.int32)
    noise = rng.standard_normal((n, 6)).astype(np.float32)
    cfg = pl.densify_config(1296, 840)
    _densify_and_compare(orc, scene, accum, count, None, noise, cfg, moments=(deg != 1))


def test_statistics_from_a_training_step_at_full_size(orc):
    """The 1M mixture at 1296x840: statistics from one real training step, the
    gradient threshold at the median of the visible Gaussians' mean statistic."""
    wl = scenes.mixture1m()
    scene = wl.scene
    g = pl.Gaussians.from_scene(scene)
    view = pl.View(scene.n, wl.cameras[0])
    tr = pl.Trainer(g, [view], [_dev(wl.targets[0])], dict(LRS), densify=True)
    tr.step()
    torch.cuda.synchronize()
    n = scene.n
    accum = tr.densify_accum[:n].cpu().numpy()
    count = tr.densify_count[:n].cpu().numpy()
    max_radius = tr.densify_max_radius[:n].cpu().numpy()
    assert np.array_equal(max_radius, tr.radii[0, :n].cpu().numpy())
    vis = count > 0
    thr = float(np.median(accum[vis] / count[vis]))
    cfg = pl.densify_config(1296, 840, grad_threshold=thr)
    noise = np.random.default_rng(3).standard_normal((n, 6)).astype(np.float32)
    # the parameters after the Adam step are the inputs of both sides
    stepped = scenes.Scene(**{k: v for k, v in tr.gauss.to_numpy().items()}, sh_degree=scene.sh_degree)
    want = _densify_and_compare(orc, stepped, accum, count, max_radius, noise, cfg, moments=True)
    counts = np.bincount(want["decision"], minlength=4)
    assert counts[abi.GS_DENSIFY_CLONE] > 1000 and counts[abi.GS_DENSIFY_SPLIT] > 1000, counts


def test_edge_cases(orc):
    rng = np.random.default_rng(4)
    n = 300
    scene = scenes.random_scene(rng, n, 1)
    noise = rng.standard_normal((n, 6)).astype(np.float32)
    ones = np.ones(n, np.int32)
    # everything pruned
    cfg = abi.gs_densify_config(0.0, 1.0, 2.0, 0)
    want = _densify_and_compare(orc, scene, np.ones(n, np.float32), ones, None, noise, cfg)
    assert want["n_out"] == 0
    # everything split (threshold 0, scale threshold 0)
    cfg = abi.gs_densify_config(0.0, 0.0, 0.0, 0)
    want = _densify_and_compare(orc, scene, np.ones(n, np.float32), ones, None, noise, cfg)
    assert want["n_out"] == 2 * n and np.all(want["decision"] == abi.GS_DENSIFY_SPLIT)
    # everything cloned
    cfg = abi.gs_densify_config(0.0, 1e30, 0.0, 0)
    want = _densify_and_compare(orc, scene, np.ones(n, np.float32), ones, None, noise, cfg)
    assert want["n_out"] == 2 * n and np.all(want["decision"] == abi.GS_DENSIFY_CLONE)
    # an empty scene
    empty = scene.subset(np.arange(0))
    g0 = pl.Gaussians.from_scene(empty)
    z = torch.zeros((1,), device="cuda")
    out, _, _, dec = pl.densify(g0, z, z.int(), None, z, abi.gs_densify_config(0.0, 1.0, 0.0, 0))
    assert out.n == 0 and dec.numel() == 0


def test_apply_rejects_a_count_that_is_not_the_plan():
    rng = np.random.default_rng(5)
    scene = scenes.random_scene(rng, 100, 0)
    g = pl.Gaussians.from_scene(scene)
    acc = torch.ones((100,), device="cuda")
    cnt = torch.ones((100,), device="cuda", dtype=torch.int32)
    ws_bytes = abi.gs_densify_workspace_bytes(100)
    ws = torch.empty((ws_bytes,), device="cuda", dtype=torch.uint8)
    dec = torch.empty((100,), device="cuda", dtype=torch.uint8)
    num = torch.zeros((1,), device="cuda", dtype=torch.int64)
    noise = torch.zeros((100, 6), device="cuda")
    cfg = abi.gs_densify_config(0.5, 1e30, 0.0, 0)   # every Gaussian cloned: 200
    s = torch.cuda.current_stream().cuda_stream
    abi.gs_densify_plan(g.params(), acc.data_ptr(), cnt.data_ptr(), 0, cfg, ws.data_ptr(), ws_bytes, dec.data_ptr(),
                        num.data_ptr(), s)
    assert int(num.item()) == 200
    out = pl.Gaussians(150, 0)
    with pytest.raises(abi.GsError) as e:
        abi.gs_densify_apply(g.params(), None, None, noise.data_ptr(), dec.data_ptr(), ws.data_ptr(), ws_bytes, 150,
                             out.grads(), None, None, s)
    assert e.value.status == abi.GS_ERR_INVALID_ARG


def test_max_radius_statistic_over_views(orc):
    rng = np.random.default_rng(6)
    scene = scenes.random_scene(rng, 700, 1, mean_box=1.0, log_scale=(-4.0, -2.0))
    cams = []
    for _ in range(3):
        eye = rng.standard_normal(3)
        R, t = scenes.look_at(4.0 * eye / np.linalg.norm(eye))
        cams.append(scenes.camera(R, t, 128.0, 128.0, 64.0, 64.0, 128, 128))
    g = pl.Gaussians.from_scene(scene)
    views = [pl.View(scene.n, c) for c in cams]
    proj = pl.Projected(scene.n)
    radii = torch.zeros((3, scene.n), dtype=torch.int32, device="cuda")
    for k, vw in enumerate(views):
        pl.project(g, vw, proj, radii[k])
    start = rng.integers(0, 40, scene.n).astype(np.int32)
    mr = _dev(start)
    m, v = g.zeros_like(), g.zeros_like()
    g2s = [pl.Grad2D(scene.n) for _ in cams]
    pl.project_bwd_views_adam(g, views, proj, radii, g2s, m, v, LRS, 1, densify_max_radius=mr)
    torch.cuda.synchronize()
    rows = np.stack([orc.project(scene, c)["radius"] for c in cams])
    assert np.array_equal(mr.cpu().numpy(), np.maximum(start, rows.max(0)))


def test_trainer_densify_then_train():
    rng = np.random.default_rng(7)
    scene = scenes.random_scene(rng, 900, 1, mean_box=1.0, log_scale=(-4.0, -2.5))
    cams = []
    for _ in range(2):
        eye = rng.standard_normal(3)
        R, t = scenes.look_at(4.0 * eye / np.linalg.norm(eye))
        cams.append(scenes.camera(R, t, 128.0, 128.0, 64.0, 64.0, 128, 128))
    targets = [_dev(rng.random((128, 128, 3)).astype(np.float32)) for _ in cams]
    tr = pl.Trainer(pl.Gaussians.from_scene(scene), [pl.View(scene.n, c) for c in cams], targets, dict(LRS),
                    densify=True)
    tr.step()
    tr.step()
    n0 = tr.gauss.n
    dec = tr.densify_and_prune(grad_threshold=1e-9, extent=0.05, max_screen_size=0.5).cpu().numpy()
    counts = np.bincount(dec, minlength=4)
    assert tr.gauss.n == counts[1] + 2 * counts[2] + 2 * counts[3] and tr.gauss.n != n0
    assert all(vw.n == tr.gauss.n for vw in tr.views)
    assert float(tr.densify_accum.abs().sum()) == 0.0
    tr.step()
    tr.step()
    torch.cuda.synchronize()
    assert np.isfinite(tr.loss.item())
    assert int(tr.densify_count.sum()) > 0
