"""16-bit (FP16) storage of the SH coefficients (the guides' FP16 mode: gsplat
guide lmnt.cn/news/262699 §4.3 mixed precision, the A100 practice page's FP16
parameters): gs_to_half against IEEE round-to-nearest-even (numpy's float16),
gs_project_sh16 against the float32 path on the rounded coefficients (bit for
bit) and the oracle, the colour and image error against the float32
coefficients within the bound the rounding allows, and the fused Adam step that
keeps the float32 master and refreshes the half copy."""
import numpy as np
import pytest
import torch

from gaussian_splatting_differentiable_02_b200 import abi, scenes
from gaussian_splatting_differentiable_02_b200 import pipeline as pl

from _parity import check_projection

pytestmark = pytest.mark.gpu

NAMES = ("means", "quats", "log_scales", "opacity_logits", "sh")
LRS = {"means": 1.6e-4, "log_scales": 5e-3, "quats": 1e-3, "opacity_logits": 5e-2, "sh": 2.5e-3}


def _half_bits(x):
    return np.asarray(x, np.float32).astype(np.float16).view(np.uint16)


def test_to_half_rounds_to_nearest_even():
    rng = np.random.default_rng(51)
    parts = [
        rng.standard_normal(10001).astype(np.float32),                          # normal range
        (rng.random(3001) * 6e-5).astype(np.float32) * rng.choice([-1, 1], 3001),  # half subnormals
        np.float32([0.0, -0.0, 65504.0, 65519.99, 65520.0, 1e6, -1e6, np.inf, -np.inf, 2.0 ** -24, 2.0 ** -25,
                    3 * 2.0 ** -26]),
        # exact ties between neighbouring halves: 1 + (2k + 1) 2^-11 rounds to the even neighbour
        np.float32(1.0 + (2 * np.arange(64) + 1) * 2.0 ** -11),
        np.float32(-(1024.0 + (2 * np.arange(64) + 1) * 0.5)),
    ]
    x = np.concatenate(parts).astype(np.float32)
    x = x[: 4 * ((len(x) - 3) // 4) + 3]    # a ragged count: the scalar tail runs too
    assert len(x) % 4 == 3
    xd = torch.from_numpy(x).cuda()
    out = pl.to_half(xd)
    torch.cuda.synchronize()
    got = out.cpu().numpy().view(np.uint16)
    assert np.array_equal(got, _half_bits(x))
    nan = torch.tensor([np.nan, 1.0, np.nan, 2.0], device="cuda")
    h = pl.to_half(nan).cpu().numpy().view(np.float16)
    assert np.isnan(h[0]) and np.isnan(h[2]) and h[1] == 1.0 and h[3] == 2.0


def _rounded(scene):
    r = scene.subset(np.arange(scene.n))
    r.sh = np.asarray(scene.sh, np.float32).astype(np.float16).astype(np.float32)
    return r


@pytest.mark.parametrize("deg", [0, 1, 3])
def test_project_sh16_is_the_float32_path_on_rounded_coefficients(orc, deg):
    rng = np.random.default_rng(52 + deg)
    scene = scenes.random_scene(rng, 5000, deg, mean_box=1.0, log_scale=(-4.0, -2.0))
    scene.sh = (np.asarray(scene.sh) * 3.0).astype(np.float32)
    scene.sh[7, 0, 0] = 7e4        # rounds to infinity in half precision: culled by the colour test
    R, t = scenes.look_at((0.3, -0.2, -3.5))
    cam = scenes.camera(R, t, 150.0, 150.0, 80.0, 61.5, 160, 123)
    g = pl.Gaussians.from_scene(scene)
    half = pl.to_half(g.sh)
    view = pl.View(scene.n, cam)
    p16 = pl.Projected(scene.n)
    pl.project_sh16(g, half, view, p16)
    rs = _rounded(scene)
    p32 = pl.Projected(scene.n)
    pl.project(pl.Gaussians.from_scene(rs), view, p32)
    torch.cuda.synchronize()
    for f in ("xy", "depth", "conic_opacity", "rgb", "radius", "rect", "tiles_touched"):
        a, b = getattr(p16, f).cpu().numpy(), getattr(p32, f).cpu().numpy()
        assert np.array_equal(a.view(np.uint8), b.view(np.uint8)), f
    assert p16.radius[7].item() == 0
    ref = orc.project(rs, cam)
    rect = p16.rect.cpu().numpy().astype(np.int32) & 0xffff
    gpu = {"xy": p16.xy.cpu().numpy(), "depth": p16.depth.cpu().numpy(),
           "conic": p16.conic_opacity[:, :3].cpu().numpy(), "opacity": p16.conic_opacity[:, 3].cpu().numpy(),
           "rgb": p16.rgb[:, :3].cpu().numpy(), "radius": p16.radius.cpu().numpy(), "rect": rect,
           "tiles_touched": p16.tiles_touched.cpu().numpy().astype(np.uint32)}
    check_projection(gpu, ref)


def _unsold_bound(sh, sh_half):
    """Per Gaussian and channel: sum over degrees l of sqrt((2l+1)/(4 pi)) ||dc_l||_2, which
    bounds |sum_m Y_lm dc_lm| for any unit direction (Unsold: sum_m Y_lm^2 = (2l+1)/(4 pi))."""
    d = np.asarray(sh, np.float64) - np.asarray(sh_half, np.float64)      # [n, nc, 3]
    nc = d.shape[1]
    deg = int(round(np.sqrt(nc))) - 1
    b = np.zeros((d.shape[0], 3))
    for l in range(deg + 1):
        blk = d[:, l * l:(l + 1) * (l + 1), :]
        b += np.sqrt((2 * l + 1) / (4 * np.pi)) * np.sqrt((blk ** 2).sum(axis=1))
    return b


def test_sh16_colour_and_image_error_within_the_rounding_bound():
    """The 1M mixture at 1296x840 (SH degree 3): the colours from 16-bit coefficients differ
    from the float32 ones by at most the Unsold bound of the coefficient rounding (plus one
    float32 rounding of each colour); the images by at most the largest colour bound, since
    the compositing weights are the same and sum to at most 1."""
    wl = scenes.mixture1m()
    scene, cam = wl.scene, wl.cameras[0]
    g = pl.Gaussians.from_scene(scene)
    half = pl.to_half(g.sh)
    out = []
    for sh16 in (False, True):
        view = pl.View(scene.n, cam)
        p = pl.Projected(scene.n)
        if sh16:
            pl.project_sh16(g, half, view, p)
        else:
            pl.project(g, view, p)
        pl.bin_sort(p, view)
        pl.raster_fwd(p, view)
        torch.cuda.synchronize()
        out.append((p.rgb[:, :3].cpu().numpy().astype(np.float64), p.radius.cpu().numpy(),
                    view.image.cpu().numpy().astype(np.float64)))
    (c32, r32, i32), (c16, r16, i16) = out
    assert np.array_equal(r32, r16)
    sh = np.asarray(scene.sh, np.float32)
    bound = _unsold_bound(sh, sh.astype(np.float16).astype(np.float32))
    vis = r32 > 0
    slack = 2.0 * np.spacing(np.float32(np.maximum(c32, c16)).astype(np.float32)).astype(np.float64)
    err = np.abs(c16 - c32)
    assert np.all(err[vis] <= bound[vis] + slack[vis])
    assert err[vis].max() > 0                     # the rounding is visible
    # plus the float32 accumulation of the two composites (the image parity tolerance)
    img_bound = bound[vis].max() + 1e-5
    assert np.abs(i16 - i32).max() <= img_bound


def _grad2d(rows, n):
    gd = pl.Grad2D(n)
    rows = np.asarray(rows, np.float32)
    gd.xy.copy_(torch.from_numpy(np.ascontiguousarray(rows[:, 0:2])))
    gd.conic_opacity.copy_(torch.from_numpy(np.ascontiguousarray(rows[:, 2:6])))
    rgb = np.zeros((n, 4), np.float32)
    rgb[:, :3] = rows[:, 6:9]
    gd.rgb.copy_(torch.from_numpy(rgb))
    return gd


def _cams(k):
    rng = np.random.default_rng(60)
    cams = []
    for _ in range(k):
        e = rng.standard_normal(3)
        R, t = scenes.look_at(3.5 * e / np.linalg.norm(e))
        cams.append(scenes.camera(R, t, 128.0, 128.0, 64.0, 64.0, 128, 128))
    return cams


def test_fused_adam_sh16(orc):
    """The chain takes the half coefficients: its gradient is the float32 path's on the rounded
    coefficients (bit for bit); Adam updates the float32 master; the half copy is refreshed in
    place with the master's rounding."""
    rng = np.random.default_rng(61)
    scene = scenes.random_scene(rng, 2000, 3, mean_box=1.0, log_scale=(-4.0, -2.0))
    n = scene.n
    cams = _cams(3)
    rows = [rng.standard_normal((n, 9)).astype(np.float32) for _ in cams]
    lr = [LRS[k] for k in NAMES]
    res = []
    for sh16 in (False, True):
        # float32 path: the scene with rounded coefficients; half path: the unrounded master
        g = pl.Gaussians.from_scene(_rounded(scene) if not sh16 else scene)
        half = pl.to_half(g.sh)
        m, v, grads = g.zeros_like(), g.zeros_like(), g.zeros_like()
        radii = torch.zeros((len(cams), n), dtype=torch.int32, device="cuda")
        proj = pl.Projected(n)
        views = [pl.View(n, c) for c in cams]
        for k, vw in enumerate(views):
            if sh16:
                pl.project_sh16(g, half, vw, proj, radii[k])
            else:
                pl.project(g, vw, proj, radii[k])
        g2 = [_grad2d(r, n) for r in rows]
        structs = [proj.struct(radii[k]) for k in range(len(cams))]
        gcams = [vw.gcam for vw in views]
        master = g.sh.clone()
        if sh16:
            abi.gs_project_bwd_views_adam_sh16(g.params(), gcams, structs, [x.struct() for x in g2], half.data_ptr(),
                                               half.data_ptr(), g.grads(), m.grads(), v.grads(), lr, 0.9, 0.99,
                                               1e-15, 1, grads=grads.grads())
        else:
            abi.gs_project_bwd_views_adam(g.params(), gcams, structs, [x.struct() for x in g2], g.grads(), m.grads(),
                                          v.grads(), lr, 0.9, 0.99, 1e-15, 1, grads=grads.grads())
        torch.cuda.synchronize()
        res.append((grads.to_numpy(), g, m, v, half, master))
    (ga, g32, m32, v32, _, _), (gb, g16, m16, v16, half, master) = res
    for k in NAMES:
        assert np.array_equal(ga[k].view(np.uint8), gb[k].view(np.uint8)), k
    # the geometric groups saw the same inputs and gradients: identical updates
    for k in ("means", "quats", "log_scales", "opacity_logits"):
        assert torch.equal(getattr(g32, k), getattr(g16, k)), k
    # the SH master: the oracle's Adam step of the unrounded coefficients with that gradient
    b1, b2, eps = (float(np.float32(x)) for x in (0.9, 0.99, 1e-15))
    p0 = master.cpu().numpy()
    gref = pl.sh_to_planes(np.asarray(gb["sh"], np.float32))
    z = np.zeros_like(p0)
    p1, _, _ = orc.adam(p0, gref, z, z, float(np.float32(LRS["sh"])), b1, b2, eps, 1)
    got = g16.sh.cpu().numpy()
    eps32 = float(np.finfo(np.float32).eps)
    upd = np.abs(p1.astype(np.float64) - p0)
    bound = eps32 * np.maximum(np.abs(p1), np.abs(p0)) + 1e-3 * upd + 1e-9
    assert np.all(np.abs(got - p1) <= bound)
    assert np.any(got != p0)
    np.testing.assert_array_equal(m16.sh.cpu().numpy(), m32.sh.cpu().numpy())
    # the refreshed half copy is the master's rounding
    assert np.array_equal(half.cpu().numpy().view(np.uint16), _half_bits(got))


def test_trainer_sh16():
    """Trainer(sh16=True): the first step on a scene whose coefficients are already halves gives
    the float32 Trainer's loss and keys; the half copy tracks the master through the steps and
    a densification."""
    rng = np.random.default_rng(62)
    scene = scenes.random_scene(rng, 3000, 2, mean_box=1.0, log_scale=(-4.0, -2.5))
    scene = _rounded(scene)
    cams = _cams(4)
    targets = [torch.from_numpy(rng.random((128, 128, 3)).astype(np.float32)).cuda() for _ in cams]
    out = []
    for sh16 in (False, True):
        tr = pl.Trainer(pl.Gaussians.from_scene(scene), [pl.View(scene.n, c) for c in cams], targets, dict(LRS),
                        densify=True, sh16=sh16)
        tr.step()
        torch.cuda.synchronize()
        out.append((tr.loss.item(), tr.kcount.cpu().numpy(),
                    [vw.keys[:int(K)].cpu().numpy() for vw, K in zip(tr.views, tr.kcount.cpu().tolist())]))
        if sh16:
            for _ in range(2):
                tr.step()
            tr.densify_and_prune(grad_threshold=1e-6, max_screen_size=0)
            tr.step()
            torch.cuda.synchronize()
            assert np.isfinite(tr.loss.item())
            assert torch.equal(tr.sh_half, pl.to_half(tr.gauss.sh))
    (la, ka, keys_a), (lb, kb, keys_b) = out
    assert abs(la - lb) <= 1e-9 * abs(la) and np.array_equal(ka, kb)
    assert all(np.array_equal(x, y) for x, y in zip(keys_a, keys_b))
