"""gs_project_views (every view of a batch projected in one launch, the parameters
read once) against gs_project view by view, bit for bit, and against the oracle:
SH degrees 0-3, the 16-bit SH copy, Gaussians culled in some views (behind the
camera, outside the image, non-finite or zero-quaternion parameters), 1, 5 (a
ragged view group) and 16 views."""
import numpy as np
import pytest
import torch

from gaussian_splatting_differentiable_02_b200 import abi, scenes
from gaussian_splatting_differentiable_02_b200 import pipeline as pl

from _parity import check_projection

pytestmark = pytest.mark.gpu

FIELDS = ("xy", "depth", "conic_opacity", "rgb", "rect", "tiles_touched")


def _cams(n_views, seed, W=200, H=120):
    rng = np.random.default_rng(seed)
    cams = []
    for _ in range(n_views):
        eye = rng.standard_normal(3)
        eye = 3.5 * eye / np.linalg.norm(eye)
        R, t = scenes.look_at(eye)
        cams.append(scenes.camera(R, t, 150.0, 150.0, W / 2 + 0.3, H / 2 - 0.2, W, H))
    return cams


def _scene(deg, seed=3, n=3001):
    rng = np.random.default_rng(seed)
    sc = scenes.random_scene(rng, n, deg, mean_box=1.5, log_scale=(-4.5, -1.0))
    sc.means[:40] *= 8.0              # behind some cameras, off-screen in others
    sc.means[40, 1] = np.nan          # non-finite
    sc.quats[41] = 0.0                # zero quaternion
    sc.log_scales[42, 0] = np.inf     # non-finite scale
    return sc


def _as_dict(p: pl.Projected, radius):
    return {"xy": p.xy.cpu().numpy(), "depth": p.depth.cpu().numpy(),
            "conic": p.conic_opacity[:, :3].cpu().numpy(), "opacity": p.conic_opacity[:, 3].cpu().numpy(),
            "rgb": p.rgb[:, :3].cpu().numpy(), "radius": radius.cpu().numpy(),
            "rect": p.rect.cpu().numpy().astype(np.int32) & 0xffff,
            "tiles_touched": p.tiles_touched.cpu().numpy().astype(np.uint32)}


@pytest.mark.parametrize("deg,n_views,half", [(0, 1, False), (1, 5, False), (2, 16, False), (3, 5, False),
                                              (3, 16, False), (3, 5, True)])
def test_project_views_equals_per_view_projection(orc, deg, n_views, half):
    sc = _scene(deg, seed=deg + 10 * n_views)
    cams = _cams(n_views, seed=deg + 7)
    g = pl.Gaussians.from_scene(sc)
    views = [pl.View(sc.n, c) for c in cams]
    sh_half = pl.to_half(g.sh) if half else None
    batched = [pl.Projected(sc.n) for _ in cams]
    radii = torch.full((n_views, sc.n), -7, dtype=torch.int32, device="cuda")
    for p in batched:                       # stale values everywhere, so every output must be written
        for t in (p.xy, p.depth, p.conic_opacity, p.rgb):
            t.fill_(3.0)
    pl.project_views(g, views, batched, [radii[k] for k in range(n_views)], sh_half)
    torch.cuda.synchronize()
    scene_ref = sc
    if half:   # the oracle projects the rounded coefficients (widening a half is exact)
        scene_ref = scenes.Scene(sc.means, sc.quats, sc.log_scales, sc.opacity_logits,
                                 np.asarray(sc.sh, np.float32).astype(np.float16).astype(np.float32), deg)
    culled_somewhere = 0
    for k, (cam, vw) in enumerate(zip(cams, views)):
        single = pl.Projected(sc.n)
        r1 = torch.zeros(sc.n, dtype=torch.int32, device="cuda")
        if half:
            pl.project_sh16(g, sh_half, vw, single, r1)
        else:
            pl.project(g, vw, single, r1)
        torch.cuda.synchronize()
        assert torch.equal(radii[k], r1), k
        for f in FIELDS:
            a, b = getattr(batched[k], f), getattr(single, f)
            assert torch.equal(a.view(torch.int32) if a.dtype == torch.float32 else a,
                               b.view(torch.int32) if b.dtype == torch.float32 else b), (k, f)
        ref = orc.project(scene_ref, cam)
        check_projection(_as_dict(batched[k], radii[k]), ref)
        culled_somewhere += int((ref["radius"] == 0).sum())
    assert culled_somewhere > 3


def test_project_views_argument_checks():
    sc = _scene(1, n=100)
    g = pl.Gaussians.from_scene(sc)
    cams = _cams(17, seed=1)
    views = [pl.View(sc.n, c) for c in cams]
    projs = [pl.Projected(sc.n) for _ in cams]
    with pytest.raises(abi.GsError) as e:
        pl.project_views(g, views, projs)
    assert e.value.status == abi.GS_ERR_INVALID_ARG and "num_views" in e.value.detail
