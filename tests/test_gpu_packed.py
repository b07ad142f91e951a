"""The packed layout (the packed option of rasterize_gaussians, gsplat guide
lmnt.cn/news/262699 §4.1): gs_project_packed against gs_project and the oracle's
visibility, and the rest of the path on packed arrays against the unpacked path.

Packing is index work: the slots must hold exactly the Gaussians the oracle keeps
(radius > 0), in ascending order, with features bit-identical to gs_project's.
Because slots ascend with the Gaussian id, the binning gives the same keys with
values mapped through the slot ids, the forward pass the same images bit for bit,
and the backward through the projection the same gradients bit for bit when fed
the same 2D gradients."""
import numpy as np
import pytest
import torch

from gaussian_splatting_differentiable_02_b200 import abi, scenes
from gaussian_splatting_differentiable_02_b200 import pipeline as pl

from _parity import BAND_ALPHA, BAND_T, check_grads, check_images

pytestmark = pytest.mark.gpu

NAMES = ("means", "quats", "log_scales", "opacity_logits", "sh")
LRS = {"means": 1.6e-4, "log_scales": 5e-3, "quats": 1e-3, "opacity_logits": 5e-2, "sh": 2.5e-3}
FEATURES = ("xy", "depth", "conic_opacity", "rgb", "radius", "rect", "tiles_touched")


def _scene(seed=41, n=4000, deg=2):
    rng = np.random.default_rng(seed)
    scene = scenes.random_scene(rng, n, deg, mean_box=1.0, log_scale=(-4.0, -2.0))
    scene.means[: n // 10] += 25.0     # outside every view
    scene.means[n // 10: n // 8, 2] = -4.0   # on the camera plane: behind the near plane
    return scene


def _cam(seed=0, w=160, h=120):
    rng = np.random.default_rng(seed)
    eye = rng.standard_normal(3)
    R, t = scenes.look_at(3.5 * eye / np.linalg.norm(eye))
    return scenes.camera(R, t, 140.0, 140.0, w / 2, h / 2, w, h)


def _pack(g, view, capacity):
    pk = pl.Packed(g.n, capacity)
    ws = pl.project_packed_workspace(g.n)
    pl.project_packed(g, view, pk, ws)
    torch.cuda.synchronize()
    return pk


def _np(t):
    return t.cpu().numpy()


@pytest.mark.parametrize("cap", ["n", "exact", "short", "zero"])
def test_packed_projection(orc, cap):
    scene = _scene()
    cam = _cam()
    g = pl.Gaussians.from_scene(scene)
    view = pl.View(scene.n, cam)
    full = pl.Projected(scene.n)
    pl.project(g, view, full)
    ref = orc.project(scene, cam)
    keep = np.nonzero(ref["radius"] > 0)[0]          # the oracle's visible set, ascending
    V = len(keep)
    assert 0 < V < scene.n
    capacity = {"n": scene.n, "exact": V, "short": V // 3, "zero": 0}[cap]
    pk = _pack(g, view, capacity)
    assert int(pk.num_visible.item()) == V
    used = min(V, capacity)
    ids = _np(pk.ids).view(np.uint32)[:capacity]
    assert np.array_equal(ids[:used], keep[:used].astype(np.uint32))
    assert np.all(ids[used:] == 0xffffffff)
    slot = _np(pk.slot_of)
    want_slot = np.full(scene.n, -1, np.int32)
    want_slot[keep[:used]] = np.arange(used, dtype=np.int32)
    assert np.array_equal(slot, want_slot)
    for f in FEATURES:
        a = _np(getattr(pk.proj, f))[:capacity]
        b = _np(getattr(full, f))
        assert np.array_equal(a[:used].view(np.uint8), b[keep[:used]].view(np.uint8)), f
        assert not np.any(a[used:].view(np.uint8)), f


def test_packed_empty_and_all_culled():
    cam = _cam()
    for n in (0, 300):
        rng = np.random.default_rng(3)
        scene = scenes.random_scene(rng, n, 0)
        scene.means[:] += 50.0
        g = pl.Gaussians.from_scene(scene)
        pk = _pack(g, pl.View(max(n, 1), cam), max(n, 4))
        assert int(pk.num_visible.item()) == 0
        assert np.all(_np(pk.ids).view(np.uint32) == 0xffffffff)
        assert np.all(_np(pk.proj.tiles_touched) == 0)
        if n:
            assert np.all(_np(pk.slot_of) == -1)


def _run_view(g, cam, proj, n, up, radius=None):
    """bin, forward, backward of one view on given projected features (n entries)."""
    view = pl.View(n, cam, capacity=60 * max(n, 1))
    K = pl.bin_sort(proj, view, radius)
    pl.raster_fwd(proj, view, radius=radius)
    view.dL_dimage.copy_(torch.from_numpy(up))
    g2 = pl.Grad2D(n)
    pl.raster_bwd(proj, view, g2, radius=radius)
    torch.cuda.synchronize()
    return view, K, g2


def test_packed_path_matches_unpacked_and_oracle(orc):
    scene = _scene(seed=42)
    cam = _cam(1)
    g = pl.Gaussians.from_scene(scene)
    rng = np.random.default_rng(9)
    up = rng.standard_normal((cam["height"], cam["width"], 3)).astype(np.float32)
    full = pl.Projected(scene.n)
    pl.project(g, pl.View(scene.n, cam), full)
    vu, Ku, gu = _run_view(g, cam, full, scene.n, up)
    V = int((_np(full.radius) > 0).sum())
    cap = V + 37                                   # a ragged tail of culled slots
    pk = _pack(g, pl.View(scene.n, cam), cap)
    vp, Kp, gp = _run_view(g, cam, pk.proj, cap, up)
    ids = _np(pk.ids).view(np.uint32)
    # binning: the same keys, values through the slot ids, the same ranges
    assert Kp == Ku
    assert np.array_equal(_np(vp.keys[:Kp]), _np(vu.keys[:Ku]))
    assert np.array_equal(ids[_np(vp.vals[:Kp]).view(np.uint32)], _np(vu.vals[:Ku]).view(np.uint32))
    assert np.array_equal(_np(vp.ranges), _np(vu.ranges))
    # forward: bit for bit
    for f in ("image", "final_T", "n_contrib"):
        assert np.array_equal(_np(getattr(vp, f)), _np(getattr(vu, f))), f
    # backward: the packed rows are the unpacked rows of the slot ids (up to the order of
    # the atomic adds of different warps)
    rows_u = gu.as_rows()
    rows_p = gp.as_rows()[:V]
    scale = np.abs(rows_u).max(axis=0)
    assert np.all(np.abs(rows_p - rows_u[ids[:V]]) <= 1e-6 * scale + 1e-5 * np.abs(rows_u[ids[:V]]))
    assert not np.any(gp.as_rows()[V:])
    # and against the oracle
    ref = orc.project(scene, cam)
    img, T, nc, amb = orc.render(ref, cam, band_alpha=BAND_ALPHA, band_T=BAND_T)
    check_images(_np(vp.image).reshape(-1, 3), _np(vp.final_T).reshape(-1), _np(vp.n_contrib).reshape(-1), img, T,
                 nc, amb)
    want, _, touched = orc.render_bwd(ref, cam, up.reshape(-1, 3).astype(np.float64), band_alpha=BAND_ALPHA,
                                      band_T=BAND_T)
    rows = np.nonzero(touched[ids[:V]] == 0)[0]
    for c, name in enumerate(("du", "dv", "dA", "dB", "dC", "do", "dr", "dg", "db")):
        check_grads(rows_p[:, c], want[ids[:V], c], name, rows=rows)


def _grad2d_from_rows(rows, n):
    gd = pl.Grad2D(n)
    rows = np.asarray(rows, np.float32)
    gd.xy.copy_(torch.from_numpy(np.ascontiguousarray(rows[:, 0:2])))
    gd.conic_opacity.copy_(torch.from_numpy(np.ascontiguousarray(rows[:, 2:6])))
    rgb = np.zeros((n, 4), np.float32)
    rgb[:, :3] = rows[:, 6:9]
    gd.rgb.copy_(torch.from_numpy(rgb))
    return gd


@pytest.mark.parametrize("adam", [False, True])
def test_packed_backward_equals_unpacked(adam):
    """The same 2D gradients, once indexed by Gaussian and once by slot: every gradient,
    statistic and (with Adam) parameter and moment identical bit for bit."""
    scene = _scene(seed=43, n=3000, deg=3)
    cams = [_cam(s) for s in range(4)]
    rng = np.random.default_rng(11)
    n = scene.n
    rows_all = [rng.standard_normal((n, 9)).astype(np.float32) for _ in cams]
    out = []
    for packed in (False, True):
        g = pl.Gaussians.from_scene(scene)
        views = [pl.View(n, c) for c in cams]
        projs, packs, g2s = [], [], []
        for k, vw in enumerate(views):
            if packed:
                pk = _pack(g, vw, n)
                V = int(pk.num_visible.item())
                ids = _np(pk.ids)[:V]
                rows = np.zeros((n, 9), np.float32)
                rows[:V] = rows_all[k][ids]
                packs.append(pk)
                projs.append(pk.proj)
            else:
                p = pl.Projected(n)
                pl.project(g, vw, p)
                projs.append(p)
                rows = rows_all[k] * (_np(p.radius) > 0)[:, None]
            g2s.append(_grad2d_from_rows(rows, n))
        acc = torch.zeros((n,), device="cuda")
        cnt = torch.zeros((n,), device="cuda", dtype=torch.int32)
        mrad = torch.zeros((n,), device="cuda", dtype=torch.int32)
        grads = g.zeros_like()
        slots = [_ptr(pk.slot_of) for pk in packs]
        structs = [p.struct() for p in projs]
        gcams = [vw.gcam for vw in views]
        if adam:
            m, v = g.zeros_like(), g.zeros_like()
            args = (g.params(), gcams, structs)
            tail = ([gd.struct() for gd in g2s], g.grads(), m.grads(), v.grads(), [LRS[k] for k in NAMES], 0.9, 0.99,
                    1e-15, 1)
            kw = dict(grads=grads.grads(), densify_accum=_ptr(acc), densify_count=_ptr(cnt),
                      densify_max_radius=_ptr(mrad))
            if packed:
                abi.gs_project_bwd_views_adam_packed(*args, slots, *tail, **kw)
            else:
                abi.gs_project_bwd_views_adam(*args, *tail, **kw)
            extra = (g.to_numpy(), m.to_numpy(), v.to_numpy())
        else:
            if packed:
                abi.gs_project_bwd_views_packed(g.params(), gcams, structs, slots, [gd.struct() for gd in g2s],
                                                grads.grads(), _ptr(acc), _ptr(cnt), _ptr(mrad))
            else:
                abi.gs_project_bwd_views(g.params(), gcams, structs, [gd.struct() for gd in g2s], grads.grads(),
                                         _ptr(acc), _ptr(cnt), _ptr(mrad))
            extra = ()
        torch.cuda.synchronize()
        out.append((grads.to_numpy(), _np(acc), _np(cnt), _np(mrad), extra))
    (ga, aa, ca, ra, ea), (gb, ab, cb, rb, eb) = out
    assert np.any(ca > 0) and np.any(ca == 0)
    for k in NAMES:
        assert np.array_equal(ga[k].view(np.uint8), gb[k].view(np.uint8)), k
    assert np.array_equal(aa, ab) and np.array_equal(ca, cb) and np.array_equal(ra, rb)
    for xa, xb in zip(ea, eb):
        for k in NAMES:
            assert np.array_equal(xa[k].view(np.uint8), xb[k].view(np.uint8)), k


def _ptr(t):
    return t.data_ptr()


def test_trainer_packed_matches_unpacked():
    """Trainer(packed=True) against the unpacked Trainer: the first step's loss, counts and
    keys identical; later steps (slot capacity shrunk after the first, then forced too
    small so that a step repeats with more slots) agree up to the order of atomic adds."""
    rng = np.random.default_rng(17)
    scene = scenes.random_scene(rng, 20000, 1, mean_box=1.0, log_scale=(-4.5, -3.0))
    scene.means[:12000] += 30.0
    cams = [_cam(s, 128, 128) for s in range(5)]
    targets = [torch.from_numpy(rng.random((128, 128, 3)).astype(np.float32)).cuda() for _ in cams]
    out = []
    for packed in (False, True):
        g = pl.Gaussians.from_scene(scene)
        tr = pl.Trainer(g, [pl.View(scene.n, c) for c in cams], targets, dict(LRS), densify=True, packed=packed)
        tr.step()
        torch.cuda.synchronize()
        first = (tr.loss.item(), tr.densify_count.cpu().numpy(), tr.kcount.cpu().numpy(),
                 [vw.keys[:int(K)].cpu().numpy() for vw, K in zip(tr.views, tr.kcount.cpu().tolist())])
        if packed:
            assert tr.pcap < scene.n     # shrunk to the visible counts
            tr._alloc_packed(64)         # too few slots: the next step grows them and repeats
        tr.step()
        tr.step()
        torch.cuda.synchronize()
        if packed:
            assert tr.pcap >= int(tr.counts[1].max().item())
        out.append((tr.gauss.to_numpy(), first, tr.densify_accum.cpu().numpy(), tr.densify_max_radius.cpu().numpy()))
    (a, (la, ca, ka, keys_a), acc_a, mr_a), (b, (lb, cb, kb, keys_b), acc_b, mr_b) = out
    assert np.array_equal(ca, cb) and np.array_equal(ka, kb)
    assert all(np.array_equal(x, y) for x, y in zip(keys_a, keys_b))
    assert abs(la - lb) <= 1e-9 * abs(la)
    for k in NAMES:
        close = np.abs(a[k] - b[k]) <= 1e-6 + 1e-5 * np.abs(a[k])
        assert close.mean() >= 0.999, (k, float(close.mean()))
    assert np.array_equal(mr_a, mr_b)
    np.testing.assert_allclose(acc_b, acc_a, rtol=1e-4, atol=1e-9)


def test_trainer_packed_densify_then_train():
    """Densification resizes the packed views (slot map and capacity follow the new count)."""
    rng = np.random.default_rng(18)
    scene = scenes.random_scene(rng, 3000, 1, mean_box=1.0, log_scale=(-4.0, -2.5))
    cams = [_cam(s, 128, 128) for s in range(3)]
    targets = [torch.from_numpy(rng.random((128, 128, 3)).astype(np.float32)).cuda() for _ in cams]
    tr = pl.Trainer(pl.Gaussians.from_scene(scene), [pl.View(scene.n, c) for c in cams], targets, dict(LRS),
                    densify=True, packed=True)
    for _ in range(3):
        tr.step()
    # no screen-size limit (2 pixels at 128 x 128 would prune almost everything)
    decision = tr.densify_and_prune(grad_threshold=1e-6, max_screen_size=0).cpu().numpy()
    n2 = tr.gauss.n
    assert n2 > scene.n and n2 == int(np.select([decision == 0, decision == 1], [0, 1], 2).sum())
    assert all(pk.slot_of.numel() == n2 for pk in tr.packs)
    tr.step()
    tr.step()
    torch.cuda.synchronize()
    assert np.isfinite(tr.loss.item())
    vis = tr.counts[1].cpu().numpy()
    assert np.all(vis > 0) and np.all(vis <= tr.pcap)


def test_packed_mixture_keys_match_unpacked():
    """The 1M mixture at 1296x840: packed and unpacked binning agree on every key and value."""
    wl = scenes.mixture1m()
    cam = wl.cameras[0]
    g = pl.Gaussians.from_scene(wl.scene)
    n = wl.scene.n
    full = pl.Projected(n)
    vu = pl.View(n, cam)
    pl.project(g, vu, full)
    Ku = pl.bin_sort(full, vu)
    V = int((full.radius > 0).sum().item())
    pk = _pack(g, pl.View(n, cam), V)
    vp = pl.View(V, cam, capacity=Ku)
    Kp = pl.bin_sort(pk.proj, vp)
    torch.cuda.synchronize()
    assert Kp == Ku
    assert torch.equal(vp.keys[:Kp], vu.keys[:Ku])
    assert torch.equal(pk.ids[vp.vals[:Kp].long()], vu.vals[:Ku])
    assert torch.equal(vp.ranges, vu.ranges)
