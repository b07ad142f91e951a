"""Host logic of the Trainer that runs without a GPU: the view groups of the
batched path, the lookup of a view's depth-order row, the packed layout's buffers
and their resizing after densification, and the option checks.  Device work is
not called: the Trainer is built on CPU tensors, whose allocations and the
library's host-side size queries need no GPU."""
import numpy as np
import pytest
import torch

from gaussian_splatting_differentiable_02_b200 import pipeline as pl
from gaussian_splatting_differentiable_02_b200 import scenes

LRS = dict(scenes.ADAM_LR)


def _trainer(n_views=5, n=300, **kw):
    rng = np.random.default_rng(0)
    scene = scenes.random_scene(rng, n, 1)
    cams = []
    for k in range(n_views):
        R, t = scenes.look_at((np.cos(k), 0.3, np.sin(k) - 4.0))
        cams.append(scenes.camera(R, t, 64.0, 64.0, 32.0, 32.0, 64, 64))
    views = [pl.View(n, c, device="cpu") for c in cams]
    targets = [torch.zeros((64, 64, 3)) for _ in cams]
    return pl.Trainer(pl.Gaussians.from_scene(scene, device="cpu"), views, targets, dict(LRS), densify=True, **kw)


@pytest.mark.parametrize("n_views,groups,want", [
    (5, 1, [[0, 1, 2, 3, 4]]),
    (5, 2, [[0, 1, 2], [3, 4]]),
    (5, 5, [[0], [1], [2], [3], [4]]),
    (5, 9, [[0], [1], [2], [3], [4]]),
    (16, 3, [list(range(0, 6)), list(range(6, 12)), list(range(12, 16))]),
    (1, 4, [[0]]),
])
def test_view_groups_cover_every_view_once_in_order(n_views, groups, want):
    tr = _trainer(n_views, groups=groups)
    got = tr.view_groups()
    assert got == want
    assert [k for ks in got for k in ks] == list(range(n_views))
    # one depth order per group, each row the view's own
    assert len(tr.depth_orders) == len(got)
    for gi, ks in enumerate(got):
        assert tr.depth_orders[gi].views == len(ks)
        for j, k in enumerate(ks):
            assert tr.order_row(k).data_ptr() == tr.depth_orders[gi].order[j].data_ptr()


def test_packed_buffers_follow_the_slot_capacity():
    tr = _trainer(3, n=500, packed=True)
    assert tr.pcap == 500 and tr.radii is None
    assert all(pk.slot_of.numel() == 500 and pk.capacity == 500 for pk in tr.packs)
    assert [p is pk.proj for p, pk in zip(tr.projs, tr.packs)] == [True] * 3
    assert all(vw.n == 500 for vw in tr.views)
    keys_before = tr.views[0].keys
    tr._alloc_packed(200)
    assert tr.pcap == 200
    assert all(pk.proj.xy.shape[0] == 200 and pk.ids.numel() == 200 for pk in tr.packs)
    assert all(d.n == 200 for d in tr.depth_orders)
    assert all(g.xy.shape[0] == 200 for g in tr.grad2ds)
    # the visible counters are rows of the step's single read-back tensor
    for k, pk in enumerate(tr.packs):
        assert pk.num_visible.data_ptr() == tr.counts[1][k:k + 1].data_ptr()
    # fewer slots keep the instance buffers (and their contents) of the views
    assert tr.views[0].keys is keys_before


def test_option_checks():
    with pytest.raises(ValueError):
        _trainer(2, packed=True, batched_sort=False)
    with pytest.raises(ValueError):
        _trainer(2, sh16=True, packed=True)
    with pytest.raises(ValueError):
        _trainer(2, sh16=True, fused=False)


def test_view_set_n_keeps_or_grows_the_instance_buffers():
    R, t = scenes.look_at((0.0, 0.0, -4.0))
    cam = scenes.camera(R, t, 64.0, 64.0, 32.0, 32.0, 64, 64)
    view = pl.View(1000, cam, device="cpu")
    assert view.capacity == 4000
    keys = view.keys
    view.set_n(200)                      # fewer Gaussians: same buffers, same contents
    assert view.keys is keys and view.capacity == 4000 and view.n == 200
    ws = view.workspace.numel()
    view.set_n(3000)                     # more: the capacity grows to 4 n, new buffers
    assert view.capacity == 12000 and view.keys is not keys
    assert view.workspace.numel() >= ws
    from gaussian_splatting_differentiable_02_b200 import abi
    assert view.workspace.numel() >= abi.gs_bin_sort_workspace_bytes(3000, 12000, view.gcam)


@pytest.mark.parametrize("cull", [True, False])
def test_tile_cull_reaches_every_view_and_its_workspace(cull):
    """Trainer(tile_cull=...) sets the flag in every view's camera and grows each view's
    sort workspace to what the culled binning needs (its runs and counts); set_n after
    densification keeps sizing it for the flag."""
    from gaussian_splatting_differentiable_02_b200 import abi
    tr = _trainer(3, n=400, tile_cull=cull)
    for vw in tr.views:
        assert vw.tile_cull is cull and vw.gcam.tile_cull == int(cull)
        need = abi.gs_bin_sort_workspace_bytes(vw.n, vw.capacity, vw.gcam)
        assert vw.workspace.numel() >= need
    plain = abi.gs_bin_sort_workspace_bytes(400, tr.views[0].capacity, abi.make_camera(tr.views[0].cam))
    culled = abi.gs_bin_sort_workspace_bytes(400, tr.views[0].capacity, abi.make_camera(tr.views[0].cam, True))
    assert culled > plain
    vw = tr.views[0]
    vw.set_n(900)
    assert vw.workspace.numel() >= abi.gs_bin_sort_workspace_bytes(900, vw.capacity, vw.gcam)
    # set_camera keeps the flag
    vw.set_camera(dict(vw.cam))
    assert vw.gcam.tile_cull == int(cull)


def test_trainer_set_tile_cull_switches_views_and_drops_the_graph():
    tr = _trainer(3, n=300, tile_cull=True)
    tr._graph = object()   # stands for a captured graph
    tr.set_tile_cull(False)
    assert tr._graph is None and tr.tile_cull is False
    assert all(not vw.tile_cull and vw.gcam.tile_cull == 0 for vw in tr.views)
