"""gs_bin_sort_static, the tile sort for callers that cannot allocate device
memory (a host that owns the whole device budget, a frame loop where cudaMalloc
would stall every stream, a foreign runtime with no allocator): its scratch is
a library-owned device array, and its results must equal those of gs_bin_sort
with a caller-owned workspace, call after call.

Collected last on purpose, so that a run that stops at the first failure has
already run every other test."""
import numpy as np
import pytest
import torch

from gaussian_splatting_differentiable_02_b200 import abi, scenes
from gaussian_splatting_differentiable_02_b200 import pipeline as pl

pytestmark = pytest.mark.gpu


def _inputs(scene, cam):
    g = pl.Gaussians.from_scene(scene)
    view = pl.View(scene.n, cam)
    proj = pl.Projected(scene.n)
    pl.project(g, view, proj)
    return g, view, proj


def _with_workspace(proj, view):
    K = pl.bin_sort(proj, view)
    torch.cuda.synchronize()
    return K, view.keys[:K].clone(), view.vals[:K].clone(), view.ranges.clone()


def _outputs(capacity, view):
    keys = torch.zeros(capacity, dtype=torch.int64, device="cuda")
    vals = torch.zeros(capacity, dtype=torch.int32, device="cuda")
    ranges = torch.full_like(view.ranges, -1)
    torch.cuda.synchronize()
    return keys, vals, ranges


def _with_static_scratch(proj, view, out):
    """One gs_bin_sort_static call into the preallocated `out`; returns its results and
    the device's free bytes and torch's allocated bytes before and after the call."""
    keys, vals, ranges = out
    ranges.fill_(-1)
    torch.cuda.synchronize()
    before = (torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated())
    st, K = abi.gs_bin_sort_static(proj.struct(), view.n, view.gcam, keys.data_ptr(), vals.data_ptr(), keys.numel(),
                                   ranges.data_ptr(), torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    after = (torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated())
    assert st == abi.GS_OK
    return (K, keys[:K], vals[:K], ranges), before, after


def test_static_scratch_matches_caller_workspace_on_consecutive_calls():
    rng = np.random.default_rng(11)
    tiny = scenes.tiny()
    ragged = scenes.random_scene(rng, 5000, 1, log_scale=(-3.5, -1.5))
    R, t = scenes.look_at((0.4, 0.3, -3.5))
    ragged_cam = scenes.camera(R, t, 180.0, 180.0, 110.0, 45.0, 220, 90)
    cases = [(tiny.scene, tiny.cameras[0]), (ragged, ragged_cam), (tiny.scene, tiny.cameras[0])]
    for scene, cam in cases:
        g, view, proj = _inputs(scene, cam)
        want = _with_workspace(proj, view)
        out = _outputs(want[0] + 1000, view)
        for call in range(2):                    # two calls in a row on the shared scratch
            got, before, after = _with_static_scratch(proj, view, out)
            assert got[0] == want[0] > 0
            for a, b in zip(got[1:], want[1:]):
                assert torch.equal(a, b)
            if call == 1:
                # the module (and with it the array) was loaded by the first call; the
                # second one takes no device memory, neither from the driver nor from torch
                assert after == before, (before, after)


def test_sizes_beyond_the_static_scratch_are_rejected():
    tiny = scenes.tiny()
    g, view, proj = _inputs(tiny.scene, tiny.cameras[0])
    too_many = abi.GS_STATIC_SCRATCH_BYTES // 8          # the ping-pong keys alone would not fit
    keys = torch.zeros(16, dtype=torch.int64, device="cuda")
    vals = torch.zeros(16, dtype=torch.int32, device="cuda")
    with pytest.raises(abi.GsError) as e:
        abi.gs_bin_sort_static(proj.struct(), view.n, view.gcam, keys.data_ptr(), vals.data_ptr(), too_many,
                               view.ranges.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert e.value.status == abi.GS_ERR_UNSUPPORTED
    assert "static scratch" in e.value.detail
    need = abi.gs_bin_sort_workspace_bytes(view.n, too_many, view.gcam)
    assert need > abi.GS_STATIC_SCRATCH_BYTES
