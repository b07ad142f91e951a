"""Device buffers (torch) and the call sequence of one view / one training step.

Argument marshalling only: every computation runs in libgs.so through the
binding in ``abi``.  torch provides device memory and the current stream.

Layouts follow include/gs.h: means/quats/log_scales are [n,4] float32,
opacity logits [n], SH [P,n,4] with P = gs_sh_planes(degree).
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
import torch

from . import abi

PARAM_NAMES = ("means", "quats", "log_scales", "opacity_logits", "sh")


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def _ptr(t: torch.Tensor | None) -> int:
    return 0 if t is None else t.data_ptr()


def sh_planes(deg: int) -> int:
    return {0: 1, 1: 3, 2: 7, 3: 12}[deg]


def sh_to_planes(sh: np.ndarray) -> np.ndarray:
    """[n, nc, 3] coefficients -> [P, n, 4] float4 planes (coefficient-major, zero tail)."""
    n, nc, _ = sh.shape
    deg = int(round(math.sqrt(nc))) - 1
    P = sh_planes(deg)
    flat = np.zeros((n, 4 * P), np.float32)
    flat[:, :3 * nc] = sh.reshape(n, 3 * nc)
    return np.ascontiguousarray(flat.reshape(n, P, 4).transpose(1, 0, 2))


def planes_to_sh(planes: np.ndarray, deg: int) -> np.ndarray:
    P, n, _ = planes.shape
    nc = (deg + 1) ** 2
    flat = planes.transpose(1, 0, 2).reshape(n, 4 * P)
    return flat[:, :3 * nc].reshape(n, nc, 3)


class Gaussians:
    """SoA device copy of a scene's parameters (or of gradients / Adam moments of the same shape)."""

    def __init__(self, n: int, sh_degree: int, device="cuda"):
        self.n = int(n)
        self.sh_degree = int(sh_degree)
        z = dict(device=device, dtype=torch.float32)
        self.means = torch.zeros((n, 4), **z)
        self.quats = torch.zeros((n, 4), **z)
        self.log_scales = torch.zeros((n, 4), **z)
        self.opacity_logits = torch.zeros((n,), **z)
        self.sh = torch.zeros((sh_planes(sh_degree), n, 4), **z)

    @classmethod
    def from_scene(cls, scene, device="cuda") -> "Gaussians":
        g = cls(scene.n, scene.sh_degree, device)
        g.load_scene(scene)
        return g

    def load_scene(self, scene):
        n = self.n
        m = np.zeros((n, 4), np.float32)
        m[:, :3] = scene.means
        self.means.copy_(torch.from_numpy(m))
        self.quats.copy_(torch.from_numpy(np.ascontiguousarray(scene.quats, np.float32)))
        s = np.zeros((n, 4), np.float32)
        s[:, :3] = scene.log_scales
        self.log_scales.copy_(torch.from_numpy(s))
        self.opacity_logits.copy_(torch.from_numpy(np.ascontiguousarray(scene.opacity_logits, np.float32)))
        self.sh.copy_(torch.from_numpy(sh_to_planes(np.asarray(scene.sh, np.float32))))

    def zeros_like(self) -> "Gaussians":
        return Gaussians(self.n, self.sh_degree, self.means.device)

    def tensors(self):
        return {k: getattr(self, k) for k in PARAM_NAMES}

    def params(self) -> abi.gs_params:
        return abi.gs_params(_ptr(self.means), _ptr(self.quats), _ptr(self.log_scales), _ptr(self.opacity_logits),
                             _ptr(self.sh), self.sh_degree, self.n)

    def grads(self) -> abi.gs_param_grads:
        return abi.gs_param_grads(_ptr(self.means), _ptr(self.quats), _ptr(self.log_scales),
                                  _ptr(self.opacity_logits), _ptr(self.sh))

    def zero_(self):
        s = _stream()
        for t in self.tensors().values():
            abi.gs_zero(_ptr(t), t.numel() * 4, s)

    def to_numpy(self) -> dict:
        """Natural layout: means [n,3], quats [n,4], log_scales [n,3], opacity_logits [n], sh [n,nc,3]."""
        return {"means": self.means[:, :3].cpu().numpy(), "quats": self.quats.cpu().numpy(),
                "log_scales": self.log_scales[:, :3].cpu().numpy(),
                "opacity_logits": self.opacity_logits.cpu().numpy(),
                "sh": planes_to_sh(self.sh.cpu().numpy(), self.sh_degree)}


class Projected:
    def __init__(self, n: int, device="cuda"):
        f = dict(device=device, dtype=torch.float32)
        i = dict(device=device, dtype=torch.int32)
        self.n = n
        n = max(n, 1)   # the raster calls take non-NULL feature arrays even for an empty scene
        self.xy = torch.zeros((n, 2), **f)
        self.depth = torch.zeros((n,), **f)
        self.conic_opacity = torch.zeros((n, 4), **f)
        self.rgb = torch.zeros((n, 4), **f)
        self.radius = torch.zeros((n,), **i)
        self.rect = torch.zeros((n, 4), device=device, dtype=torch.int16)   # uint16 values < 2^15
        self.tiles_touched = torch.zeros((n,), **i)                         # uint32 values < 2^31

    def struct(self, radius: torch.Tensor = None) -> abi.gs_projected:
        """The C struct; `radius` replaces the radius array (a view's own copy)."""
        r = self.radius if radius is None else radius
        return abi.gs_projected(_ptr(self.xy), _ptr(self.depth), _ptr(self.conic_opacity), _ptr(self.rgb),
                                _ptr(r), _ptr(self.rect), _ptr(self.tiles_touched))


class Grad2D:
    """2D gradients of one view; absgrad=True also keeps the absolute gradient xy_abs."""

    def __init__(self, n: int, device="cuda", absgrad: bool = False):
        f = dict(device=device, dtype=torch.float32)
        n = max(n, 1)
        self.xy = torch.zeros((n, 2), **f)
        self.conic_opacity = torch.zeros((n, 4), **f)
        self.rgb = torch.zeros((n, 4), **f)
        self.xy_abs = torch.zeros((n, 2), **f) if absgrad else None

    def struct(self) -> abi.gs_grad2d:
        return abi.gs_grad2d(_ptr(self.xy), _ptr(self.conic_opacity), _ptr(self.rgb), _ptr(self.xy_abs))

    def zero_(self):
        s = _stream()
        for t in (self.xy, self.conic_opacity, self.rgb, self.xy_abs):
            if t is not None:
                abi.gs_zero(_ptr(t), t.numel() * 4, s)

    def as_rows(self) -> np.ndarray:
        """[n, 9]: u, v, A, B, C, o, r, g, b (the oracle's order)."""
        return np.concatenate([self.xy.cpu().numpy(), self.conic_opacity.cpu().numpy(),
                               self.rgb[:, :3].cpu().numpy()], axis=1)


class Packed:
    """One view's projection in the packed layout (gs_project_packed, the gsplat guide §4.1
    packed option): `capacity` slots of projected features (`proj`), the Gaussian of every
    slot (`ids`), the slot of every Gaussian (`slot_of`, -1: not in the view) and the number
    of Gaussians the view keeps (`num_visible`, on the device)."""

    def __init__(self, n: int, capacity: int, device="cuda", num_visible: torch.Tensor = None):
        self.n, self.capacity = int(n), int(capacity)
        self.proj = Projected(self.capacity, device)
        self.ids = torch.zeros((max(self.capacity, 1),), device=device, dtype=torch.int32)
        self.slot_of = torch.zeros((max(self.n, 1),), device=device, dtype=torch.int32)
        self.num_visible = torch.zeros((1,), device=device, dtype=torch.int64) if num_visible is None \
            else num_visible


def project_packed_workspace(n: int, device="cuda") -> torch.Tensor:
    return torch.empty((abi.gs_project_packed_workspace_bytes(n),), device=device, dtype=torch.uint8)


def project_packed(g: Gaussians, view: View, packed: Packed, workspace: torch.Tensor):
    """gs_project_packed into `packed` (visible count left on the device)."""
    abi.gs_project_packed(g.params(), view.gcam, _ptr(workspace), workspace.numel(), packed.proj.struct(),
                          packed.capacity, _ptr(packed.ids), _ptr(packed.slot_of), _ptr(packed.num_visible),
                          _stream())


class View:
    """Per-camera buffers: sorted instances, tile ranges, image and its gradient."""

    def __init__(self, n: int, cam: dict, device="cuda", capacity: int = 0, tile_cull: bool = False):
        self.cam = cam
        self.tile_cull = bool(tile_cull)
        self.gcam = abi.make_camera(cam, self.tile_cull)
        self.n = n
        self.device = device
        self.tiles_x, self.tiles_y = abi.gs_tile_grid(self.gcam)
        T = self.tiles_x * self.tiles_y
        H, W = cam["height"], cam["width"]
        self.ranges = torch.zeros((T, 2), device=device, dtype=torch.int32)
        self.image = torch.zeros((H, W, 3), device=device, dtype=torch.float32)
        self.final_T = torch.zeros((H, W), device=device, dtype=torch.float32)
        self.n_contrib = torch.zeros((H, W), device=device, dtype=torch.int32)
        self.dL_dimage = torch.zeros((H, W, 3), device=device, dtype=torch.float32)
        self.order = torch.zeros((T,), device=device, dtype=torch.int32)  # longest tiles first
        self.num_instances = 0
        self.capacity = 0
        self._alloc(max(capacity, 4 * n, 1024))

    def set_camera(self, cam: dict):
        """Another pose of the same image size (the tile grid and the buffers stay)."""
        if (cam["width"], cam["height"]) != (self.cam["width"], self.cam["height"]):
            raise ValueError("set_camera keeps the image size")
        self.cam = cam
        self.gcam = abi.make_camera(cam, self.tile_cull)

    def set_tile_cull(self, on: bool):
        """Bin each Gaussian only into the tiles of its rectangle that its footprint
        reaches (gs_camera.tile_cull), or into the whole rectangle.  The workspace may
        be reallocated: for the views of a Trainer use Trainer.set_tile_cull, which
        also drops a captured CUDA graph."""
        self.tile_cull = bool(on)
        self.gcam = abi.make_camera(self.cam, self.tile_cull)
        nbytes = abi.gs_bin_sort_workspace_bytes(self.n, self.capacity, self.gcam)   # the culled binning's runs
        if nbytes > self.workspace.numel():
            self.workspace = torch.zeros((nbytes,), device=self.device, dtype=torch.uint8)

    def set_n(self, n: int):
        """Resize for a new Gaussian (or packed slot) count: the sort workspace depends on n.
        The instance buffers and their contents stay unless the capacity has to grow."""
        self.n = int(n)
        cap = max(self.capacity, 4 * self.n, 1024)
        if cap != self.capacity:
            self._alloc(cap)
            return
        nbytes = abi.gs_bin_sort_workspace_bytes(self.n, self.capacity, self.gcam)
        if nbytes > self.workspace.numel():
            self.workspace = torch.zeros((nbytes,), device=self.device, dtype=torch.uint8)

    def _alloc(self, capacity: int):
        self.capacity = int(capacity)
        self.keys = torch.zeros((self.capacity,), device=self.device, dtype=torch.int64)
        self.vals = torch.zeros((self.capacity,), device=self.device, dtype=torch.int32)
        nbytes = abi.gs_bin_sort_workspace_bytes(self.n, self.capacity, self.gcam)
        self.workspace = torch.zeros((nbytes,), device=self.device, dtype=torch.uint8)


def project(g: Gaussians, view: View, proj: Projected, radius: torch.Tensor = None):
    abi.gs_project(g.params(), view.gcam, proj.struct(radius), _stream())


def project_views(g: Gaussians, views: list, projs: list, radii: list = None, sh_half: torch.Tensor = None):
    """gs_project of every view in one launch (projs[k] with radius row radii[k] for view k;
    sh_half: project from the 16-bit SH copy)."""
    abi.gs_project_views(g.params(), [vw.gcam for vw in views],
                         [p.struct(None if radii is None else radii[k]) for k, p in enumerate(projs)],
                         _ptr(sh_half), _stream())


def to_half(x: torch.Tensor, out: torch.Tensor = None) -> torch.Tensor:
    """x (float32) rounded to IEEE half, nearest even (gs_to_half); out: an int16 tensor of
    x's shape holding the bit patterns (allocated when None)."""
    if x.dtype != torch.float32 or not x.is_contiguous():
        raise TypeError("to_half takes a contiguous float32 tensor")
    if out is None:
        out = torch.empty(x.shape, device=x.device, dtype=torch.int16)
    abi.gs_to_half(_ptr(x), x.numel(), _ptr(out), _stream())
    return out


def project_sh16(g: Gaussians, sh_half: torch.Tensor, view: View, proj: Projected, radius: torch.Tensor = None):
    """gs_project with the SH coefficients read from their 16-bit copy sh_half ([P, n, 4] halves)."""
    abi.gs_project_sh16(g.params(), _ptr(sh_half), view.gcam, proj.struct(radius), _stream())


def bin_sort(proj: Projected, view: View, radius: torch.Tensor = None):
    """Sort the instances; grows the view's buffers when they are too small.  Returns K."""
    s = _stream()
    while True:
        st, K = abi.gs_bin_sort(proj.struct(radius), view.n, view.gcam, _ptr(view.workspace), view.workspace.numel(),
                                _ptr(view.keys), _ptr(view.vals), view.capacity, _ptr(view.ranges), s, check=False)
        if st == abi.GS_OK:
            view.num_instances = K
            abi.gs_tile_order(_ptr(view.ranges), view.gcam, _ptr(view.order), s)
            return K
        view._alloc(int(K * 1.25) + 1024)


def bin_sort_async(proj: Projected, view: View, counter: torch.Tensor, radius: torch.Tensor = None):
    """Sort without waiting; K lands in `counter` (one int64 on the device).  The
    caller checks K against view.capacity later and repeats the view if it overflowed."""
    abi.gs_bin_sort_async(proj.struct(radius), view.n, view.gcam, _ptr(view.workspace), view.workspace.numel(),
                          _ptr(view.keys), _ptr(view.vals), view.capacity, _ptr(counter), _ptr(view.ranges),
                          _stream())
    abi.gs_tile_order(_ptr(view.ranges), view.gcam, _ptr(view.order), _stream())


class DepthOrder:
    """Depth orders of several views of the same n Gaussians ([views, n] uint32) and the
    workspace of the batched sort that computes them."""

    def __init__(self, n: int, views: int, device="cuda"):
        self.n, self.views = int(n), int(views)
        self.order = torch.empty((views, max(n, 1)), device=device, dtype=torch.int32)
        nbytes = abi.gs_depth_order_workspace_bytes(n, views)
        self.workspace = torch.empty((nbytes,), device=device, dtype=torch.uint8)


def depth_order_views(projs: list, radii: torch.Tensor, d: DepthOrder):
    """Every view's stable depth order in one batched sort (projs[k] with radius row radii[k])."""
    abi.gs_depth_order_views([p.struct(None if radii is None else radii[k]) for k, p in enumerate(projs)], d.n,
                             _ptr(d.workspace),
                             d.workspace.numel(), _ptr(d.order), _stream())


def bin_sort_ordered_async(proj: Projected, view: View, order_row: torch.Tensor, counter: torch.Tensor,
                           radius: torch.Tensor = None):
    """bin_sort_async from a precomputed depth order (a row of DepthOrder.order)."""
    abi.gs_bin_sort_ordered_async(proj.struct(radius), view.n, _ptr(order_row), view.gcam, _ptr(view.workspace),
                                  view.workspace.numel(), _ptr(view.keys), _ptr(view.vals), view.capacity,
                                  _ptr(counter), _ptr(view.ranges), _stream())
    abi.gs_tile_order(_ptr(view.ranges), view.gcam, _ptr(view.order), _stream())


def bin_sort_ordered_views_async(projs: list, views: list, d: DepthOrder, counters: torch.Tensor, radii=None):
    """bin_sort_ordered_async for several views of the same image size at once (view k:
    projs[k] with radius row radii[k], views[k], row k of d.order, counters[k]): every
    binning kernel launched once for all of them, then their tile orders in one launch."""
    nv = len(views)
    abi.gs_bin_sort_ordered_views_async(
        [p.struct(None if radii is None else radii[k]) for k, p in enumerate(projs)], views[0].n, _ptr(d.order),
        [vw.gcam for vw in views], [_ptr(vw.workspace) for vw in views], [vw.workspace.numel() for vw in views],
        [_ptr(vw.keys) for vw in views], [_ptr(vw.vals) for vw in views], [vw.capacity for vw in views],
        [counters.data_ptr() + 8 * k for k in range(nv)], [_ptr(vw.ranges) for vw in views], _stream())
    abi.gs_tile_order_views([_ptr(vw.ranges) for vw in views], views[0].gcam, [_ptr(vw.order) for vw in views],
                            _stream())


def raster_fwd(proj: Projected, view: View, bg=(0.0, 0.0, 0.0), radius: torch.Tensor = None):
    abi.gs_raster_fwd(proj.struct(radius), _ptr(view.vals), _ptr(view.ranges), _ptr(view.order), view.gcam, bg,
                      _ptr(view.image), _ptr(view.final_T), _ptr(view.n_contrib), _stream())


def raster_fwd_l1(proj: Projected, view: View, target: torch.Tensor, loss_dev: torch.Tensor, bg=(0.0, 0.0, 0.0),
                  radius: torch.Tensor = None):
    """raster_fwd and l1_loss_grad in one kernel: image, final_T, n_contrib, dL/dimage
    into the view and loss_dev += mean |image - target|."""
    abi.gs_raster_fwd_l1(proj.struct(radius), _ptr(view.vals), _ptr(view.ranges), _ptr(view.order), view.gcam, bg,
                         _ptr(target), _ptr(view.image), _ptr(view.final_T), _ptr(view.n_contrib),
                         _ptr(view.dL_dimage), _ptr(loss_dev), _stream())


def raster_bwd(proj: Projected, view: View, grad2d: Grad2D, bg=(0.0, 0.0, 0.0), dL_dimage: torch.Tensor = None,
               radius: torch.Tensor = None):
    d = view.dL_dimage if dL_dimage is None else dL_dimage
    abi.gs_raster_bwd(proj.struct(radius), _ptr(view.vals), _ptr(view.ranges), _ptr(view.order), view.gcam, bg,
                      _ptr(view.final_T), _ptr(view.n_contrib), _ptr(d), grad2d.struct(), _stream())


def raster_fwd_counted(proj: Projected, view: View, counts: torch.Tensor, bg=(0.0, 0.0, 0.0),
                       radius: torch.Tensor = None):
    """raster_fwd that also adds its work counters to counts (5 int64 on the device, gs.h)."""
    if counts.numel() < 5:
        raise ValueError("the counted raster calls add to 5 counters")
    abi.gs_raster_fwd_counted(proj.struct(radius), _ptr(view.vals), _ptr(view.ranges), _ptr(view.order), view.gcam,
                              bg, _ptr(view.image), _ptr(view.final_T), _ptr(view.n_contrib), _ptr(counts),
                              _stream())


def raster_bwd_counted(proj: Projected, view: View, grad2d: Grad2D, counts: torch.Tensor, bg=(0.0, 0.0, 0.0),
                       radius: torch.Tensor = None):
    """raster_bwd (upstream view.dL_dimage) that also adds its work counters to counts."""
    if counts.numel() < 5:
        raise ValueError("the counted raster calls add to 5 counters")
    abi.gs_raster_bwd_counted(proj.struct(radius), _ptr(view.vals), _ptr(view.ranges), _ptr(view.order), view.gcam,
                              bg, _ptr(view.final_T), _ptr(view.n_contrib), _ptr(view.dL_dimage), grad2d.struct(),
                              _ptr(counts), _stream())


def project_bwd(g: Gaussians, view: View, proj: Projected, grad2d: Grad2D, grads: Gaussians,
                densify_accum: torch.Tensor = None, densify_count: torch.Tensor = None,
                radius: torch.Tensor = None, densify_max_radius: torch.Tensor = None):
    abi.gs_project_bwd(g.params(), view.gcam, proj.struct(radius), grad2d.struct(), grads.grads(),
                       _ptr(densify_accum), _ptr(densify_count), _ptr(densify_max_radius), _stream())


def l1_loss_grad(view: View, target: torch.Tensor, loss_dev: torch.Tensor):
    abi.gs_l1_loss_grad(_ptr(view.image), _ptr(target), view.image.numel(), _ptr(view.dL_dimage), _ptr(loss_dev),
                        _stream())


def l1_dssim_loss_grad(view: View, target: torch.Tensor, loss_dev: torch.Tensor, l1_weight: float = 1.0,
                       ssim_weight: float = 0.2):
    """loss += l1_weight L1 + ssim_weight (1 - SSIM) of the view's image against target, and
    dL/dimage into the view (gsplat guide §4.1); the view keeps the SSIM workspace."""
    H, W = view.image.shape[0], view.image.shape[1]
    nbytes = abi.gs_l1_dssim_workspace_bytes(W, H)
    if getattr(view, "ssim_workspace", None) is None or view.ssim_workspace.numel() < nbytes:
        view.ssim_workspace = torch.empty((nbytes,), device=view.image.device, dtype=torch.uint8)
    abi.gs_l1_dssim_loss_grad(_ptr(view.image), _ptr(target), W, H, l1_weight, ssim_weight,
                              _ptr(view.ssim_workspace), view.ssim_workspace.numel(), _ptr(view.dL_dimage),
                              _ptr(loss_dev), _stream())


def adam_step(g: Gaussians, grads: Gaussians, m: Gaussians, v: Gaussians, lrs: dict, step: int,
              betas=(0.9, 0.99), eps=1e-15):
    s = _stream()
    for name in PARAM_NAMES:
        p = getattr(g, name)
        abi.gs_adam(_ptr(p), _ptr(getattr(grads, name)), _ptr(getattr(m, name)), _ptr(getattr(v, name)), p.numel(),
                    lrs[name], betas[0], betas[1], eps, step, s)


def _grad_buffer(g: Gaussians, grads: Gaussians):
    """The gradient buffer of a backward + Adam call (the chain passes the step's gradient
    through it to the Adam launch): the caller's, else one kept beside the Gaussians."""
    if grads is not None:
        return grads.grads()
    buf = getattr(g, "_step_grads", None)
    if buf is None or buf.n != g.n or buf.sh_degree != g.sh_degree or buf.means.device != g.means.device:
        buf = g._step_grads = g.zeros_like()
    return buf.grads()


def project_bwd_views_adam(g: Gaussians, views: list, proj: Projected, radii: torch.Tensor, grad2ds: list,
                           m: Gaussians, v: Gaussians, lrs: dict, step: int, grads: Gaussians = None,
                           densify_accum: torch.Tensor = None, densify_count: torch.Tensor = None,
                           betas=(0.9, 0.99), eps=1e-15, densify_max_radius: torch.Tensor = None,
                           sparse: bool = False):
    """Backward through the projection for all views (each with its own radius row and 2D
    gradients) with the Adam step of all five groups fused in; sparse=True leaves Gaussians
    visible in no view untouched (the gsplat guide §4.1 sparse_grad option)."""
    abi.gs_project_bwd_views_adam(
        g.params(), [vw.gcam for vw in views], [proj.struct(radii[k]) for k in range(len(views))],
        [gd.struct() for gd in grad2ds], g.grads(), m.grads(), v.grads(), [lrs[k] for k in PARAM_NAMES],
        betas[0], betas[1], eps, step, _grad_buffer(g, grads), _ptr(densify_accum),
        _ptr(densify_count), _ptr(densify_max_radius), int(sparse), _stream())


def project_bwd_views_adam_sh16(g: Gaussians, sh_half: torch.Tensor, views: list, proj: Projected,
                                radii: torch.Tensor, grad2ds: list, m: Gaussians, v: Gaussians, lrs: dict, step: int,
                                grads: Gaussians = None, densify_accum: torch.Tensor = None,
                                densify_count: torch.Tensor = None, betas=(0.9, 0.99), eps=1e-15,
                                densify_max_radius: torch.Tensor = None, sparse: bool = False):
    """project_bwd_views_adam for views projected from the 16-bit SH copy: the chain reads
    sh_half, Adam updates the float32 SH, and sh_half is refreshed from it in place."""
    abi.gs_project_bwd_views_adam_sh16(
        g.params(), [vw.gcam for vw in views], [proj.struct(radii[k]) for k in range(len(views))],
        [gd.struct() for gd in grad2ds], _ptr(sh_half), _ptr(sh_half), g.grads(), m.grads(), v.grads(),
        [lrs[k] for k in PARAM_NAMES], betas[0], betas[1], eps, step, _grad_buffer(g, grads),
        _ptr(densify_accum), _ptr(densify_count), _ptr(densify_max_radius), int(sparse), _stream())


def project_bwd_views_adam_packed(g: Gaussians, views: list, packs: list, grad2ds: list, m: Gaussians, v: Gaussians,
                                  lrs: dict, step: int, grads: Gaussians = None, densify_accum: torch.Tensor = None,
                                  densify_count: torch.Tensor = None, betas=(0.9, 0.99), eps=1e-15,
                                  densify_max_radius: torch.Tensor = None, sparse: bool = False):
    """project_bwd_views_adam for views in the packed layout (packs[k]: view k's Packed)."""
    abi.gs_project_bwd_views_adam_packed(
        g.params(), [vw.gcam for vw in views], [pk.proj.struct() for pk in packs], [_ptr(pk.slot_of) for pk in packs],
        [gd.struct() for gd in grad2ds], g.grads(), m.grads(), v.grads(), [lrs[k] for k in PARAM_NAMES], betas[0],
        betas[1], eps, step, _grad_buffer(g, grads), _ptr(densify_accum), _ptr(densify_count),
        _ptr(densify_max_radius), int(sparse), _stream())


# densify_and_prune parameters of the gsplat guide §4.1 (every 100 steps): gradient
# threshold, minimum opacity, extent (read as the largest scale, in world units,
# up to which a densified Gaussian is cloned rather than split) and maximum screen
# size (read as a fraction of the image's larger side).
DENSIFY_DEFAULTS = {"grad_threshold": 0.0002, "min_opacity": 0.005, "extent": 0.01, "max_screen_size": 0.02}


def densify_config(width: int, height: int, grad_threshold=0.0002, min_opacity=0.005, extent=0.01,
                   max_screen_size=0.02) -> abi.gs_densify_config:
    return abi.gs_densify_config(grad_threshold, extent, min_opacity,
                                 int(max_screen_size * max(width, height)) if max_screen_size > 0 else 0)


def densify(g: Gaussians, accum: torch.Tensor, count: torch.Tensor, max_radius: torch.Tensor, noise: torch.Tensor,
            cfg: abi.gs_densify_config, m: Gaussians = None, v: Gaussians = None):
    """Prune / clone / split (gs_densify_plan, one wait for the output count, gs_densify_apply).
    noise: [n, 6] float32 N(0, 1) draws for the split children.  Returns the new Gaussians,
    the carried moments (None without m, v) and the per-Gaussian decisions."""
    s = _stream()
    dev = g.means.device
    ws_bytes = abi.gs_densify_workspace_bytes(g.n)
    ws = torch.empty((ws_bytes,), device=dev, dtype=torch.uint8)
    decision = torch.empty((max(g.n, 1),), device=dev, dtype=torch.uint8)
    num_out = torch.zeros((1,), device=dev, dtype=torch.int64)
    abi.gs_densify_plan(g.params(), _ptr(accum), _ptr(count), _ptr(max_radius), cfg, _ptr(ws), ws_bytes,
                        _ptr(decision), _ptr(num_out), s)
    n_out = int(num_out.item())
    out = Gaussians(n_out, g.sh_degree, dev)
    om = ov = None
    if m is not None:
        om = Gaussians(n_out, g.sh_degree, dev)
        ov = Gaussians(n_out, g.sh_degree, dev)
    abi.gs_densify_apply(g.params(), m.params() if m is not None else None, v.params() if v is not None else None,
                         _ptr(noise), _ptr(decision), _ptr(ws), ws_bytes, n_out, out.grads(),
                         om.grads() if om is not None else None, ov.grads() if ov is not None else None, s)
    return out, om, ov, decision[:g.n]


@dataclass
class Trainer:
    """One or several views of L1 (or L1 + D-SSIM) training with Adam (the training loop of the
    gsplat guide §4.1-4.2), optionally accumulating the densification statistics.

    fused=True (default, up to GS_MAX_VIEWS views): every view keeps its own 2D
    gradients and visibility, and one pass chains all views back to the parameters
    and applies Adam.  fused=False: per view project_bwd into a gradient buffer,
    then gs_adam per parameter group."""
    gauss: Gaussians
    views: list
    targets: list
    lrs: dict
    bg: tuple = (0.0, 0.0, 0.0)
    densify: bool = False
    fused: bool = True
    ssim_weight: float = 0.0   # > 0: L1 + ssim_weight * (1 - SSIM) (the gsplat guide §4.1 uses 0.2)
    absgrad: bool = False      # densify on the absolute 2D gradient (the gsplat guide §4.1 absgrad option)
    sparse_grad: bool = False  # Adam skips Gaussians seen in no view of the step (sparse_grad option; fused only)
    streams: int = 3           # fused path: views alternate over this many CUDA streams, so that one
                               # view's sort overlaps another view's compositing
    batched_sort: bool = True  # fused path: project every view first and sort all views by depth in one
                               # batched sort (gs_depth_order_views), then bin and composite per view
    groups: int = 1            # fused batched path: the views are projected, depth-sorted and binned in
                               # this many consecutive groups, so that a group's projection and depth sort
                               # overlap the compositing of the groups before it (slower on the 16-view
                               # 1080p step: compositing already fills the device, and the overlap only
                               # adds launches)
    packed: bool = False       # fused batched path: views in the packed layout (gs_project_packed, the
                               # gsplat guide §4.1 packed option); the slot capacity follows the largest
                               # visible count seen
    sh16: bool = False         # fused unpacked path: the projections read a 16-bit (FP16) copy of the SH
                               # coefficients, which the fused Adam step refreshes from the float32 ones
    bin_views: bool = True     # fused batched path: each view group's binning (emission, passes by tile,
                               # ranges) launched once for all its views instead of once per view
    tile_cull: bool = True     # every view bins a Gaussian only into the tiles of its rectangle where its
                               # alpha can reach 1/255 (gs_camera.tile_cull): the same images and gradients
                               # from about half the instances of the 3-sigma rectangles
    graph: bool = False        # fused path: the views' part of a step (projections, sorts, compositing,
                               # losses and their backward) is captured once into a CUDA graph and
                               # replayed every step, so its few-microsecond launches cost no host time
                               # and little device time between them; recaptured whenever a buffer it
                               # uses is reallocated (instance or slot growth, densification); the
                               # cameras and target tensors are those seen at capture, so after
                               # View.set_camera or new targets call drop_graph()

    def __post_init__(self):
        n = self.gauss.n
        dev = self.gauss.means.device
        self.fused = self.fused and len(self.views) <= abi.GS_MAX_VIEWS
        for vw in self.views:
            vw.set_tile_cull(self.tile_cull)
        if self.packed and not (self.fused and self.batched_sort):
            raise ValueError("packed=True runs on the fused path with the batched sort")
        if self.sh16 and (self.packed or not self.fused):
            raise ValueError("sh16=True runs on the fused path with unpacked views")
        # per view: instance count and (packed) visible count, read back with one wait per step
        self.counts = torch.zeros((2, len(self.views)), device=dev, dtype=torch.int64)
        self.kcount = self.counts[0]
        self._alloc_per_gaussian(n)
        self.m = self.gauss.zeros_like()
        self.v = self.gauss.zeros_like()
        self.loss = torch.zeros((1,), device=dev, dtype=torch.float64)
        self.step_count = 0
        self.noise_gen = torch.Generator(device=dev)
        self.noise_gen.manual_seed(0)

    def _alloc_per_gaussian(self, n: int):
        """Buffers sized by the Gaussian count (the projection, 2D gradients, visibility rows,
        gradients and densification statistics)."""
        self._graph = None  # it holds the old buffers' addresses
        dev = self.gauss.means.device
        nv = len(self.views) if self.fused else 1
        if self.packed:
            self.pack_ws = project_packed_workspace(n, dev)
            self.radii = None
            self._alloc_packed(n)
        else:
            self.proj = Projected(n, dev)
            # concurrent views need their own projected features
            if self.fused and self.batched_sort:
                # every view's projection is kept until its binning
                self.projs = [self.proj] + [Projected(n, dev) for _ in range(nv - 1)]
                self._alloc_orders(n)
            else:
                self.projs = [self.proj] + [Projected(n, dev) for _ in range(min(self.streams, nv) - 1)] \
                    if self.fused else [self.proj]
                self.depth_orders = None
            self.grad2ds = [Grad2D(n, dev, absgrad=self.absgrad) for _ in range(nv)]
            self.grad2d = self.grad2ds[0]
            self.radii = torch.zeros((nv, max(n, 1)), device=dev, dtype=torch.int32)
        # the unfused path accumulates into it; the fused step passes its gradient through
        # it to the Adam launch
        self.grads = self.gauss.zeros_like()
        self.sh_half = to_half(self.gauss.sh) if self.sh16 else None
        self.densify_accum = torch.zeros((max(n, 1),), device=dev, dtype=torch.float32) if self.densify else None
        self.densify_count = torch.zeros((max(n, 1),), device=dev, dtype=torch.int32) if self.densify else None
        self.densify_max_radius = torch.zeros((max(n, 1),), device=dev, dtype=torch.int32) if self.densify else None

    def _alloc_packed(self, capacity: int):
        """Packed views of `capacity` slots: features, 2D gradients, depth order and sort buffers."""
        self._graph = None
        dev = self.gauss.means.device
        n, nv = self.gauss.n, len(self.views)
        self.pcap = int(capacity)
        self.packs = [Packed(n, self.pcap, dev, self.counts[1][k:k + 1]) for k in range(nv)]
        self.projs = [pk.proj for pk in self.packs]
        self.proj = self.projs[0]
        self._alloc_orders(self.pcap)
        self.grad2ds = [Grad2D(self.pcap, dev, absgrad=self.absgrad) for _ in range(nv)]
        self.grad2d = self.grad2ds[0]
        for view in self.views:
            view.set_n(self.pcap)

    def set_tile_cull(self, on: bool):
        """Switch every view between the culled binning and the rectangles; a captured
        CUDA graph holds the old camera flags and workspace addresses, so it is dropped
        and the next step captures again."""
        self.tile_cull = bool(on)
        for vw in self.views:
            vw.set_tile_cull(self.tile_cull)
        self.drop_graph()

    def drop_graph(self):
        """Forget the captured CUDA graph (graph=True): the next step captures the views'
        part again with the current cameras, targets and buffers."""
        self._graph = None

    def view_groups(self) -> list:
        """The consecutive groups of view indices the batched path projects, sorts and bins together."""
        nv = len(self.views)
        size = -(-nv // max(1, min(self.groups, nv)))
        return [list(range(i, min(i + size, nv))) for i in range(0, nv, size)]

    def _alloc_orders(self, n: int):
        """One batched depth order (and its workspace) per view group, over n entries."""
        dev = self.gauss.means.device
        groups = self.view_groups()
        self.depth_orders = [DepthOrder(n, len(ks), dev) for ks in groups]
        self._order_at = {k: (gi, j) for gi, ks in enumerate(groups) for j, k in enumerate(ks)}

    def order_row(self, k: int) -> torch.Tensor:
        """View k's depth order (a row of its group's DepthOrder)."""
        gi, j = self._order_at[k]
        return self.depth_orders[gi].order[j]

    def _project(self, view: View, proj: Projected, radius: torch.Tensor):
        if self.sh16:
            project_sh16(self.gauss, self.sh_half, view, proj, radius)
        else:
            project(self.gauss, view, proj, radius)

    def _radius(self, k: int):
        """View k's radius row (None: the packed projection's own)."""
        return None if self.packed else self.radii[k if self.fused else 0]

    def densify_and_prune(self, **kw) -> torch.Tensor:
        """Adaptive density control from the statistics accumulated since the last call
        (thresholds as in DENSIFY_DEFAULTS, overridable by keyword; the screen limit is a
        fraction of the first view's larger side).  Parameters and Adam moments are
        compacted into new arrays, every per-Gaussian buffer is resized and the
        statistics restart from zero.  Returns the per-Gaussian decisions."""
        if not self.densify:
            raise RuntimeError("Trainer(densify=True) accumulates the statistics densification needs")
        p = dict(DENSIFY_DEFAULTS)
        p.update(kw)
        cam = self.views[0].cam
        cfg = densify_config(cam["width"], cam["height"], **p)
        noise = torch.randn((max(self.gauss.n, 1), 6), device=self.gauss.means.device, dtype=torch.float32,
                            generator=self.noise_gen)
        g, m, v, decision = densify(self.gauss, self.densify_accum, self.densify_count, self.densify_max_radius,
                                    noise, cfg, self.m, self.v)
        self.gauss, self.m, self.v = g, m, v
        for view in self.views:
            view.set_n(g.n)
        self._alloc_per_gaussian(g.n)
        return decision

    def view_forward_backward(self, k: int, target: torch.Tensor, proj: Projected = None,
                              projected: bool = False) -> None:
        """project -> sort -> raster forward -> L1 -> raster backward of view k (on the
        current stream).  The fused path sorts without waiting (instance count checked
        once per step); with `projected` the view was projected and depth-ordered
        already (the batched sort) and only the binning from that order runs here."""
        view = self.views[k]
        proj = self.proj if proj is None else proj
        r = self.radii[k if self.fused else 0]
        g2 = self.grad2ds[k if self.fused else 0]
        if projected:
            bin_sort_ordered_async(proj, view, self.order_row(k), self.kcount[k:k + 1], r)
        else:
            self._project(view, proj, r)
            if self.fused:
                bin_sort_async(proj, view, self.kcount[k:k + 1], r)
            else:
                bin_sort(proj, view, r)
        if self.ssim_weight > 0.0:
            raster_fwd(proj, view, self.bg, r)
            l1_dssim_loss_grad(view, target, self.loss, 1.0, self.ssim_weight)
        else:
            raster_fwd_l1(proj, view, target, self.loss, self.bg, r)
        g2.zero_()
        raster_bwd(proj, view, g2, self.bg, radius=r)

    def _all_views(self, targets=None, ready=None, after_view=None) -> None:
        """Every view's forward and backward; in the fused path view k runs on stream
        k mod `streams`, joined before return.  targets: per-view target images
        (default self.targets); ready: per-view CUDA events view k's compositing waits
        for (e.g. the copy of its target); after_view(k, event): called once view k
        is enqueued, with an event recorded after it."""
        targets = self.targets if targets is None else targets
        if not self.fused or (self.depth_orders is None and len(self.projs) == 1):
            for k, tgt in enumerate(targets):
                if ready is not None:
                    torch.cuda.current_stream().wait_event(ready[k])
                self.view_forward_backward(k, tgt)
                if after_view is not None:
                    after_view(k, torch.cuda.current_stream().record_event())
            return
        main = torch.cuda.current_stream()
        side = self.side_streams()
        batched = self.depth_orders is not None
        if batched:
            # binning of every view on a high-priority stream: its small, latency-bound
            # kernels take SM slots as soon as compositing blocks retire, instead of
            # queueing behind whole compositing launches
            bin_stream = self.bin_stream()
            for gi, ks in enumerate(self.view_groups()):
                # this group's projections and depth sort on the current stream run while
                # the groups before it composite
                self.project_and_order(gi)
                bin_stream.wait_stream(main)
                binned = {}
                with torch.cuda.stream(bin_stream):
                    sizes = {(self.views[k].cam["width"], self.views[k].cam["height"]) for k in ks}
                    if self.bin_views and not self.packed and len(sizes) == 1:
                        bin_sort_ordered_views_async([self.projs[k] for k in ks], [self.views[k] for k in ks],
                                                     self.depth_orders[gi], self.kcount[ks[0]:ks[-1] + 1],
                                                     [self._radius(k) for k in ks])
                        done = bin_stream.record_event()
                        binned = {k: done for k in ks}
                    else:
                        for k in ks:
                            bin_sort_ordered_async(self.projs[k], self.views[k], self.order_row(k),
                                                   self.kcount[k:k + 1], self._radius(k))
                            binned[k] = bin_stream.record_event()
                for k in ks:
                    st = side[k % len(side)]
                    st.wait_event(binned[k])
                    if ready is not None:
                        st.wait_event(ready[k])
                    with torch.cuda.stream(st):
                        self.view_composite(k, targets[k], self.projs[k])
                    if after_view is not None:
                        after_view(k, st.record_event())
            for st in side + [bin_stream]:
                main.wait_stream(st)
            return
        start = main.record_event()
        for st in side:
            st.wait_event(start)
        for k, tgt in enumerate(targets):
            j = k % len(side)
            if ready is not None:
                side[j].wait_event(ready[k])
            with torch.cuda.stream(side[j]):
                self.view_forward_backward(k, tgt, self.projs[j])
            if after_view is not None:
                after_view(k, side[j].record_event())
        for st in side:
            main.wait_stream(st)

    def view_composite(self, k: int, target: torch.Tensor, proj: Projected) -> None:
        """raster forward -> loss -> raster backward of an already binned view k."""
        view = self.views[k]
        r = self._radius(k)
        if self.ssim_weight > 0.0:
            raster_fwd(proj, view, self.bg, r)
            l1_dssim_loss_grad(view, target, self.loss, 1.0, self.ssim_weight)
        else:
            raster_fwd_l1(proj, view, target, self.loss, self.bg, r)
        self.grad2ds[k].zero_()
        raster_bwd(proj, view, self.grad2ds[k], self.bg, radius=r)

    def bin_stream(self) -> torch.cuda.Stream:
        """The high-priority stream the batched path bins every view on."""
        if getattr(self, "_bin_stream", None) is None:
            hi = torch.cuda.Stream.priority_range()[1] if hasattr(torch.cuda.Stream, "priority_range") else -1
            self._bin_stream = torch.cuda.Stream(device=self.gauss.means.device, priority=hi)
        return self._bin_stream

    def project_and_order(self, group: int = None) -> None:
        """The projection of every view of a view group (packed or not), then the batched
        depth sort of the group (current stream); every group when group is None."""
        groups = self.view_groups()
        for gi in range(len(groups)) if group is None else [group]:
            ks = groups[gi]
            if self.packed:
                for k in ks:
                    project_packed(self.gauss, self.views[k], self.packs[k], self.pack_ws)
            else:
                # every view of the group in one launch (the parameters are read once)
                project_views(self.gauss, [self.views[k] for k in ks], [self.projs[k] for k in ks],
                              [self.radii[k] for k in ks], self.sh_half if self.sh16 else None)
            depth_order_views([self.projs[k] for k in ks], None if self.radii is None else [self.radii[k] for k in ks],
                              self.depth_orders[gi])

    def _views_part(self) -> None:
        abi.gs_zero(_ptr(self.loss), 8, _stream())
        self._all_views()

    def _replay_views(self) -> None:
        """The views' part of the step from the CUDA graph, captured first when there is none."""
        if getattr(self, "_graph", None) is None:
            self.side_streams()  # the streams exist before the capture forks onto them
            self.bin_stream()
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                self._views_part()
            self._graph = graph
        self._graph.replay()

    def side_streams(self) -> list:
        """The streams the fused path runs views on."""
        if getattr(self, "_side", None) is None:
            count = min(self.streams, len(self.views))
            self._side = [torch.cuda.Stream(device=self.gauss.means.device) for _ in range(count)]
        return self._side

    def step(self) -> None:
        """forward + L1 + backward for every view, then one Adam step; loss stays on the device."""
        s = _stream()
        while True:
            if self.fused and self.graph:
                self._replay_views()
            else:
                abi.gs_zero(_ptr(self.loss), 8, s)
            if not self.fused:
                self.grads.zero_()
                for k, tgt in enumerate(self.targets):
                    self.view_forward_backward(k, tgt)
                    project_bwd(self.gauss, self.views[k], self.proj, self.grad2d, self.grads, self.densify_accum,
                                self.densify_count, radius=self.radii[0], densify_max_radius=self.densify_max_radius)
                break
            if not self.graph:
                self._all_views()
            # one wait per step: every view's instance count against its capacity (and in the
            # packed layout its visible count against the slot capacity)
            both = self.counts.cpu().tolist()
            counts, visible = both[0], both[1]
            if self.packed and max(visible) > self.pcap:
                # some view kept more Gaussians than there are slots: more slots, repeat the step
                self._alloc_packed(min(self.gauss.n, int(max(visible) * 1.25) + 1024))
                continue
            over = [k for k, K in enumerate(counts) if K > self.views[k].capacity]
            for k, K in enumerate(counts):
                self.views[k].num_instances = K
            if not over:
                break
            for k in over:  # grow and repeat the step's views (nothing was applied yet)
                self.views[k]._alloc(int(counts[k] * 1.25) + 1024)
                self._graph = None
        self.step_count += 1
        if self.packed:
            project_bwd_views_adam_packed(self.gauss, self.views, self.packs, self.grad2ds, self.m, self.v, self.lrs,
                                          self.step_count, self.grads, self.densify_accum, self.densify_count,
                                          densify_max_radius=self.densify_max_radius, sparse=self.sparse_grad)
            # far more slots than Gaussians kept (the first step starts with n): fewer slots from
            # the next step on
            if self.pcap > 1.5 * max(visible) + 4096:
                self._alloc_packed(min(self.gauss.n, int(max(visible) * 1.25) + 1024))
        elif self.sh16:
            project_bwd_views_adam_sh16(self.gauss, self.sh_half, self.views, self.proj, self.radii, self.grad2ds,
                                        self.m, self.v, self.lrs, self.step_count, self.grads, self.densify_accum,
                                        self.densify_count, densify_max_radius=self.densify_max_radius,
                                        sparse=self.sparse_grad)
        elif self.fused:
            project_bwd_views_adam(self.gauss, self.views, self.proj, self.radii, self.grad2ds, self.m, self.v,
                                   self.lrs, self.step_count, self.grads, self.densify_accum, self.densify_count,
                                   densify_max_radius=self.densify_max_radius, sparse=self.sparse_grad)
        else:
            adam_step(self.gauss, self.grads, self.m, self.v, self.lrs, self.step_count)
