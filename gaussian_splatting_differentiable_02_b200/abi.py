"""ctypes binding of libgs.so: the C structures of include/gs.h and one Python
function per C entry point, with the same name and argument order.

Marshalling only.  Pointers are passed as integers (device addresses, e.g.
``tensor.data_ptr()``), streams as the integer handle of a cudaStream_t.  A
non-OK status raises ``GsError`` carrying gs_last_error_detail().  The library
must have been built (``python -m gaussian_splatting_differentiable_02_b200.build``
or ``__graft_entry__.build()``); a missing library is an error, never a fallback.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libgs.so")

GS_OK = 0
GS_ERR_INVALID_ARG = 1
GS_ERR_UNSUPPORTED = 2
GS_ERR_CAPACITY = 3
GS_ERR_CUDA = 4
GS_TILE = 16


class GsError(RuntimeError):
    def __init__(self, status: int, detail: str):
        super().__init__(f"status {status}: {detail}")
        self.status = status
        self.detail = detail


class gs_camera(C.Structure):
    _fields_ = [("R", C.c_float * 9), ("t", C.c_float * 3), ("fx", C.c_float), ("fy", C.c_float),
                ("cx", C.c_float), ("cy", C.c_float), ("width", C.c_int32), ("height", C.c_int32),
                ("near_plane", C.c_float), ("eps2d", C.c_float), ("tile_cull", C.c_int32)]


class gs_params(C.Structure):
    _fields_ = [("means", C.c_void_p), ("quats", C.c_void_p), ("log_scales", C.c_void_p),
                ("opacity_logits", C.c_void_p), ("sh", C.c_void_p), ("sh_degree", C.c_int32), ("n", C.c_int64)]


class gs_param_grads(C.Structure):
    _fields_ = [("means", C.c_void_p), ("quats", C.c_void_p), ("log_scales", C.c_void_p),
                ("opacity_logits", C.c_void_p), ("sh", C.c_void_p)]


class gs_projected(C.Structure):
    _fields_ = [("xy", C.c_void_p), ("depth", C.c_void_p), ("conic_opacity", C.c_void_p), ("rgb", C.c_void_p),
                ("radius", C.c_void_p), ("rect", C.c_void_p), ("tiles_touched", C.c_void_p)]


class gs_grad2d(C.Structure):
    _fields_ = [("xy", C.c_void_p), ("conic_opacity", C.c_void_p), ("rgb", C.c_void_p), ("xy_abs", C.c_void_p)]


class gs_densify_config(C.Structure):
    _fields_ = [("grad_threshold", C.c_float), ("scale_threshold", C.c_float), ("min_opacity", C.c_float),
                ("max_screen_radius", C.c_int32)]


GS_DENSIFY_PRUNE = 0
GS_DENSIFY_KEEP = 1
GS_DENSIFY_CLONE = 2
GS_DENSIFY_SPLIT = 3


# name -> (restype, argtypes), exactly the declarations of include/gs.h
_P = C.c_void_p
SIGNATURES = {
    "gs_status_string": (C.c_char_p, [C.c_int32]),
    "gs_last_error_detail": (C.c_char_p, []),
    "gs_sh_planes": (C.c_int32, [C.c_int32]),
    "gs_tile_grid": (C.c_int32, [C.POINTER(gs_camera), C.POINTER(C.c_int32), C.POINTER(C.c_int32)]),
    "gs_project": (C.c_int32, [C.POINTER(gs_params), C.POINTER(gs_camera), C.POINTER(gs_projected), _P]),
    "gs_bin_sort_workspace_bytes": (C.c_size_t, [C.c_int64, C.c_int64, C.POINTER(gs_camera)]),
    "gs_bin_sort": (C.c_int32, [C.POINTER(gs_projected), C.c_int64, C.POINTER(gs_camera), _P, C.c_size_t, _P, _P,
                                C.c_int64, C.POINTER(C.c_int64), _P, _P]),
    "gs_bin_sort_static": (C.c_int32, [C.POINTER(gs_projected), C.c_int64, C.POINTER(gs_camera), _P, _P, C.c_int64,
                                       C.POINTER(C.c_int64), _P, _P]),
    "gs_bin_sort_async": (C.c_int32, [C.POINTER(gs_projected), C.c_int64, C.POINTER(gs_camera), _P, C.c_size_t, _P, _P,
                                      C.c_int64, _P, _P, _P]),
    "gs_depth_order_workspace_bytes": (C.c_size_t, [C.c_int64, C.c_int32]),
    "gs_depth_order_views": (C.c_int32, [C.POINTER(gs_projected), C.c_int32, C.c_int64, _P, C.c_size_t, _P, _P]),
    "gs_bin_sort_ordered_async": (C.c_int32, [C.POINTER(gs_projected), C.c_int64, _P, C.POINTER(gs_camera), _P,
                                              C.c_size_t, _P, _P, C.c_int64, _P, _P, _P]),
    "gs_bin_sort_ordered_views_async": (C.c_int32, [C.POINTER(gs_projected), C.c_int32, C.c_int64, _P,
                                                    C.POINTER(gs_camera), C.POINTER(_P), C.POINTER(C.c_size_t),
                                                    C.POINTER(_P), C.POINTER(_P), C.POINTER(C.c_int64),
                                                    C.POINTER(_P), C.POINTER(_P), _P]),
    "gs_tile_order": (C.c_int32, [_P, C.POINTER(gs_camera), _P, _P]),
    "gs_tile_order_views": (C.c_int32, [C.c_int32, C.POINTER(_P), C.POINTER(gs_camera), C.POINTER(_P), _P]),
    "gs_raster_fwd": (C.c_int32, [C.POINTER(gs_projected), _P, _P, _P, C.POINTER(gs_camera), C.POINTER(C.c_float),
                                  _P, _P, _P, _P]),
    "gs_raster_fwd_l1": (C.c_int32, [C.POINTER(gs_projected), _P, _P, _P, C.POINTER(gs_camera),
                                     C.POINTER(C.c_float), _P, _P, _P, _P, _P, _P, _P]),
    "gs_raster_bwd": (C.c_int32, [C.POINTER(gs_projected), _P, _P, _P, C.POINTER(gs_camera), C.POINTER(C.c_float),
                                  _P, _P, _P, C.POINTER(gs_grad2d), _P]),
    "gs_project_bwd": (C.c_int32, [C.POINTER(gs_params), C.POINTER(gs_camera), C.POINTER(gs_projected),
                                   C.POINTER(gs_grad2d), C.POINTER(gs_param_grads), _P, _P, _P, _P]),
    "gs_project_bwd_views": (C.c_int32, [C.POINTER(gs_params), C.c_int32, C.POINTER(gs_camera),
                                         C.POINTER(gs_projected), C.POINTER(gs_grad2d), C.POINTER(gs_param_grads),
                                         _P, _P, _P, _P]),
    "gs_project_bwd_views_adam": (C.c_int32, [C.POINTER(gs_params), C.c_int32, C.POINTER(gs_camera),
                                              C.POINTER(gs_projected), C.POINTER(gs_grad2d),
                                              C.POINTER(gs_param_grads), C.POINTER(gs_param_grads),
                                              C.POINTER(gs_param_grads), C.POINTER(C.c_float), C.c_float, C.c_float,
                                              C.c_float, C.c_int32, C.POINTER(gs_param_grads), _P, _P, _P, C.c_int32,
                                              _P]),
    "gs_project_packed_workspace_bytes": (C.c_size_t, [C.c_int64]),
    "gs_project_packed": (C.c_int32, [C.POINTER(gs_params), C.POINTER(gs_camera), _P, C.c_size_t,
                                      C.POINTER(gs_projected), C.c_int64, _P, _P, _P, _P]),
    "gs_project_bwd_views_packed": (C.c_int32, [C.POINTER(gs_params), C.c_int32, C.POINTER(gs_camera),
                                                C.POINTER(gs_projected), C.POINTER(_P), C.POINTER(gs_grad2d),
                                                C.POINTER(gs_param_grads), _P, _P, _P, _P]),
    "gs_project_bwd_views_adam_packed": (C.c_int32, [C.POINTER(gs_params), C.c_int32, C.POINTER(gs_camera),
                                                     C.POINTER(gs_projected), C.POINTER(_P), C.POINTER(gs_grad2d),
                                                     C.POINTER(gs_param_grads), C.POINTER(gs_param_grads),
                                                     C.POINTER(gs_param_grads), C.POINTER(C.c_float), C.c_float,
                                                     C.c_float, C.c_float, C.c_int32, C.POINTER(gs_param_grads), _P,
                                                     _P, _P, C.c_int32, _P]),
    "gs_to_half": (C.c_int32, [_P, C.c_int64, _P, _P]),
    "gs_project_sh16": (C.c_int32, [C.POINTER(gs_params), _P, C.POINTER(gs_camera), C.POINTER(gs_projected), _P]),
    "gs_project_views": (C.c_int32, [C.POINTER(gs_params), C.c_int32, C.POINTER(gs_camera), C.POINTER(gs_projected),
                                     _P, _P]),
    "gs_project_bwd_views_adam_sh16": (C.c_int32, [C.POINTER(gs_params), C.c_int32, C.POINTER(gs_camera),
                                                   C.POINTER(gs_projected), C.POINTER(gs_grad2d), _P, _P,
                                                   C.POINTER(gs_param_grads), C.POINTER(gs_param_grads),
                                                   C.POINTER(gs_param_grads), C.POINTER(C.c_float), C.c_float,
                                                   C.c_float, C.c_float, C.c_int32, C.POINTER(gs_param_grads), _P,
                                                   _P, _P, C.c_int32, _P]),
    "gs_l1_dssim_workspace_bytes": (C.c_size_t, [C.c_int32, C.c_int32]),
    "gs_l1_dssim_loss_grad": (C.c_int32, [_P, _P, C.c_int32, C.c_int32, C.c_float, C.c_float, _P, C.c_size_t, _P, _P,
                                          _P]),
    "gs_densify_workspace_bytes": (C.c_size_t, [C.c_int64]),
    "gs_densify_plan": (C.c_int32, [C.POINTER(gs_params), _P, _P, _P, C.POINTER(gs_densify_config), _P, C.c_size_t,
                                    _P, _P, _P]),
    "gs_densify_apply": (C.c_int32, [C.POINTER(gs_params), C.POINTER(gs_params), C.POINTER(gs_params), _P, _P, _P,
                                     C.c_size_t, C.c_int64, C.POINTER(gs_param_grads), C.POINTER(gs_param_grads),
                                     C.POINTER(gs_param_grads), _P]),
    "gs_adam": (C.c_int32, [_P, _P, _P, _P, C.c_int64, C.c_float, C.c_float, C.c_float, C.c_float, C.c_int32, _P]),
    "gs_l1_loss_grad": (C.c_int32, [_P, _P, C.c_int64, _P, _P, _P]),
    "gs_zero": (C.c_int32, [_P, C.c_size_t, _P]),
    "gs_kernel_launches": (C.c_uint64, []),
    "gs_raster_fwd_counted": (C.c_int32, [C.POINTER(gs_projected), _P, _P, _P, C.POINTER(gs_camera),
                                          C.POINTER(C.c_float), _P, _P, _P, _P, _P]),
    "gs_raster_bwd_counted": (C.c_int32, [C.POINTER(gs_projected), _P, _P, _P, C.POINTER(gs_camera),
                                          C.POINTER(C.c_float), _P, _P, _P, C.POINTER(gs_grad2d), _P, _P]),
    "gs_alu_probe_slots": (C.c_int64, []),
    "gs_alu_probe": (C.c_int32, [C.c_int32, C.c_int64, _P, C.c_int64, C.POINTER(C.c_double), _P]),
}

_lib = None


def lib():
    """Load libgs.so (once).  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libgs.so not built ({LIB_PATH}); run the package's build.py")
        L = C.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _check(status: int):
    if status != GS_OK:
        raise GsError(status, lib().gs_last_error_detail().decode())
    return status


def make_camera(cam: dict, tile_cull: bool = False) -> gs_camera:
    """gs_camera from a scene camera dict (R 3x3 row-major, t, fx, fy, cx, cy, width, height, near, eps2d);
    tile_cull bins each Gaussian only into the tiles its footprint reaches."""
    c = gs_camera()
    R = [float(v) for v in np.asarray(cam["R"], np.float32).reshape(9)]
    t = [float(v) for v in np.asarray(cam["t"], np.float32).reshape(3)]
    for i in range(9):
        c.R[i] = R[i]
    for i in range(3):
        c.t[i] = t[i]
    c.fx, c.fy, c.cx, c.cy = cam["fx"], cam["fy"], cam["cx"], cam["cy"]
    c.width, c.height = int(cam["width"]), int(cam["height"])
    c.near_plane = cam.get("near", 0.2)
    c.eps2d = cam.get("eps2d", 0.3)
    c.tile_cull = int(tile_cull)
    return c


# ------------------------------------------------------------ entry points

def gs_status_string(status: int) -> str:
    return lib().gs_status_string(status).decode()


def gs_last_error_detail() -> str:
    return lib().gs_last_error_detail().decode()


def gs_sh_planes(sh_degree: int) -> int:
    return lib().gs_sh_planes(sh_degree)


def gs_tile_grid(cam: gs_camera):
    tx, ty = C.c_int32(), C.c_int32()
    _check(lib().gs_tile_grid(C.byref(cam), C.byref(tx), C.byref(ty)))
    return tx.value, ty.value


def gs_project(params: gs_params, cam: gs_camera, out: gs_projected, stream: int = 0):
    return _check(lib().gs_project(C.byref(params), C.byref(cam), C.byref(out), stream))


def gs_bin_sort_workspace_bytes(n: int, capacity: int, cam: gs_camera) -> int:
    return lib().gs_bin_sort_workspace_bytes(n, capacity, C.byref(cam))


def gs_bin_sort(proj: gs_projected, n: int, cam: gs_camera, workspace: int, workspace_bytes: int, keys: int,
                vals: int, capacity: int, tile_ranges: int, stream: int = 0, check: bool = True):
    """Returns (status, K).  With check=False a GS_ERR_CAPACITY status is returned, not raised."""
    K = C.c_int64(0)
    st = lib().gs_bin_sort(C.byref(proj), n, C.byref(cam), workspace, workspace_bytes, keys, vals, capacity,
                           C.byref(K), tile_ranges, stream)
    if check or st not in (GS_OK, GS_ERR_CAPACITY):
        _check(st)
    return st, K.value


def gs_bin_sort_async(proj: gs_projected, n: int, cam: gs_camera, workspace: int, workspace_bytes: int, keys: int,
                      vals: int, capacity: int, num_instances_dev: int, tile_ranges: int, stream: int = 0):
    """gs_bin_sort without a host wait: K goes to the device uint64 at num_instances_dev."""
    return _check(lib().gs_bin_sort_async(C.byref(proj), n, C.byref(cam), workspace, workspace_bytes, keys, vals,
                                          capacity, num_instances_dev, tile_ranges, stream))


GS_STATIC_SCRATCH_BYTES = 32 << 20


def gs_bin_sort_static(proj: gs_projected, n: int, cam: gs_camera, keys: int, vals: int, capacity: int,
                       tile_ranges: int, stream: int = 0, check: bool = True):
    """gs_bin_sort with the library's static scratch instead of a caller workspace
    (for callers that cannot allocate device memory).  Returns (status, K)."""
    K = C.c_int64(0)
    st = lib().gs_bin_sort_static(C.byref(proj), n, C.byref(cam), keys, vals, capacity, C.byref(K), tile_ranges,
                                  stream)
    if check or st not in (GS_OK, GS_ERR_CAPACITY):
        _check(st)
    return st, K.value


def gs_depth_order_workspace_bytes(n: int, num_views: int) -> int:
    return lib().gs_depth_order_workspace_bytes(n, num_views)


def gs_depth_order_views(projs, n: int, workspace: int, workspace_bytes: int, order: int, stream: int = 0):
    """projs: a sequence of gs_projected (one per view); order: device [views][n] uint32."""
    projs = list(projs)
    return _check(lib().gs_depth_order_views(_arr(gs_projected, projs), len(projs), n, workspace, workspace_bytes,
                                             order, stream))


def gs_bin_sort_ordered_async(proj: gs_projected, n: int, order: int, cam: gs_camera, workspace: int,
                              workspace_bytes: int, keys: int, vals: int, capacity: int, num_instances_dev: int,
                              tile_ranges: int, stream: int = 0):
    return _check(lib().gs_bin_sort_ordered_async(C.byref(proj), n, order or None, C.byref(cam), workspace,
                                                  workspace_bytes, keys, vals, capacity, num_instances_dev,
                                                  tile_ranges, stream))


def gs_bin_sort_ordered_views_async(projs, n: int, orders: int, cams, workspaces, workspace_bytes, keys, vals,
                                    capacities, num_instances_dev, tile_ranges, stream: int = 0):
    """projs, cams: sequences of gs_projected / gs_camera (one per view); orders: device
    pointer of the [views][n] depth orders; the rest: per-view device pointers and sizes."""
    V = len(projs)
    ptrs = lambda xs: (_P * V)(*[x or None for x in xs])
    return _check(lib().gs_bin_sort_ordered_views_async(
        _arr(gs_projected, projs), V, n, orders or None, _arr(gs_camera, cams), ptrs(workspaces),
        (C.c_size_t * V)(*workspace_bytes), ptrs(keys), ptrs(vals), (C.c_int64 * V)(*capacities),
        ptrs(num_instances_dev), ptrs(tile_ranges), stream))


def gs_tile_order_views(tile_ranges, cam: gs_camera, tile_orders, stream: int = 0):
    """tile_ranges, tile_orders: per-view device pointers."""
    V = len(tile_ranges)
    return _check(lib().gs_tile_order_views(V, (_P * V)(*tile_ranges), C.byref(cam), (_P * V)(*tile_orders), stream))


def gs_tile_order(tile_ranges: int, cam: gs_camera, tile_order: int, stream: int = 0):
    return _check(lib().gs_tile_order(tile_ranges, C.byref(cam), tile_order, stream))


def gs_raster_fwd(proj: gs_projected, vals: int, tile_ranges: int, tile_order: int, cam: gs_camera, bg, image: int,
                  final_T: int, n_contrib: int, stream: int = 0):
    """tile_order: device pointer from gs_tile_order, or 0 for the natural tile order."""
    b = (C.c_float * 3)(*[float(x) for x in bg])
    return _check(lib().gs_raster_fwd(C.byref(proj), vals, tile_ranges, tile_order or None, C.byref(cam), b, image,
                                      final_T, n_contrib, stream))


def gs_raster_fwd_l1(proj: gs_projected, vals: int, tile_ranges: int, tile_order: int, cam: gs_camera, bg, target: int,
                     image: int, final_T: int, n_contrib: int, dL_dimage: int, loss_dev: int, stream: int = 0):
    """gs_raster_fwd with the L1 term against target in the same kernel."""
    b = (C.c_float * 3)(*[float(x) for x in bg])
    return _check(lib().gs_raster_fwd_l1(C.byref(proj), vals, tile_ranges, tile_order or None, C.byref(cam), b, target,
                                         image, final_T, n_contrib, dL_dimage, loss_dev, stream))


def gs_raster_bwd(proj: gs_projected, vals: int, tile_ranges: int, tile_order: int, cam: gs_camera, bg, final_T: int,
                  n_contrib: int, dL_dimage: int, grad2d: gs_grad2d, stream: int = 0):
    b = (C.c_float * 3)(*[float(x) for x in bg])
    return _check(lib().gs_raster_bwd(C.byref(proj), vals, tile_ranges, tile_order or None, C.byref(cam), b,
                                      final_T, n_contrib, dL_dimage, C.byref(grad2d), stream))


def gs_raster_fwd_counted(proj: gs_projected, vals: int, tile_ranges: int, tile_order: int, cam: gs_camera, bg,
                          image: int, final_T: int, n_contrib: int, counts: int, stream: int = 0):
    """gs_raster_fwd that also adds its work counters to counts (4 uint64 on the device)."""
    b = (C.c_float * 3)(*[float(x) for x in bg])
    return _check(lib().gs_raster_fwd_counted(C.byref(proj), vals, tile_ranges, tile_order or None, C.byref(cam), b,
                                              image, final_T, n_contrib, counts, stream))


def gs_raster_bwd_counted(proj: gs_projected, vals: int, tile_ranges: int, tile_order: int, cam: gs_camera, bg,
                          final_T: int, n_contrib: int, dL_dimage: int, grad2d: gs_grad2d, counts: int,
                          stream: int = 0):
    """gs_raster_bwd that also adds its work counters to counts (4 uint64 on the device)."""
    b = (C.c_float * 3)(*[float(x) for x in bg])
    return _check(lib().gs_raster_bwd_counted(C.byref(proj), vals, tile_ranges, tile_order or None, C.byref(cam), b,
                                              final_T, n_contrib, dL_dimage, C.byref(grad2d), counts, stream))


GS_PROBE_FFMA, GS_PROBE_FFMA2, GS_PROBE_EX2, GS_PROBE_RCP = 0, 1, 2, 3


def gs_alu_probe_slots() -> int:
    return lib().gs_alu_probe_slots()


def gs_alu_probe(op: int, iters: int, out: int, out_count: int, stream: int = 0) -> float:
    """One throughput-probe launch; returns the operations it performs."""
    ops = C.c_double(0.0)
    _check(lib().gs_alu_probe(op, iters, out, out_count, C.byref(ops), stream))
    return ops.value


def gs_project_bwd(params: gs_params, cam: gs_camera, proj: gs_projected, grad2d: gs_grad2d, grads: gs_param_grads,
                   densify_accum: int = 0, densify_count: int = 0, densify_max_radius: int = 0, stream: int = 0):
    return _check(lib().gs_project_bwd(C.byref(params), C.byref(cam), C.byref(proj), C.byref(grad2d),
                                       C.byref(grads), densify_accum or None, densify_count or None,
                                       densify_max_radius or None, stream))


GS_MAX_VIEWS = 16
# views up to which the fused backward runs the chain and Adam in one kernel (grads optional)
GS_ADAM_ONE_PASS_MAX_VIEWS = 2


def _arr(ctype, items):
    items = list(items)
    a = (ctype * len(items))()
    for i, x in enumerate(items):
        a[i] = x
    return a


def gs_project_bwd_views(params: gs_params, cams, projs, grad2ds, grads: gs_param_grads, densify_accum: int = 0,
                         densify_count: int = 0, densify_max_radius: int = 0, stream: int = 0):
    """cams, projs, grad2ds: sequences of gs_camera / gs_projected / gs_grad2d (one per view)."""
    V = len(cams)
    return _check(lib().gs_project_bwd_views(C.byref(params), V, _arr(gs_camera, cams), _arr(gs_projected, projs),
                                             _arr(gs_grad2d, grad2ds), C.byref(grads), densify_accum or None,
                                             densify_count or None, densify_max_radius or None, stream))


def gs_project_bwd_views_adam(params: gs_params, cams, projs, grad2ds, params_inout: gs_param_grads,
                              adam_m: gs_param_grads, adam_v: gs_param_grads, lrs, beta1: float, beta2: float,
                              eps: float, step: int, grads: gs_param_grads = None, densify_accum: int = 0,
                              densify_count: int = 0, densify_max_radius: int = 0, sparse_adam: int = 0,
                              stream: int = 0):
    """Multi-view backward through the projection with the Adam step fused; lrs = 5 learning rates
    (means, quats, log_scales, opacity_logits, sh); sparse_adam = 1 skips Gaussians visible in no view."""
    V = len(cams)
    lr = (C.c_float * 5)(*[float(x) for x in lrs])
    return _check(lib().gs_project_bwd_views_adam(
        C.byref(params), V, _arr(gs_camera, cams), _arr(gs_projected, projs), _arr(gs_grad2d, grad2ds),
        C.byref(params_inout), C.byref(adam_m), C.byref(adam_v), lr, beta1, beta2, eps, step,
        C.byref(grads) if grads is not None else None, densify_accum or None, densify_count or None,
        densify_max_radius or None, int(sparse_adam), stream))


def gs_project_packed_workspace_bytes(n: int) -> int:
    return lib().gs_project_packed_workspace_bytes(n)


def gs_project_packed(params: gs_params, cam: gs_camera, workspace: int, workspace_bytes: int,
                      packed: gs_projected, capacity: int, gaussian_ids: int, slot_of: int, num_visible_dev: int,
                      stream: int = 0):
    """The packed projection: packed arrays of `capacity` slots, their Gaussian ids, the slot of every
    Gaussian, the visible count on the device."""
    return _check(lib().gs_project_packed(C.byref(params), C.byref(cam), workspace, workspace_bytes,
                                          C.byref(packed), capacity, gaussian_ids or None, slot_of or None,
                                          num_visible_dev, stream))


def _slots(slot_of):
    return _arr(_P, [int(p) for p in slot_of])


def gs_project_bwd_views_packed(params: gs_params, cams, projs, slot_of, grad2ds, grads: gs_param_grads,
                                densify_accum: int = 0, densify_count: int = 0, densify_max_radius: int = 0,
                                stream: int = 0):
    """gs_project_bwd_views for packed views; slot_of: one device pointer per view."""
    V = len(cams)
    return _check(lib().gs_project_bwd_views_packed(C.byref(params), V, _arr(gs_camera, cams),
                                                    _arr(gs_projected, projs), _slots(slot_of),
                                                    _arr(gs_grad2d, grad2ds), C.byref(grads), densify_accum or None,
                                                    densify_count or None, densify_max_radius or None, stream))


def gs_project_bwd_views_adam_packed(params: gs_params, cams, projs, slot_of, grad2ds, params_inout: gs_param_grads,
                                     adam_m: gs_param_grads, adam_v: gs_param_grads, lrs, beta1: float, beta2: float,
                                     eps: float, step: int, grads: gs_param_grads = None, densify_accum: int = 0,
                                     densify_count: int = 0, densify_max_radius: int = 0, sparse_adam: int = 0,
                                     stream: int = 0):
    """gs_project_bwd_views_adam for packed views; slot_of: one device pointer per view."""
    V = len(cams)
    lr = (C.c_float * 5)(*[float(x) for x in lrs])
    return _check(lib().gs_project_bwd_views_adam_packed(
        C.byref(params), V, _arr(gs_camera, cams), _arr(gs_projected, projs), _slots(slot_of),
        _arr(gs_grad2d, grad2ds), C.byref(params_inout), C.byref(adam_m), C.byref(adam_v), lr, beta1, beta2, eps,
        step, C.byref(grads) if grads is not None else None, densify_accum or None, densify_count or None,
        densify_max_radius or None, int(sparse_adam), stream))


def gs_to_half(x: int, count: int, out: int, stream: int = 0):
    """float32 -> IEEE half, round to nearest even (count values)."""
    return _check(lib().gs_to_half(x or None, count, out or None, stream))


def gs_project_views(params: gs_params, cams, outs, sh_half: int = 0, stream: int = 0):
    """gs_project of every view in cams into the matching gs_projected of outs, in one launch."""
    V = len(cams)
    return _check(lib().gs_project_views(C.byref(params), V, _arr(gs_camera, cams), _arr(gs_projected, outs),
                                         sh_half or None, stream))


def gs_project_sh16(params: gs_params, sh_half: int, cam: gs_camera, out: gs_projected, stream: int = 0):
    """gs_project with the SH coefficients read from a 16-bit copy."""
    return _check(lib().gs_project_sh16(C.byref(params), sh_half or None, C.byref(cam), C.byref(out), stream))


def gs_project_bwd_views_adam_sh16(params: gs_params, cams, projs, grad2ds, sh_half: int, sh_half_out: int,
                                   params_inout: gs_param_grads, adam_m: gs_param_grads, adam_v: gs_param_grads, lrs,
                                   beta1: float, beta2: float, eps: float, step: int, grads: gs_param_grads = None,
                                   densify_accum: int = 0, densify_count: int = 0, densify_max_radius: int = 0,
                                   sparse_adam: int = 0, stream: int = 0):
    """gs_project_bwd_views_adam for views projected from 16-bit SH; the updated SH is
    rounded into sh_half_out."""
    V = len(cams)
    lr = (C.c_float * 5)(*[float(x) for x in lrs])
    return _check(lib().gs_project_bwd_views_adam_sh16(
        C.byref(params), V, _arr(gs_camera, cams), _arr(gs_projected, projs), _arr(gs_grad2d, grad2ds),
        sh_half or None, sh_half_out or None, C.byref(params_inout), C.byref(adam_m), C.byref(adam_v), lr, beta1,
        beta2, eps, step, C.byref(grads) if grads is not None else None, densify_accum or None,
        densify_count or None, densify_max_radius or None, int(sparse_adam), stream))


def gs_l1_dssim_workspace_bytes(width: int, height: int) -> int:
    return lib().gs_l1_dssim_workspace_bytes(width, height)


def gs_l1_dssim_loss_grad(image: int, target: int, width: int, height: int, l1_weight: float, ssim_weight: float,
                          workspace: int, workspace_bytes: int, dL_dimage: int, loss_dev: int, stream: int = 0):
    return _check(lib().gs_l1_dssim_loss_grad(image, target, width, height, l1_weight, ssim_weight, workspace,
                                              workspace_bytes, dL_dimage, loss_dev, stream))


def gs_densify_workspace_bytes(n: int) -> int:
    return lib().gs_densify_workspace_bytes(n)


def gs_densify_plan(params: gs_params, densify_accum: int, densify_count: int, densify_max_radius: int,
                    cfg: gs_densify_config, workspace: int, workspace_bytes: int, decision: int, num_out_dev: int,
                    stream: int = 0):
    return _check(lib().gs_densify_plan(C.byref(params), densify_accum or None, densify_count or None,
                                        densify_max_radius or None, C.byref(cfg), workspace, workspace_bytes,
                                        decision or None, num_out_dev, stream))


def gs_densify_apply(params: gs_params, adam_m, adam_v, split_noise: int, decision: int, workspace: int,
                     workspace_bytes: int, n_out: int, out_params: gs_param_grads, out_m=None, out_v=None,
                     stream: int = 0):
    """adam_m / adam_v: gs_params of the moments or None; out_m / out_v: gs_param_grads or None."""
    ref = lambda x: C.byref(x) if x is not None else None  # noqa: E731
    return _check(lib().gs_densify_apply(C.byref(params), ref(adam_m), ref(adam_v), split_noise or None,
                                         decision or None, workspace, workspace_bytes, n_out, C.byref(out_params),
                                         ref(out_m), ref(out_v), stream))


def gs_adam(param: int, grad: int, m: int, v: int, count: int, lr: float, beta1: float, beta2: float, eps: float,
            step: int, stream: int = 0):
    return _check(lib().gs_adam(param, grad, m, v, count, lr, beta1, beta2, eps, step, stream))


def gs_l1_loss_grad(image: int, target: int, count: int, dL_dimage: int, loss_dev: int, stream: int = 0):
    return _check(lib().gs_l1_loss_grad(image, target, count, dL_dimage, loss_dev, stream))


def gs_kernel_launches() -> int:
    return lib().gs_kernel_launches()


def gs_zero(ptr: int, nbytes: int, stream: int = 0):
    return _check(lib().gs_zero(ptr, nbytes, stream))
