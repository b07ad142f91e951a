"""CPU oracle of the differentiable Gaussian-splatting tile rasterizer.

TEST INFRASTRUCTURE ONLY: imported by tests/, by the smoke check and by the
benchmark's CPU-baseline leg.  The product path (the CUDA library and its
binding) never imports it.  The arithmetic lives in oracle.cpp, which this
module calls through ctypes, except for a few short numpy formulas written
out here (the L1 + D-SSIM combination, the tile-reach bound of the culled
binning).

Parity status: every function here is pinned by tests/test_oracle_*.py against
closed forms, invariants, brute force, a library routine (scipy's spherical
harmonics) or central finite differences.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

from .build import LIB, build

_lib = None

_f32p = np.ctypeslib.ndpointer(np.float32, flags="C_CONTIGUOUS")
_f64p = np.ctypeslib.ndpointer(np.float64, flags="C_CONTIGUOUS")
_i32p = np.ctypeslib.ndpointer(np.int32, flags="C_CONTIGUOUS")
_u32p = np.ctypeslib.ndpointer(np.uint32, flags="C_CONTIGUOUS")
_u64p = np.ctypeslib.ndpointer(np.uint64, flags="C_CONTIGUOUS")
_u8p = np.ctypeslib.ndpointer(np.uint8, flags="C_CONTIGUOUS")
_vp = C.c_void_p


class OrcCamera(C.Structure):
    _fields_ = [("R", C.c_double * 9), ("t", C.c_double * 3), ("fx", C.c_double), ("fy", C.c_double),
                ("cx", C.c_double), ("cy", C.c_double), ("near_plane", C.c_double), ("eps2d", C.c_double),
                ("width", C.c_int32), ("height", C.c_int32)]


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB):
            build()
        L = C.CDLL(LIB)
        L.orc_project.argtypes = [C.c_int64, _f64p, _f64p, _f64p, _f64p, _f64p, C.c_int, C.POINTER(OrcCamera),
                                  C.c_int, _vp, C.c_int64, _f64p, _f64p, _f64p, _f64p, _f64p, _i32p, _i32p, _u32p]
        L.orc_keys.argtypes = [C.c_int64, _f64p, _i32p, _i32p, C.c_int, C.c_int, C.c_int64, _u64p, _u32p, _u32p]
        L.orc_keys.restype = C.c_int64
        L.orc_render.argtypes = [C.c_int64, _f64p, _f64p, _f64p, _f64p, _f64p, _i32p, _i32p, C.POINTER(OrcCamera),
                                 _f64p, C.c_int64, _vp, C.c_double, C.c_double, _f64p, _f64p, _i32p, _u8p]
        L.orc_render_bwd.argtypes = [C.c_int64, _f64p, _f64p, _f64p, _f64p, _f64p, _i32p, _i32p,
                                     C.POINTER(OrcCamera), _f64p, C.c_int64, _vp, _f64p, C.c_double, C.c_double,
                                     _f64p, _f64p, _u8p, _vp]
        L.orc_project_bwd.argtypes = [C.c_int64, _f64p, _f64p, _f64p, _f64p, _f64p, C.c_int, C.POINTER(OrcCamera),
                                      _vp, C.c_int64, _f64p, _f64p, _f64p, _f64p, _f64p, _f64p, _vp, _vp]
        L.orc_adam.argtypes = [C.c_int64, _f32p, _f32p, _f32p, _f32p, C.c_double, C.c_double, C.c_double,
                               C.c_double, C.c_int]
        L.orc_l1.argtypes = [C.c_int64, _f32p, _f32p, _f32p]
        L.orc_l1.restype = C.c_double
        L.orc_sh_basis.argtypes = [C.c_int64, _f64p, C.c_int, _f64p]
        L.orc_densify.argtypes = [C.c_int64, C.c_int, _f64p, _f64p, _f64p, _f64p, _f64p, _f64p, _i32p, _i32p,
                                  _f64p, C.c_double, C.c_double, C.c_double, C.c_int32, _u8p,
                                  np.ctypeslib.ndpointer(np.int64, flags="C_CONTIGUOUS"), _u8p, _f64p, _f64p, _f64p,
                                  _f64p, _f64p]
        L.orc_densify.restype = C.c_int64
        L.orc_ssim.argtypes = [C.c_int, C.c_int, C.c_int, _f64p, _f64p, _vp, _vp]
        L.orc_ssim.restype = C.c_double
        L.orc_set_threads.argtypes = [C.c_int]
        L.orc_set_threads.restype = C.c_int
        _lib = L
    return _lib


def set_threads(t: int = 0) -> int:
    """Set the OpenMP thread count (0 = leave as is); returns the count in use."""
    return lib().orc_set_threads(int(t))


def camera(cam: dict) -> OrcCamera:
    c = OrcCamera()
    R = np.asarray(cam["R"], np.float32).astype(np.float64).reshape(9)
    t = np.asarray(cam["t"], np.float32).astype(np.float64).reshape(3)
    for i in range(9):
        c.R[i] = R[i]
    for i in range(3):
        c.t[i] = t[i]
    for k in ("fx", "fy", "cx", "cy", "eps2d"):
        setattr(c, k, float(np.float32(cam[k])))
    c.near_plane = float(np.float32(cam["near"]))
    c.width = int(cam["width"])
    c.height = int(cam["height"])
    return c


def tiles(cam: dict):
    return (cam["width"] + 15) // 16, (cam["height"] + 15) // 16


def _c(a, dt):
    return np.ascontiguousarray(a, dtype=dt)


def _scene_arrays(scene):
    """Scene parameters widened to float64 (exact for float32 scenes)."""
    return (_c(scene.means, np.float64).reshape(-1), _c(scene.quats, np.float64).reshape(-1),
            _c(scene.log_scales, np.float64).reshape(-1), _c(scene.opacity_logits, np.float64).reshape(-1),
            _c(scene.sh, np.float64).reshape(-1))


def _idx(idx):
    if idx is None:
        return None, 0, None
    a = _c(idx, np.int64)
    return a.ctypes.data_as(_vp), len(a), a


def project(scene, cam: dict, quantize: bool = True, idx=None) -> dict:
    """Per-Gaussian projection; with quantize the outputs are float32 values (held in float64)."""
    n = scene.n
    ip, ni, keep = _idx(idx)
    m = ni if idx is not None else n
    out = {"xy": np.zeros((m, 2)), "depth": np.zeros(m), "conic": np.zeros((m, 3)), "opacity": np.zeros(m),
           "rgb": np.zeros((m, 3)), "radius": np.zeros(m, np.int32), "rect": np.zeros((m, 4), np.int32),
           "tiles_touched": np.zeros(m, np.uint32)}
    mu, q, ls, lo, sh = _scene_arrays(scene)
    oc = camera(cam)
    rc = lib().orc_project(n, mu, q, ls, lo, sh, scene.sh_degree, C.byref(oc), int(quantize), ip, ni,
                           out["xy"].reshape(-1), out["depth"], out["conic"].reshape(-1), out["opacity"],
                           out["rgb"].reshape(-1), out["radius"], out["rect"].reshape(-1), out["tiles_touched"])
    if rc != 0:
        raise ValueError("orc_project failed")
    return out


def keys(proj: dict, cam: dict):
    """Sorted (key, gid) instance list and per-tile [begin, end) ranges."""
    tx, ty = tiles(cam)
    n = len(proj["depth"])
    K = int(proj["tiles_touched"].astype(np.int64).sum())
    keys_ = np.zeros(max(K, 1), np.uint64)
    vals = np.zeros(max(K, 1), np.uint32)
    ranges = np.zeros(2 * tx * ty, np.uint32)
    got = lib().orc_keys(n, _c(proj["depth"], np.float64), _c(proj["rect"], np.int32).reshape(-1),
                         _c(proj["radius"], np.int32), tx, ty, K, keys_, vals, ranges)
    assert got == K, (got, K)
    return keys_[:K], vals[:K], ranges.reshape(-1, 2)


def render(proj: dict, cam: dict, bg=(0.0, 0.0, 0.0), pix=None, band_alpha=1e-5, band_T=1e-4):
    """Per-pixel composite.  Returns image [npix,3], final_T, n_contrib, ambiguous flags
    (for every pixel in row-major order when pix is None)."""
    n = len(proj["depth"])
    ip, ni, keep = _idx(pix)
    m = ni if pix is not None else cam["width"] * cam["height"]
    image = np.zeros((m, 3))
    fT = np.zeros(m)
    nc = np.zeros(m, np.int32)
    amb = np.zeros(m, np.uint8)
    oc = camera(cam)
    lib().orc_render(n, _c(proj["xy"], np.float64).reshape(-1), _c(proj["depth"], np.float64),
                     _c(proj["conic"], np.float64).reshape(-1), _c(proj["opacity"], np.float64),
                     _c(proj["rgb"], np.float64).reshape(-1), _c(proj["radius"], np.int32),
                     _c(proj["rect"], np.int32).reshape(-1), C.byref(oc), _c(bg, np.float64), ni, ip,
                     band_alpha, band_T, image.reshape(-1), fT, nc, amb)
    return image, fT, nc, amb


def render_bwd(proj: dict, cam: dict, dL_dpix, bg=(0.0, 0.0, 0.0), pix=None, band_alpha=1e-5, band_T=1e-4,
               straddle: bool = False):
    """Reverse compositing.  dL_dpix is [npix,3] for the listed pixels (or the
    whole image, row-major, when pix is None).  Returns grad2d [n,9]
    (u, v, A, B, C, o, r, g, b), the per-element sum of |terms|, and the
    touched-ambiguous flags [n]; with straddle=True also [n,9], the sum over the
    straddling decisions of |terms with the decision taken the other way - terms|."""
    n = len(proj["depth"])
    ip, ni, keep = _idx(pix)
    g2 = np.zeros((n, 9))
    g2a = np.zeros((n, 9))
    touched = np.zeros(n, np.uint8)
    st = np.zeros((n, 9)) if straddle else None
    oc = camera(cam)
    lib().orc_render_bwd(n, _c(proj["xy"], np.float64).reshape(-1), _c(proj["depth"], np.float64),
                         _c(proj["conic"], np.float64).reshape(-1), _c(proj["opacity"], np.float64),
                         _c(proj["rgb"], np.float64).reshape(-1), _c(proj["radius"], np.int32),
                         _c(proj["rect"], np.int32).reshape(-1), C.byref(oc), _c(bg, np.float64), ni, ip,
                         _c(dL_dpix, np.float64).reshape(-1), band_alpha, band_T, g2.reshape(-1),
                         g2a.reshape(-1), touched, None if st is None else st.ctypes.data_as(C.c_void_p))
    if straddle:
        return g2, g2a, touched, st
    return g2, g2a, touched


def project_bwd(scene, cam: dict, grad2d, idx=None, densify: bool = False) -> dict:
    """Parameter gradients from 2D gradients grad2d [m,9] (rows follow idx, or all n)."""
    n = scene.n
    ip, ni, keep = _idx(idx)
    m = ni if idx is not None else n
    nc = (scene.sh_degree + 1) ** 2
    out = {"means": np.zeros((m, 3)), "quats": np.zeros((m, 4)), "log_scales": np.zeros((m, 3)),
           "opacity_logits": np.zeros(m), "sh": np.zeros((m, nc, 3))}
    acc = np.zeros(m) if densify else None
    cnt = np.zeros(m, np.int32) if densify else None
    mu, q, ls, lo, sh = _scene_arrays(scene)
    oc = camera(cam)
    rc = lib().orc_project_bwd(n, mu, q, ls, lo, sh, scene.sh_degree, C.byref(oc), ip, ni,
                               _c(grad2d, np.float64).reshape(-1), out["means"].reshape(-1),
                               out["quats"].reshape(-1), out["log_scales"].reshape(-1), out["opacity_logits"],
                               out["sh"].reshape(-1), acc.ctypes.data_as(_vp) if densify else None,
                               cnt.ctypes.data_as(_vp) if densify else None)
    if rc != 0:
        raise ValueError("orc_project_bwd failed")
    if densify:
        out["densify_accum"] = acc
        out["densify_count"] = cnt
    return out


def adam(param, grad, m, v, lr, beta1, beta2, eps, step):
    """One Adam step; returns new (param, m, v) float32 arrays."""
    p = _c(param, np.float32).copy().reshape(-1)
    mm = _c(m, np.float32).copy().reshape(-1)
    vv = _c(v, np.float32).copy().reshape(-1)
    lib().orc_adam(p.size, p, _c(grad, np.float32).reshape(-1), mm, vv, lr, beta1, beta2, eps, int(step))
    shape = np.shape(param)
    return p.reshape(shape), mm.reshape(shape), vv.reshape(shape)


def l1(image, target):
    """(loss, dL/dimage) of mean |image - target|."""
    img = _c(image, np.float32).reshape(-1)
    tgt = _c(target, np.float32).reshape(-1)
    g = np.zeros_like(img)
    loss = lib().orc_l1(img.size, img, tgt, g)
    return loss, g.reshape(np.shape(image))


def sh_basis(dirs, deg: int):
    d = _c(dirs, np.float64).reshape(-1, 3)
    nc = (deg + 1) ** 2
    Y = np.zeros((len(d), nc))
    lib().orc_sh_basis(len(d), d.reshape(-1), deg, Y.reshape(-1))
    return Y


def densify(scene, accum, count, max_radius, noise, grad_threshold, scale_threshold, min_opacity,
            max_screen_radius, moments=(), quantize: bool = True) -> dict:
    """Adaptive density control of oracle.cpp's orc_densify.

    accum [n] float, count [n] int, max_radius [n] int, noise [n, 2, 3] (the N(0, I)
    draws of the two split children).  Thresholds are taken as given (pass float32
    values to decide in the same precision as a float32 configuration).  moments:
    optimizer-state arrays laid out like the parameters, a dict per state with the
    keys means, quats, log_scales, opacity_logits, sh; each is carried to the
    outputs (kept Gaussians keep theirs, new ones start at zero).  Returns the
    decision per input, source / fresh per output, the output scene arrays
    (float32 values when quantize) and the carried moments."""
    n = scene.n
    nc = (scene.sh_degree + 1) ** 2
    mu, q, ls, lo, sh = _scene_arrays(scene)
    cap = 2 * n
    out = {"means": np.zeros((cap, 3)), "quats": np.zeros((cap, 4)), "log_scales": np.zeros((cap, 3)),
           "opacity_logits": np.zeros(cap), "sh": np.zeros((cap, nc, 3))}
    decision = np.zeros(n, np.uint8)
    source = np.zeros(cap, np.int64)
    fresh = np.zeros(cap, np.uint8)
    k = lib().orc_densify(n, nc, mu, q, ls, lo, sh, _c(accum, np.float64), _c(count, np.int32),
                          _c(max_radius, np.int32), _c(noise, np.float64).reshape(-1), float(grad_threshold),
                          float(scale_threshold), float(min_opacity), int(max_screen_radius), decision, source, fresh,
                          out["means"].reshape(-1), out["quats"].reshape(-1), out["log_scales"].reshape(-1),
                          out["opacity_logits"], out["sh"].reshape(-1))
    res = {"decision": decision, "n_out": int(k), "source": source[:k], "fresh": fresh[:k].astype(bool)}
    for key, a in out.items():
        a = a[:k]
        res[key] = a.astype(np.float32).astype(np.float64) if quantize else a
    carried = []
    for mom in moments:
        c = {}
        for key, a in mom.items():
            a = np.asarray(a)
            o = a[res["source"]].copy()
            o[res["fresh"]] = 0
            c[key] = o
        carried.append(c)
    res["moments"] = carried
    return res


def ssim(x, y, want_map: bool = False, want_grad: bool = False):
    """Mean structural similarity of two [H, W, ch] images (11x11 Gaussian window,
    sigma 1.5, zero outside the image); optionally the per-pixel map and the
    gradient with respect to x.  Returns (ssim, map or None, grad or None)."""
    xa = _c(x, np.float64)
    ya = _c(y, np.float64)
    H, W, ch = xa.shape
    m = np.zeros_like(xa) if want_map else None
    g = np.zeros_like(xa) if want_grad else None
    v = lib().orc_ssim(H, W, ch, xa.reshape(-1), ya.reshape(-1), m.ctypes.data_as(_vp) if want_map else None,
                       g.ctypes.data_as(_vp) if want_grad else None)
    return v, m, g


def l1_dssim(image, target, l1_weight: float = 1.0, ssim_weight: float = 0.2):
    """loss = l1_weight * mean|image - target| + ssim_weight * (1 - ssim(image, target))
    and its gradient with respect to image (gsplat guide §4.1)."""
    img = _c(image, np.float64)
    tgt = _c(target, np.float64)
    n = img.size
    l1v = float(np.abs(img - tgt).mean())
    s, _, gs = ssim(img, tgt, want_grad=True)
    g = l1_weight * np.sign(img - tgt) / n - ssim_weight * gs
    return l1_weight * l1v + ssim_weight * (1.0 - s), g


def tile_min_sigma(xy, conic, tx, ty, widen: float = 0.0):
    """Smallest sigma = 1/2 (A dx^2 + C dy^2) + B dx dy (dx = x - u, dy = y - v) over the
    box of pixel centres of tile (tx, ty), [16 tx + 0.5 - widen, 16 tx + 15.5 + widen] in x
    and the same in y, for every row of xy [m, 2] and conic [m, 3] (A, B, C), in float64.

    For a positive definite form the minimum over the box is 0 when the mean lies in
    it; otherwise it lies on the box's boundary, and along an edge (one coordinate
    fixed) sigma is a parabola in the other coordinate, smallest at its vertex
    clamped to the edge.  Rows whose form is not positive definite get NaN."""
    xy = np.asarray(xy, np.float64).reshape(-1, 2)
    con = np.asarray(conic, np.float64).reshape(-1, 3)
    u, v = xy[:, 0], xy[:, 1]
    A, B, Cc = con[:, 0], con[:, 1], con[:, 2]
    x0 = 16.0 * np.asarray(tx, np.float64) + 0.5 - widen
    x1 = 16.0 * np.asarray(tx, np.float64) + 15.5 + widen
    y0 = 16.0 * np.asarray(ty, np.float64) + 0.5 - widen
    y1 = 16.0 * np.asarray(ty, np.float64) + 15.5 + widen
    pd = (A > 0) & (Cc > 0) & (A * Cc - B * B > 0)
    with np.errstate(divide="ignore", invalid="ignore"):
        def sig(dx, dy):
            return 0.5 * (A * dx * dx + Cc * dy * dy) + B * dx * dy
        best = np.full(len(u), np.inf)
        for xe in (x0, x1):   # x fixed: d sigma / d dy = B dx + C dy = 0
            dx = xe - u
            yc = np.clip(v - B * dx / Cc, y0, y1)
            best = np.minimum(best, sig(dx, yc - v))
        for ye in (y0, y1):   # y fixed: d sigma / d dx = A dx + B dy = 0
            dy = ye - v
            xc = np.clip(u - B * dy / A, x0, x1)
            best = np.minimum(best, sig(xc - u, dy))
    inside = (u >= x0) & (u <= x1) & (v >= y0) & (v <= y1)
    best = np.where(inside, 0.0, best)
    return np.where(pd, best, np.nan)


def tile_reach_classes(proj: dict, keys, vals, tiles_x: int):
    """For every instance (key, gid) of a rectangle binning (the list keys() returns):
    (must_keep, must_drop) under the tile culling rule, "bin a Gaussian into a tile of
    its rectangle only when its alpha = o e^-sigma can reach 1/255 somewhere in the
    tile's box of pixel centres".  must_keep: the box meets the region sigma <= ln(255 o);
    must_drop: even the box widened by 4/1024 px stays beyond sigma = ln(255 o) +
    3e-4 (|ln(255 o)| + 1).  Between the two a culled binning may go either way (its
    margins, and features 1 ulp apart).  A form that is clearly not positive definite
    (det < -1e-6 A C, or A or C <= 0) must keep the tile; one within 1e-6 of
    singular is left free."""
    gid = np.asarray(vals).astype(np.int64)
    tile = (np.asarray(keys).astype(np.uint64) >> np.uint64(32)).astype(np.int64)
    tx, ty = tile % tiles_x, tile // tiles_x
    xy = np.asarray(proj["xy"], np.float64)[gid]
    con = np.asarray(proj["conic"], np.float64)[gid]
    o = np.asarray(proj["opacity"], np.float64)[gid]
    A, B, Cc = con[:, 0], con[:, 1], con[:, 2]
    det = A * Cc - B * B
    clearly_pd = (A > 0) & (Cc > 0) & (det > 1e-6 * A * Cc)
    clearly_not = (A <= 0) | (Cc <= 0) | (det < -1e-6 * np.abs(A * Cc))
    with np.errstate(divide="ignore"):
        lnb = np.log(255.0 * o)
    m0 = tile_min_sigma(xy, con, tx, ty, 0.0)
    m1 = tile_min_sigma(xy, con, tx, ty, 4.0 / 1024.0)
    with np.errstate(invalid="ignore"):
        must_keep = clearly_not | (clearly_pd & (m0 <= lnb))
        bound = np.where(np.isfinite(lnb), lnb + 3e-4 * (np.abs(lnb) + 1.0), lnb)   # o = 0: -inf
        must_drop = clearly_pd & (m1 > bound)
    return must_keep, must_drop
