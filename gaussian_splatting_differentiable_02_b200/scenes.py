"""Seeded synthetic scenes, cameras and upstream signals for the five workloads.

This module only draws numbers and lays them out; it holds none of the
rasterizer's arithmetic, so both the CUDA path and the CPU oracle can take
their inputs from it without sharing any of the method.

Everything is a pure function of (workload, seed).  Arrays come out in the
natural "array of structures" layout (numpy, float32):

    means          [N, 3]
    quats          [N, 4]   (w, x, y, z), normalised draws of N(0, I4)
    log_scales     [N, 3]
    opacity_logits [N]
    sh             [N, (d+1)^2, 3]   coefficient-major, channel-minor

Cameras are dicts with a world-to-camera rotation ``R`` (3x3, row-major) and
translation ``t`` (x_cam = R x_world + t), OpenCV axes (x right, y down,
z forward), intrinsics fx, fy, cx, cy, the image size, the near plane and the
screen-space dilation.  Scene parameters are stored pre-activation (log-scale,
opacity logit, unit quaternion w-first), as the gsplat guide
(lmnt.cn/news/262699) §3.3 initialises them.

Stand-ins: the pages train on Mip-NeRF 360 / DTU captures, which are not
available here; the mixture workload reproduces the per-tile load imbalance
that such scenes show, the box and ground-plane workloads the uniform spread
of a large outdoor capture.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

NEAR_PLANE = 0.2
EPS2D = 0.3


@dataclass
class Scene:
    means: np.ndarray
    quats: np.ndarray
    log_scales: np.ndarray
    opacity_logits: np.ndarray
    sh: np.ndarray
    sh_degree: int

    @property
    def n(self) -> int:
        return int(self.means.shape[0])

    def subset(self, idx) -> "Scene":
        return Scene(self.means[idx], self.quats[idx], self.log_scales[idx],
                     self.opacity_logits[idx], self.sh[idx], self.sh_degree)


@dataclass
class Workload:
    name: str
    scene: Scene
    cameras: list
    upstream: list = field(default_factory=list)   # dL/dimage [H,W,3] per camera (tiny case)
    targets: list = field(default_factory=list)    # target images [H,W,3] per camera (L1 cases)
    bg: tuple = (0.0, 0.0, 0.0)
    adam_lr: dict = field(default_factory=dict)


# Adam learning rates per parameter group (gsplat guide, lmnt.cn/news/262699, §4.2 table)
ADAM_LR = {"means": 1.6e-4, "log_scales": 5e-3, "quats": 1e-3,
           "opacity_logits": 5e-2, "sh": 2.5e-3}
ADAM_BETAS = (0.9, 0.99)
ADAM_EPS = 1e-15


def camera(R, t, fx, fy, cx, cy, width, height, near=NEAR_PLANE, eps2d=EPS2D) -> dict:
    return {"R": np.asarray(R, np.float32).reshape(3, 3), "t": np.asarray(t, np.float32).reshape(3),
            "fx": float(fx), "fy": float(fy), "cx": float(cx), "cy": float(cy),
            "width": int(width), "height": int(height), "near": float(near), "eps2d": float(eps2d)}


def look_at(eye, target=(0.0, 0.0, 0.0)):
    """World-to-camera (R, t) for a camera at ``eye`` facing ``target``.

    Rows of R are the camera axes in world coordinates: x_c = y_c x f,
    y_c = the component of world "down" (-y, or -z when looking along y)
    orthogonal to the viewing direction f.  t = -R eye.
    """
    eye = np.asarray(eye, np.float64)
    f = np.asarray(target, np.float64) - eye
    f = f / np.linalg.norm(f)
    up = np.array([0.0, 1.0, 0.0])
    if np.linalg.norm(np.cross(f, up)) < 1e-6:
        up = np.array([0.0, 0.0, 1.0])
    down = -up
    y = down - np.dot(down, f) * f
    y = y / np.linalg.norm(y)
    x = np.cross(y, f)
    R = np.stack([x, y, f])
    t = -R @ eye
    return R.astype(np.float32), t.astype(np.float32)


def _unit_quats(rng, n):
    q = rng.standard_normal((n, 4))
    q /= np.linalg.norm(q, axis=1, keepdims=True)
    return q.astype(np.float32)


def _sh3(rng, n, dc):
    """Degree-3 SH block: DC given, the other 45 coefficients N(0, 0.1)."""
    sh = np.empty((n, 16, 3), np.float32)
    sh[:, 0, :] = dc
    sh[:, 1:, :] = (0.1 * rng.standard_normal((n, 15, 3))).astype(np.float32)
    return sh


def _sphere_poses(rng, count, radius):
    g = rng.standard_normal((count, 3))
    return [radius * v / np.linalg.norm(v) for v in g]


# Spherical-harmonic DC normalisation 1/Y_00 = 2 sqrt(pi): lets the tiny scene
# draw its base colour directly (colour = dc * Y_00 + 0.5 at degree 0).
_INV_Y00 = 2.0 * math.sqrt(math.pi)


def tiny(seed: int = 0) -> Workload:
    """1,000 Gaussians in [-1,1]^3, 128x128, SH degree 0, upstream dL/dimage ~ N(0,1)."""
    rng = np.random.default_rng(seed)
    n = 1000
    means = rng.uniform(-1.0, 1.0, (n, 3)).astype(np.float32)
    log_scales = rng.uniform(-4.0, -2.0, (n, 3)).astype(np.float32)
    quats = _unit_quats(rng, n)
    logits = rng.standard_normal(n).astype(np.float32)
    rgb = rng.uniform(0.0, 1.0, (n, 3))
    sh = ((rgb - 0.5) * _INV_Y00).astype(np.float32).reshape(n, 1, 3)
    R, t = look_at((0.0, 0.0, -4.0))
    cam = camera(R, t, 128.0, 128.0, 64.0, 64.0, 128, 128)
    g = rng.standard_normal((128, 128, 3)).astype(np.float32)
    return Workload("tiny-1k-128x128", Scene(means, quats, log_scales, logits, sh, 0), [cam], upstream=[g])


def box100k(seed: int = 0, poses: int = 100) -> Workload:
    """100k Gaussians in a 4x4x4 box, SH degree 3, 1920x1080, poses on a radius-6 sphere."""
    rng = np.random.default_rng(seed)
    n = 100_000
    means = rng.uniform(-2.0, 2.0, (n, 3)).astype(np.float32)
    log_scales = rng.normal(-4.0, 0.5, (n, 3)).astype(np.float32)
    quats = _unit_quats(rng, n)
    logits = rng.standard_normal(n).astype(np.float32)
    sh = _sh3(rng, n, rng.uniform(0.0, 1.0, (n, 3)))
    cams = []
    for eye in _sphere_poses(rng, poses, 6.0):
        R, t = look_at(eye)
        cams.append(camera(R, t, 1600.0, 1600.0, 960.0, 540.0, 1920, 1080))
    return Workload("box-100k-1920x1080", Scene(means, quats, log_scales, logits, sh, 3), cams)


def _mixture_scene(rng, n):
    k = 64
    d = rng.standard_normal((k, 3))
    d /= np.linalg.norm(d, axis=1, keepdims=True)
    centres = d * (3.0 * rng.uniform(0.0, 1.0, (k, 1)) ** (1.0 / 3.0))
    comp = rng.integers(0, k, n)
    means = (centres[comp] + 0.3 * rng.standard_normal((n, 3))).astype(np.float32)
    log_scales = rng.normal(-4.5, 0.7, (n, 3)).astype(np.float32)
    quats = _unit_quats(rng, n)
    logits = rng.normal(-1.0, 1.5, n).astype(np.float32)
    sh = _sh3(rng, n, rng.uniform(0.0, 1.0, (n, 3)))
    return Scene(means, quats, log_scales, logits, sh, 3)


def mixture1m(seed: int = 0, n: int = 1_000_000) -> Workload:
    """1M-Gaussian 64-cluster mixture, SH degree 3, one 1296x840 view, L1 target ~ U[0,1]."""
    rng = np.random.default_rng(seed)
    scene = _mixture_scene(rng, n)
    R, t = look_at((0.0, 0.0, -6.0))
    cam = camera(R, t, 1100.0, 1100.0, 648.0, 420.0, 1296, 840)
    target = rng.uniform(0.0, 1.0, (840, 1296, 3)).astype(np.float32)
    return Workload("mixture-1m-1296x840-train", scene, [cam], targets=[target], adam_lr=dict(ADAM_LR))


def city3m(seed: int = 0, poses: int = 50, n: int = 3_000_000) -> Workload:
    """3M Gaussians: 80% uniform in [-5,5]^3, 20% on a checkerboard ground plane y=-1; 3840x2160."""
    rng = np.random.default_rng(seed)
    n_plane = n // 5
    n_box = n - n_plane
    box = rng.uniform(-5.0, 5.0, (n_box, 3))
    xz = rng.uniform(-5.0, 5.0, (n_plane, 2))
    plane = np.stack([xz[:, 0], np.full(n_plane, -1.0), xz[:, 1]], axis=1)
    means = np.concatenate([box, plane]).astype(np.float32)
    log_scales = rng.normal(-5.0, 0.8, (n, 3)).astype(np.float32)
    quats = _unit_quats(rng, n)
    logits = rng.standard_normal(n).astype(np.float32)
    dc = np.empty((n, 3))
    dc[:n_box] = rng.uniform(0.0, 1.0, (n_box, 3))
    checker = (np.floor(xz[:, 0]).astype(np.int64) + np.floor(xz[:, 1]).astype(np.int64)) & 1
    dc[n_box:] = np.where(checker[:, None] == 0, 0.9, 0.1)
    sh = _sh3(rng, n, dc)
    cams = []
    for k in range(poses):
        a = 2.0 * math.pi * k / poses
        R, t = look_at((8.0 * math.cos(a), 0.0, 8.0 * math.sin(a)))
        cams.append(camera(R, t, 3000.0, 3000.0, 1920.0, 1080.0, 3840, 2160))
    return Workload("city-3m-3840x2160", Scene(means, quats, log_scales, logits, sh, 3), cams)


def multiview1m(seed: int = 0, views: int = 16, n: int = 1_000_000) -> Workload:
    """The 1M mixture seen from a fixed batch of 16 poses on a radius-6 sphere at 1920x1080,
    each view with its own L1 target ~ U[0,1]. A smaller `views` keeps the first poses
    of the 16 (the poses are drawn before the targets)."""
    rng = np.random.default_rng(seed)
    scene = _mixture_scene(rng, n)
    cams, targets = [], []
    for eye in _sphere_poses(rng, views, 6.0):
        R, t = look_at(eye)
        cams.append(camera(R, t, 1600.0, 1600.0, 960.0, 540.0, 1920, 1080))
    for _ in range(views):
        targets.append(rng.uniform(0.0, 1.0, (1080, 1920, 3)).astype(np.float32))
    return Workload(f"multiview-1m-{views}x1920x1080-train", scene, cams, targets=targets, adam_lr=dict(ADAM_LR))


WORKLOADS = {1: tiny, 2: box100k, 3: mixture1m, 4: city3m, 5: multiview1m}


def random_scene(rng, n, sh_degree, mean_box=1.0, log_scale=(-4.0, -2.0), logit=(0.0, 1.0)) -> Scene:
    """Small generic scene for edge-case and ragged-size tests."""
    means = rng.uniform(-mean_box, mean_box, (n, 3)).astype(np.float32)
    log_scales = rng.uniform(log_scale[0], log_scale[1], (n, 3)).astype(np.float32)
    quats = _unit_quats(rng, n)
    logits = rng.normal(logit[0], logit[1], n).astype(np.float32)
    nc = (sh_degree + 1) ** 2
    sh = np.empty((n, nc, 3), np.float32)
    sh[:, 0, :] = rng.uniform(0.0, 1.0, (n, 3))
    if nc > 1:
        sh[:, 1:, :] = 0.1 * rng.standard_normal((n, nc - 1, 3))
    return Scene(means, quats, log_scales, logits, sh, sh_degree)
