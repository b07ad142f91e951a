"""Benchmark of the differentiable tile rasterizer (one JSON line on rank 0).

Default workload: 1M-Gaussian 64-cluster mixture (SH degree 3) seen from a batch
of 16 camera poses at 1920x1080; one step (iteration) = for every view
project -> bin/sort -> raster forward -> L1 loss -> raster backward ->
project backward (with the densification statistic), then one Adam update of
all five parameter groups.  Metric: iterations/s (fwd+bwd), plus the step's
algorithmic HBM bytes against the measured copy bandwidth.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload multiview|mixture|box|city|tiny]

Other workloads: mixture (the 1M mixture, one 1296x840 view per training step),
tiny (1,000 Gaussians at 128x128), and the forward-only box (100k Gaussians, 1080p,
a step renders its 100 poses) and city (3M Gaussians, 3840x2160, 50 poses), which
report frames/s.

--impl reference times the CPU oracle (the plain double-precision per-pixel
renderer the tests use as ground truth) on a bounded sample of the same
workload.  With N > 1 every rank runs an independent replica (the path has no
exchange step); the reported value is the sum over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "fwd+bwd iterations/s and HBM GB/s vs roofline at 1M Gaussians, 1920x1080"
RENDER_METRIC = "forward rendering frames/s"
PEAK_FALLBACK = {"hbm_gbs": 6650.0, "source": "fallback"}
# FP32 lanes per SM and SMs of a B200 (the nominal ALU peak, context beside the measured one)
FP32_LANES_PER_SM = 128
NUM_SMS = 148
# float32 operations per (pixel, list entry) pair, counted from the kernels'
# arithmetic with an FMA as two: alpha evaluation (dx, dy, quadratic form,
# exponent, clamp, threshold tests) = 14, done for every pair a pixel traverses
# (its list up to n_contrib); forward blend = 8 and backward transmittance
# recovery, colour/alpha gradients and the chain to (u, v, A, B, C, o) = 46,
# done only for the pairs the pixel blends.
FLOPS_ALPHA = 14
FLOPS_FWD_BLEND = 8
FLOPS_BWD_GRAD = 46
# special-function instructions per evaluated (pixel, entry) pair: ex2 for alpha;
# the reverse pass adds rcp(1 - alpha)
SFU_FWD = 1
SFU_BWD = 2


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        d["source"] = "measured"
        return d
    return dict(PEAK_FALLBACK)


# --------------------------------------------------------------------- workloads

def make_workload(name: str, views: int = 16):
    from gaussian_splatting_differentiable_02_b200 import scenes
    if name == "multiview":
        return scenes.multiview1m(views=views)
    if name == "mixture":
        return scenes.mixture1m()
    if name == "box":
        return scenes.box100k(poses=100)     # forward only, timed over the 100 poses
    if name == "city":
        return scenes.city3m(poses=50)       # forward only, timed over the 50 poses
    if name == "tiny":
        wl = scenes.tiny()
        wl.targets = [np.full((128, 128, 3), 0.5, np.float32)]
        return wl
    raise ValueError(name)


def step_bytes(n, sh_degree, views_stats, tiles, pixels):
    """Algorithmic HBM bytes of one step: the multi-view projection (parameters once,
    outputs per view), per view the sum of the other stage terms, then the fused
    multi-view backward through the projection with Adam."""
    pb = 4 * (11 + 3 * (sh_degree + 1) ** 2)
    total = n * pb                             # project: the parameters, read once for all views
    for (K, V, passes) in views_stats:
        total += n * 52                        # project: this view's outputs
        total += n * (8 + 20 * 4)              # depth keys + 4 depth passes
        total += n * 16 + K * 8                # count (depth order) + emit (tile, gid)
        total += K * 20 * passes + K * 4       # tile passes (the last writes 12 instead of 8)
        total += K * 8 + tiles * 8             # tile ranges
        total += K * 4 + V * 36 + pixels * 20  # raster forward
        total += pixels * 36                   # L1 + dL/dimage
        total += K * 4 + V * 108 + pixels * 20  # raster backward
        total += n * 44                        # this view's radius + 2D gradients, read by the fused pass
    total += n * 6 * pb + n * 8                # fused pass: params read+write, m and v read+write, densify
    return total


# ----------------------------------------------------------------- clock sampling

class ClockSampler:
    def __init__(self, device_index: int):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--query-gpu={q}", "--format=csv,noheader,nounits",
                                       "-i", str(device_index), "-lms", "200"], stdout=self.f,
                                      stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None

    def stop(self):
        if self.p is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.p.terminate()
        try:
            self.p.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.p.kill()
        self.f.flush()
        self.f.seek(0)
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.f.read().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        os.unlink(self.f.name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ distributed

def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    return world, rank, local


def max_over_ranks(value: float, world: int) -> float:
    """Largest value over all ranks (identity for one rank)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------- reference arm

def cpu_oracle_sample(wl, fraction: float, seed: int = 0):
    """Time the oracle on a bounded sample of one view of the workload and scale
    to one iteration.  Returns (seconds per iteration, threads, description)."""
    import oracle
    threads = oracle.set_threads(0)   # 0: keep the current thread count, return it
    rng = np.random.default_rng(seed)
    scene, cam = wl.scene, wl.cameras[0]
    n = scene.n
    W, H = cam["width"], cam["height"]
    tx, ty = (W + 15) // 16, (H + 15) // 16
    ntiles = max(1, int(round(fraction * tx * ty)))
    tiles = rng.choice(tx * ty, ntiles, replace=False)
    pix = np.concatenate([[(t // tx) * 16 * W + (t % tx) * 16 + yy * W + xx for yy in range(16) for xx in range(16)
                           if (t // tx) * 16 + yy < H and (t % tx) * 16 + xx < W] for t in tiles]).astype(np.int64)
    gidx = np.sort(rng.choice(n, max(1, int(round(fraction * n))), replace=False))
    t0 = time.perf_counter()
    proj = oracle.project(scene, cam)                      # all Gaussians (needed by every pixel)
    t_proj = time.perf_counter() - t0
    t0 = time.perf_counter()
    keys, vals, ranges = oracle.keys(proj, cam)
    t_keys = time.perf_counter() - t0
    t0 = time.perf_counter()
    img, T, nc, amb = oracle.render(proj, cam, pix=pix)
    tgt = wl.targets[0].reshape(-1, 3)[pix] if wl.targets else np.zeros((len(pix), 3), np.float32)
    loss, g = oracle.l1(img.astype(np.float32), tgt)
    g2, _, _ = oracle.render_bwd(proj, cam, g.astype(np.float64), pix=pix)
    t_pix = time.perf_counter() - t0
    t0 = time.perf_counter()
    oracle.project_bwd(scene, cam, g2[gidx], idx=gidx, densify=True)
    t_pb = time.perf_counter() - t0
    nv = len(wl.cameras)
    per_view = t_proj + t_keys + t_pix * (tx * ty) / ntiles + t_pb * n / len(gidx)
    t0 = time.perf_counter()
    p = np.zeros(len(gidx) * 59, np.float32)
    oracle.adam(p, p, p, p, 1e-3, 0.9, 0.99, 1e-15, 1)
    t_adam = (time.perf_counter() - t0) * n / len(gidx)
    per_iter = nv * per_view + t_adam
    desc = (f"1 of {nv} views: projection+sort of all {n} Gaussians, forward+L1+backward on {ntiles} of {tx*ty} "
            f"tiles, project_bwd on {len(gidx)} Gaussians, Adam on {len(gidx)*59} floats; scaled to "
            f"{tx*ty} tiles, {n} Gaussians and {nv} views per iteration")
    return per_iter, threads, desc


def cpu_baseline(sample, wl, fraction, unit):
    """The oracle timed on the host on a bounded sample (`sample` returns seconds per
    unit, threads, description): once on every core OpenMP is given and once on a
    single thread (a quarter of the sample, scaled the same way)."""
    import oracle
    per_all, threads, desc = sample(wl, fraction)
    oracle.set_threads(1)
    try:
        per_one, _, desc_one = sample(wl, fraction / 4)
    finally:
        oracle.set_threads(threads)
    return {"value": 1.0 / per_all, "unit": unit, "cores": threads, "kind": "oracle", "sample": desc,
            "host_cpu_count": os.cpu_count(),
            "single_thread": {"value": 1.0 / per_one, "unit": unit, "cores": 1, "sample": desc_one},
            "thread_speedup": per_one / per_all}


def run_reference(args, world, rank):
    if rank != 0:
        return 0
    wl = make_workload(args.workload, args.views)
    fraction = args.cpu_fraction
    render = args.workload in ("box", "city")
    sample = cpu_oracle_render_sample if render else cpu_oracle_sample
    vals = []
    per_iter = threads = desc = None
    for i in range(args.warmup + args.steps):
        per_iter, threads, desc = sample(wl, fraction, seed=i)
        if i >= args.warmup:
            vals.append(per_iter)
    sec = statistics.mean(vals)
    value = 1.0 / sec
    unit = "frames/s" if render else "iterations/s"
    line = {"metric": RENDER_METRIC if render else METRIC, "value": value, "unit": unit, "n_gpus": args.gpus,
            "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": wl.name, "gaussians": wl.scene.n, "views_per_step": len(wl.cameras)},
            "cpu_baseline": {"value": value, "unit": unit, "cores": threads, "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------- our arm

def cpu_oracle_render_sample(wl, fraction: float, seed: int = 0):
    """The oracle's forward pass on a bounded sample of one pose (projection and keys
    of all Gaussians, compositing of a fraction of the tiles), scaled to one frame."""
    import oracle
    threads = oracle.set_threads(0)   # 0: keep the current thread count, return it
    rng = np.random.default_rng(seed)
    scene, cam = wl.scene, wl.cameras[0]
    W, H = cam["width"], cam["height"]
    tx, ty = (W + 15) // 16, (H + 15) // 16
    ntiles = max(1, int(round(fraction * tx * ty)))
    tiles = rng.choice(tx * ty, ntiles, replace=False)
    pix = np.concatenate([[(t // tx) * 16 * W + (t % tx) * 16 + yy * W + xx for yy in range(16) for xx in range(16)
                           if (t // tx) * 16 + yy < H and (t % tx) * 16 + xx < W] for t in tiles]).astype(np.int64)
    t0 = time.perf_counter()
    proj = oracle.project(scene, cam)
    oracle.keys(proj, cam)
    t_all = time.perf_counter() - t0
    t0 = time.perf_counter()
    oracle.render(proj, cam, pix=pix)
    t_pix = time.perf_counter() - t0
    per_frame = t_all + t_pix * (tx * ty) / ntiles
    desc = (f"1 pose: projection+sort of all {scene.n} Gaussians, compositing of {ntiles} of {tx * ty} tiles, "
            f"scaled to the whole frame")
    return per_frame, threads, desc


def measure_graph_frames(run_poses, poses, torch, stream, reps: int = 5):
    """Every pose rendered once, eagerly and replayed from a CUDA graph captured from the
    same calls (the poses' cameras are kernel arguments, fixed in the graph), ms per frame
    with CUDA events over `reps` rounds each."""
    def timed(fn):
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / (reps * poses)
    eager = timed(run_poses)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        run_poses()
    graph.replay()
    graphed = timed(graph.replay)
    return {"ms_per_frame_eager": eager, "ms_per_frame_graph": graphed, "speedup": eager / graphed,
            "frames_per_s_graph": 1e3 / graphed}


def run_render(args, world, rank, local):
    """Forward-only workloads (the 100k box at 1080p over 100 poses, the 3M city at
    4K over 50 poses): one step renders every pose once (projection, binning,
    compositing); the metric is frames/s."""
    import torch

    from gaussian_splatting_differentiable_02_b200 import abi
    from gaussian_splatting_differentiable_02_b200 import pipeline as pl

    if not torch.cuda.is_available():
        raise RuntimeError("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    abi.lib()
    wl = make_workload(args.workload, args.views)
    scene, cams = wl.scene, wl.cameras
    g = pl.Gaussians.from_scene(scene)
    view = pl.View(scene.n, cams[0], tile_cull=not args.no_tile_cull)
    proj = pl.Projected(scene.n)
    stream = torch.cuda.current_stream()
    # size the instance buffers for the largest pose
    for cam in cams:
        view.set_camera(cam)
        pl.project(g, view, proj)
        pl.bin_sort(proj, view)
    counter = torch.zeros((len(cams),), device=g.means.device, dtype=torch.int64)
    fwd_ev = []

    def frame(k, cam, record):
        view.set_camera(cam)
        pl.project(g, view, proj)
        pl.bin_sort_async(proj, view, counter[k:k + 1])
        if record:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
        pl.raster_fwd(proj, view)
        if record:
            e1.record(stream)
            fwd_ev.append((e0, e1))

    for _ in range(args.warmup):
        for k, cam in enumerate(cams):
            frame(k, cam, False)
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    barrier(world)
    launches0 = abi.gs_kernel_launches()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(args.steps):
        for k, cam in enumerate(cams):
            frame(k, cam, True)
    end.record(stream)
    torch.cuda.synchronize()
    launches = abi.gs_kernel_launches() - launches0
    barrier(world)
    clk = clocks.stop()
    if any(K > view.capacity for K in counter.cpu().tolist()):
        raise RuntimeError("instance buffers overflowed after the warm-up")
    ms = max_over_ranks(start.elapsed_time(end), world)
    frames = args.steps * len(cams)
    # work counters of the last pose's compositing (counted variant, outside the timing) and
    # the measured float32 / special-function peaks, for the roofline of raster_fwd
    counts = torch.zeros(5, device="cuda", dtype=torch.int64)
    pl.raster_fwd_counted(proj, view, counts)
    torch.cuda.synchronize()
    c = counts.cpu().tolist()
    work = {"traversed_pairs": float(view.n_contrib.sum().item()), "fwd_evaluated_pairs": float(c[0]),
            "fwd_blended_pairs": float(c[1]), "fwd_staged_entries": float(c[2]), "fwd_visited_pairs": float(c[4])}
    fwd_ms = statistics.mean(a.elapsed_time(b) for a, b in fwd_ev[-len(cams):])
    peaks = measured_peaks()
    alu = measure_alu_peaks(torch, local)
    last_ms = fwd_ev[-1][0].elapsed_time(fwd_ev[-1][1])
    roof = raster_roofline("raster_fwd", last_ms, work, alu)
    cam0 = cams[0]
    graph_row = None
    if not args.no_rows:
        graph_row = measure_graph_frames(lambda: [frame(k, cam, False) for k, cam in enumerate(cams)], len(cams),
                                         torch, stream)
    line = {"metric": RENDER_METRIC, "value": world * frames / (ms / 1e3), "unit": "frames/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": wl.name, "gaussians": scene.n, "poses_per_step": len(cams),
                       "image": f"{cam0['width']}x{cam0['height']}", "sh_degree": scene.sh_degree,
                       "tile_cull": not args.no_tile_cull,
                       "parallelism": f"replicas x{world}",
                       "l2": "a step renders every pose once; the instance lists of a pose exceed L2"},
            "stages_ms_per_frame": {"raster_fwd": fwd_ms, "frame": ms / frames},
            "roofline": roof, "raster_work_last_pose": work, "alu_peaks": alu,
            "gpu_launches": int(launches), "clocks": clk,
            "e2e": None, "hbm_peak_gbs": peaks["hbm_gbs"]}
    if graph_row is not None:
        line["rows"] = {"cuda_graph": graph_row}
    if rank == 0 and not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"] = cpu_baseline(cpu_oracle_render_sample, wl, args.cpu_fraction, "frames/s")
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def run_ours(args, world, rank, local):
    import torch

    from gaussian_splatting_differentiable_02_b200 import abi
    from gaussian_splatting_differentiable_02_b200 import pipeline as pl

    if not torch.cuda.is_available():
        raise RuntimeError("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    abi.lib()
    wl = make_workload(args.workload, args.views)
    scene = wl.scene
    nv = len(wl.cameras)
    gauss = pl.Gaussians.from_scene(scene)
    views = [pl.View(scene.n, cam) for cam in wl.cameras]
    targets_host = torch.from_numpy(np.stack(wl.targets)).pin_memory() if wl.targets else None
    targets = targets_host.cuda() if targets_host is not None else None
    lrs = dict(wl.adam_lr) if wl.adam_lr else {"means": 1.6e-4, "log_scales": 5e-3, "quats": 1e-3,
                                                  "opacity_logits": 5e-2, "sh": 2.5e-3}
    tr = pl.Trainer(gauss, views, [targets[i] for i in range(nv)], lrs, densify=True, streams=args.streams,
                    batched_sort=not args.per_view_sort, groups=args.groups, bin_views=not args.per_view_bin,
                    tile_cull=not args.no_tile_cull)
    stream = torch.cuda.current_stream()

    # warm-up (also sizes every view's instance buffers)
    for _ in range(args.warmup):
        tr.step()
    torch.cuda.synchronize()

    # per-stage breakdown of one untimed step, to find the dominant kernel
    stages = stage_breakdown(tr, pl, torch)
    dominant = max(stages, key=lambda k: stages[k])

    # ---- timed region: K steps on resident inputs
    ev_dom = []
    # stage -> the pipeline function whose calls make it
    stage_fn = {"raster_bwd": "raster_bwd", "raster_fwd": "raster_fwd", "project_bwd_adam": "project_bwd_views_adam",
                "project": "project_views"}
    orig = {name: getattr(pl, name) for name in stage_fn.values()}

    def wrap(fn):
        # events on the stream the kernel is launched on (the Trainer spreads views over streams)
        def inner(*a, **k):
            st = torch.cuda.current_stream()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(st)
            fn(*a, **k)
            e1.record(st)
            ev_dom.append((e0, e1))
        return inner

    if dominant in stage_fn:
        setattr(pl, stage_fn[dominant], wrap(orig[stage_fn[dominant]]))
    clocks = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    launches0 = abi.gs_kernel_launches()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(args.steps):
        tr.step()
    end.record(stream)
    torch.cuda.synchronize()
    launches = abi.gs_kernel_launches() - launches0
    barrier(world)
    clk = clocks.stop()
    for k, f in orig.items():
        setattr(pl, k, f)
    ms_local = start.elapsed_time(end)
    ms = max_over_ranks(ms_local, world)
    ms_per_step = ms / args.steps
    value = world * args.steps / (ms / 1e3)

    # ---- instance statistics for the byte / flop model
    stats = []
    pairs = 0
    for v in views:
        T = v.tiles_x * v.tiles_y
        passes = max(1, (math.ceil(math.log2(T)) + 7) // 8)
        stats.append((v.num_instances, int((tr.radii[len(stats)] > 0).sum().item()), passes))
        pairs += int(v.n_contrib.sum().item())
    cam0 = wl.cameras[0]
    P = cam0["width"] * cam0["height"]
    nbytes = step_bytes(scene.n, scene.sh_degree, stats, views[0].tiles_x * views[0].tiles_y, P)
    peaks = measured_peaks()
    hbm_peak = peaks["hbm_gbs"]
    step_gbs = nbytes / (ms_per_step * 1e-3) / 1e9

    dom_ms = statistics.mean(e0.elapsed_time(e1) for e0, e1 in ev_dom) if ev_dom else stages[dominant]
    # measured float32 / special-function peaks and the compositing kernels' work counters
    # (both after the timed region)
    alu = measure_alu_peaks(torch, local)
    work = raster_work_counts(tr, torch)
    roof = roofline_for(dominant, dom_ms, stats, scene, P, peaks, profile_key(wl), work=work, alu=alu)
    raster_roofs = {st: raster_roofline(st, stages[st] / nv, work, alu) for st in ("raster_fwd", "raster_bwd")}

    line = {"metric": METRIC, "value": value, "unit": "iterations/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": wl.name, "gaussians": scene.n, "views_per_step": nv, "streams": args.streams,
                       "depth_sort": "per view" if args.per_view_sort else "batched over the views" + (
                           f", in {len(tr.view_groups())} pipelined view groups" if len(tr.view_groups()) > 1 else ""),
                       "binning": ("per view" if (args.per_view_bin or args.per_view_sort) else
                                   "one launch per kernel for all the views of a group") +
                                  ("; each Gaussian in the tiles its footprint reaches" if tr.tile_cull else
                                   "; each Gaussian in every tile of its 3-sigma rectangle"),
                       "tile_cull": bool(tr.tile_cull),
                       "image": f"{cam0['width']}x{cam0['height']}", "sh_degree": scene.sh_degree,
                       "mean_instances_per_view": int(np.mean([s[0] for s in stats])),
                       "parallelism": f"replicas x{world}",
                       "l2": "inputs larger than L2: each step streams %.2f GB of parameters, optimizer state, "
                             "instances and images" % (nbytes / 1e9)},
            "hbm": {"algorithmic_bytes_per_step": nbytes, "achieved_gbs": step_gbs, "peak_gbs": hbm_peak,
                    "frac": step_gbs / hbm_peak, "peak_source": peaks["source"],
                    "frac_of_nominal_8000_gbs": step_gbs / 8000.0},
            "stages_ms_per_step": {k: round(v, 4) for k, v in stages.items()},
            "roofline": roof,
            "raster_alone": {k: {x: v[x] for x in ("achieved", "peak", "frac", "sfu")} for k, v in raster_roofs.items()},
            "raster_work_per_view": work,
            "alu_peaks": alu,
            "gpu_launches": int(launches),
            "clocks": clk}
    # e2e: the same step with the per-step inputs (16 target images) copied from
    # pinned host memory and the loss read back, inside the timed region
    line["e2e"] = run_e2e(tr, targets_host, targets, args, world, torch)
    # rows outside the per-step path, measured after the step timing
    with_oracle = rank == 0 and not args.no_cpu_baseline and world == 1
    if not args.no_rows:
        line["rows"] = {"cuda_graph": measure_graph_steps(tr, torch, abi),
                        "densify": measure_densify(tr, wl, peaks, torch, with_oracle),
                        "l1_dssim": measure_dssim(tr, wl, peaks, torch, with_oracle),
                        "absgrad_and_sparse_adam": measure_variants(tr, torch),
                        "packed": measure_packed(tr, wl, peaks, torch),
                        "sh16": measure_sh16(tr, wl, peaks, torch),
                        "tile_cull": measure_tile_cull(tr, wl, torch)}
        # the two options where they are meant to pay: packed views that keep a small part
        # of the scene, FP16 SH on a single-view step
        torch.cuda.empty_cache()
        line["rows"]["packed_narrow_views"] = measure_packed_narrow(torch)
        line["rows"]["sh16_single_view"] = measure_sh16_single_view(torch)
    if rank == 0 and not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"] = cpu_baseline(cpu_oracle_sample, wl, args.cpu_fraction, "iterations/s")
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def measure_graph_steps(tr, torch, abi, steps: int = 10):
    """The step with the views' part replayed from a CUDA graph (Trainer(graph=True)),
    against the eager step, both timed with CUDA events over `steps` steps of the same
    Trainer right after each other (the graph is captured in an untimed step first).
    Kernel timing events cannot be captured into a graph, which is why the line's own
    timing and roofline use the eager step."""
    def timed():
        torch.cuda.synchronize()
        l0 = abi.gs_kernel_launches()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(steps):
            tr.step()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / steps, (abi.gs_kernel_launches() - l0) / steps
    tr.graph = False
    tr.step()
    eager_ms, eager_launches = timed()
    tr.graph = True
    l0 = abi.gs_kernel_launches()
    tr.step()  # captures the views' part, then replays it
    torch.cuda.synchronize()
    captured = abi.gs_kernel_launches() - l0
    graph_ms, host_launches = timed()
    tr.graph = False
    tr._graph = None
    return {"step_ms_eager": eager_ms, "step_ms_graph": graph_ms, "speedup": eager_ms / graph_ms,
            "library_launches_per_step": eager_launches,
            "launches_per_step_from_the_graph": captured - host_launches,
            "launches_per_step_from_the_host": host_launches}


def measure_variants(tr, torch, reps: int = 10):
    """Cost of the absgrad option (raster backward with the absolute 2D gradient) on
    the first view, and of the sparse Adam option of the fused backward, each
    against the default, with CUDA events over `reps` launches."""
    from gaussian_splatting_differentiable_02_b200 import pipeline as pl
    s = torch.cuda.current_stream()
    view, r = tr.views[0], tr.radii[0]
    pl.project(tr.gauss, view, tr.proj, r)
    pl.bin_sort(tr.proj, view, r)
    pl.raster_fwd(tr.proj, view, tr.bg, r)
    plain = pl.Grad2D(tr.gauss.n)
    absg = pl.Grad2D(tr.gauss.n, absgrad=True)

    def timed(fn):
        for _ in range(3):
            fn()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s)
        for _ in range(reps):
            fn()
        e1.record(s)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps

    res = {"raster_bwd_ms": timed(lambda: pl.raster_bwd(tr.proj, view, plain, tr.bg, radius=r)),
           "raster_bwd_absgrad_ms": timed(lambda: pl.raster_bwd(tr.proj, view, absg, tr.bg, radius=r))}
    # the fused backward with Adam on copies of the parameters and moments
    g, m, v, gbuf = (x.zeros_like() for x in (tr.gauss, tr.gauss, tr.gauss, tr.gauss))
    for dst, src in ((g, tr.gauss), (m, tr.m), (v, tr.v)):
        for a, b in zip(dst.tensors().values(), src.tensors().values()):
            a.copy_(b)
    for sparse in (False, True):
        res["project_bwd_adam_sparse_ms" if sparse else "project_bwd_adam_ms"] = timed(
            lambda: pl.project_bwd_views_adam(g, tr.views, tr.proj, tr.radii, tr.grad2ds, m, v, tr.lrs,
                                              tr.step_count + 1, gbuf, sparse=sparse))
    res["visible_fraction"] = float((tr.radii > 0).any(dim=0).float().mean().item())
    return res


def paired_step_ms(tr_a, tr_b, steps, torch, rounds: int = 2):
    """Mean step time of two Trainers started from the same scene, timed in alternating
    segments of `steps` steps (a, b, a, b, ...) after 3 warm-up steps each, so that a
    drift of the clocks over the run affects both alike."""
    s = torch.cuda.current_stream()
    for t in (tr_a, tr_b):
        for _ in range(3):
            t.step()
    tot = [0.0, 0.0]
    for _ in range(rounds):
        for i, t in enumerate((tr_a, tr_b)):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(s)
            for _ in range(steps):
                t.step()
            e1.record(s)
            torch.cuda.synchronize()
            tot[i] += e0.elapsed_time(e1)
    return tot[0] / (rounds * steps), tot[1] / (rounds * steps)


def measure_packed(tr, wl, peaks, torch, steps: int = 5, reps: int = 10):
    """The packed layout (gs_project_packed): the training step with packed views against
    the same step unpacked (paired_step_ms), and the packed projection of the first view
    against the plain projection, with the HBM roofline of its algorithmic bytes (the
    projection's bytes as in step_bytes, the visibility read twice and the slot map
    written, and the visible Gaussians' 52 bytes of features read, written packed, and
    their ids written)."""
    from gaussian_splatting_differentiable_02_b200 import pipeline as pl
    s = torch.cuda.current_stream()
    scene = wl.scene
    trp = pl.Trainer(pl.Gaussians.from_scene(scene), [pl.View(scene.n, c) for c in wl.cameras], tr.targets,
                     dict(tr.lrs), densify=True, streams=tr.streams, groups=tr.groups, packed=True,
                     tile_cull=tr.tile_cull)

    # the unpacked arm starts from the same scene (the benchmark's own Trainer has
    # trained for many steps by now, and its Gaussians have moved)
    tru = pl.Trainer(pl.Gaussians.from_scene(scene), [pl.View(scene.n, c) for c in wl.cameras], tr.targets,
                     dict(tr.lrs), densify=True, streams=tr.streams, groups=tr.groups, tile_cull=tr.tile_cull)
    ms_packed, ms_unpacked = paired_step_ms(trp, tru, steps, torch)
    del tru
    res = {"step_ms_packed": ms_packed, "step_ms_unpacked": ms_unpacked}
    visible = trp.counts[1].cpu().numpy()
    res["visible_fraction_per_view"] = float(visible.mean() / max(scene.n, 1))
    res["slot_capacity"] = int(trp.pcap)

    def timed(fn):
        for _ in range(3):
            fn()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s)
        for _ in range(reps):
            fn()
        e1.record(s)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps

    view = trp.views[0]
    res["project_ms"] = timed(lambda: pl.project(tr.gauss, tr.views[0], tr.projs[0], tr.radii[0]))
    ms = timed(lambda: pl.project_packed(trp.gauss, view, trp.packs[0], trp.pack_ws))
    res["project_packed_ms"] = ms
    n, V = scene.n, int(visible[0])
    pb = 4 * (11 + 3 * (scene.sh_degree + 1) ** 2)
    nbytes = n * (pb + 52) + n * 12 + V * (52 + 52 + 4)
    gbs = nbytes / (ms * 1e-3) / 1e9
    res["project_packed_roofline"] = {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                      "frac": gbs / peaks["hbm_gbs"], "bytes_per_launch": nbytes}
    del trp
    return res


def narrow_views(views: int = 4, f: float = 3600.0):
    """The 3M city scene seen through narrow cameras (1920x1080, focal length 3600: a
    half-angle of 15 degrees horizontally) from the first poses of its radius-8 circle:
    each view keeps a small part of the scene, the regime the packed layout is for.
    Seeded random targets for an L1 training step."""
    from gaussian_splatting_differentiable_02_b200 import scenes
    wl = scenes.city3m(poses=views)
    cams = []
    for c in wl.cameras:
        R = np.asarray(c["R"], np.float64)
        eye = -R.T @ np.asarray(c["t"], np.float64)
        Rn, tn = scenes.look_at(eye)
        cams.append(scenes.camera(Rn, tn, f, f, 960.0, 540.0, 1920, 1080))
    rng = np.random.default_rng(7)
    targets = [rng.uniform(0.0, 1.0, (1080, 1920, 3)).astype(np.float32) for _ in cams]
    return wl.scene, cams, targets


def measure_packed_narrow(torch, steps: int = 5):
    """The packed layout where a view keeps a small part of the scene (narrow_views):
    training step time and device memory (held after the warm-up steps, and the peak
    over the timed steps, both above what was allocated before the Trainer) of
    Trainer(packed=True) against the same step unpacked, both from the same scene."""
    from gaussian_splatting_differentiable_02_b200 import pipeline as pl
    from gaussian_splatting_differentiable_02_b200 import scenes
    scene, cams, targets_h = narrow_views()
    targets = [torch.from_numpy(t).cuda() for t in targets_h]
    lrs = dict(scenes.ADAM_LR)
    res = {"workload": f"city 3M, {len(cams)} views of 1920x1080 at focal length {cams[0]['fx']:.0f}",
           "gaussians": scene.n}
    for packed in (True, False):
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
        base = torch.cuda.memory_allocated()
        tr = pl.Trainer(pl.Gaussians.from_scene(scene), [pl.View(scene.n, c) for c in cams], targets, dict(lrs),
                        densify=True, packed=packed)
        for _ in range(3):  # the packed Trainer sizes its slots to the views in these steps
            tr.step()
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
        # memory held by the Trainer in the steady state, and its peak over the timed steps
        res[f"resident_memory_gb_{'packed' if packed else 'unpacked'}"] = (torch.cuda.memory_allocated() - base) / 1e9
        torch.cuda.reset_peak_memory_stats()
        s = torch.cuda.current_stream()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s)
        for _ in range(steps):
            tr.step()
        e1.record(s)
        torch.cuda.synchronize()
        key = "packed" if packed else "unpacked"
        res[f"step_ms_{key}"] = e0.elapsed_time(e1) / steps
        res[f"peak_memory_gb_{key}"] = (torch.cuda.max_memory_allocated() - base) / 1e9
        if packed:
            res["visible_fraction_per_view"] = float(tr.counts[1].cpu().numpy().mean() / scene.n)
            res["slot_capacity"] = int(tr.pcap)
        del tr
    res["speedup"] = res["step_ms_unpacked"] / res["step_ms_packed"]
    return res


def measure_sh16_single_view(torch, steps: int = 10):
    """16-bit SH storage on the single-view training step of the 1M mixture at 1296x840,
    against the float32 step (paired_step_ms), both from the same scene."""
    from gaussian_splatting_differentiable_02_b200 import pipeline as pl
    from gaussian_splatting_differentiable_02_b200 import scenes
    wl = scenes.mixture1m()
    targets = [torch.from_numpy(t).cuda() for t in wl.targets]
    mk = [pl.Trainer(pl.Gaussians.from_scene(wl.scene), [pl.View(wl.scene.n, c) for c in wl.cameras], targets,
                     dict(wl.adam_lr), densify=True, sh16=h) for h in (True, False)]
    ms_h, ms_f = paired_step_ms(mk[0], mk[1], steps, torch)
    del mk
    return {"workload": "mixture 1M, one 1296x840 view per step", "step_ms_sh16": ms_h, "step_ms_f32": ms_f,
            "speedup": ms_f / ms_h}


def measure_sh16(tr, wl, peaks, torch, steps: int = 5, reps: int = 10):
    """16-bit SH storage: the training step with the projections reading the half copy
    (Trainer(sh16=True)) against the float32 step (paired_step_ms), and the projection of the first view
    from half against float32 coefficients, each with the HBM roofline of its algorithmic
    bytes (the parameters read, with 2 or 4 bytes per SH coefficient, and 52 bytes of
    projected features written)."""
    from gaussian_splatting_differentiable_02_b200 import pipeline as pl
    s = torch.cuda.current_stream()
    scene = wl.scene
    trh = pl.Trainer(pl.Gaussians.from_scene(scene), [pl.View(scene.n, c) for c in wl.cameras], tr.targets,
                     dict(tr.lrs), densify=True, streams=tr.streams, groups=tr.groups, sh16=True,
                     tile_cull=tr.tile_cull)

    def timed(fn, count):
        for _ in range(3):
            fn()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s)
        for _ in range(count):
            fn()
        e1.record(s)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / count

    trf = pl.Trainer(pl.Gaussians.from_scene(scene), [pl.View(scene.n, c) for c in wl.cameras], tr.targets,
                     dict(tr.lrs), densify=True, streams=tr.streams, groups=tr.groups, tile_cull=tr.tile_cull)
    ms_sh16, ms_f32 = paired_step_ms(trh, trf, steps, torch)
    del trf
    res = {"step_ms_sh16": ms_sh16, "step_ms_f32": ms_f32}
    n, nc = scene.n, 3 * (scene.sh_degree + 1) ** 2
    for name, fn, sh_bytes in (
            ("f32", lambda: pl.project(tr.gauss, tr.views[0], tr.projs[0], tr.radii[0]), 4),
            ("sh16", lambda: pl.project_sh16(trh.gauss, trh.sh_half, trh.views[0], trh.projs[0], trh.radii[0]), 2)):
        ms = timed(fn, reps)
        nbytes = n * (44 + sh_bytes * nc + 52)
        gbs = nbytes / (ms * 1e-3) / 1e9
        res[f"project_{name}_ms"] = ms
        res[f"project_{name}_roofline"] = {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                           "frac": gbs / peaks["hbm_gbs"], "bytes_per_launch": nbytes}
    del trh
    return res


def measure_tile_cull(tr, wl, torch, steps: int = 5):
    """Binning each Gaussian only into the tiles its footprint reaches (gs_camera.tile_cull)
    against binning it into its whole 3-sigma rectangle: the training step of two Trainers
    started from the same scene (paired_step_ms), the other settings those of the timed
    Trainer, and the instances per view."""
    from gaussian_splatting_differentiable_02_b200 import pipeline as pl
    scene = wl.scene

    def make(cull):
        return pl.Trainer(pl.Gaussians.from_scene(scene), [pl.View(scene.n, c) for c in wl.cameras], tr.targets,
                          dict(tr.lrs), densify=True, streams=tr.streams, groups=tr.groups, bin_views=tr.bin_views,
                          tile_cull=cull)

    on, off = make(True), make(False)
    ms_on, ms_off = paired_step_ms(on, off, steps, torch)
    k_on = float(on.kcount.double().mean().item())
    k_off = float(off.kcount.double().mean().item())
    del on, off
    torch.cuda.empty_cache()
    return {"step_ms_culled": ms_on, "step_ms_rectangles": ms_off, "instances_per_view_culled": k_on,
            "instances_per_view_rectangles": k_off, "instances_kept": k_on / k_off}


def measure_dssim(tr, wl, peaks, torch, with_oracle: bool, reps: int = 10):
    """The L1 + D-SSIM loss and gradient (weights 1 and 0.2) of the first view's
    rendered image against its target, timed with CUDA events over `reps` calls,
    against the HBM roofline of its algorithmic bytes (image and target read
    twice, the 72-byte-per-pixel derivative maps written and read, dL/dimage
    written); the oracle timed on a 256 x 256 crop and scaled by pixel count."""
    from gaussian_splatting_differentiable_02_b200 import pipeline as pl
    view, target = tr.views[0], tr.targets[0]
    H, W = view.image.shape[0], view.image.shape[1]
    loss = torch.zeros((1,), device=view.image.device, dtype=torch.float64)
    s = torch.cuda.current_stream()
    for _ in range(3):
        pl.l1_dssim_loss_grad(view, target, loss)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s)
    for _ in range(reps):
        pl.l1_dssim_loss_grad(view, target, loss)
    e1.record(s)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    nbytes = H * W * (24 + 72 + 72 + 24 + 12)
    hbm = peaks["hbm_gbs"]
    res = {"image": f"{W}x{H}", "ms": ms,
           "roofline": {"kernel": "ssim_moments + ssim_grad", "bound": "hbm", "achieved": nbytes / ms / 1e6,
                        "peak": hbm, "unit": "GB/s", "frac": nbytes / ms / 1e6 / hbm, "traffic": None,
                        "algorithmic_bytes": nbytes, "peak_source": peaks["source"]}}
    if with_oracle:
        import oracle
        c = 256
        x = view.image[:c, :c].double().cpu().numpy()
        y = target[:c, :c].double().cpu().numpy()
        t0 = time.perf_counter()
        oracle.l1_dssim(x, y)
        dt = time.perf_counter() - t0
        res["cpu_oracle"] = {"ms": dt * 1e3 * (H * W) / (c * c), "cores": oracle.set_threads(0), "kind": "oracle",
                             "sample": f"{c}x{c} crop, scaled by pixel count"}
    return res


def measure_densify(tr, wl, peaks, torch, with_oracle: bool, reps: int = 10):
    """Adaptive density control on the trainer's Gaussians and statistics (the
    gradient threshold at the median of the visible Gaussians' mean statistic, so
    that about half of them densify): gs_densify_plan and gs_densify_apply timed
    with CUDA events over `reps` launches each, against the HBM roofline of their
    algorithmic bytes; the oracle timed on the same inputs."""
    from gaussian_splatting_differentiable_02_b200 import abi
    from gaussian_splatting_differentiable_02_b200 import pipeline as pl
    g, n = tr.gauss, tr.gauss.n
    s = torch.cuda.current_stream()
    acc, cnt = tr.densify_accum[:n], tr.densify_count[:n]
    vis = cnt > 0
    thr = float((acc[vis] / cnt[vis]).median().item()) if bool(vis.any()) else 0.0
    cam = wl.cameras[0]
    cfg = pl.densify_config(cam["width"], cam["height"], grad_threshold=thr)
    gen = torch.Generator(device=g.means.device)
    gen.manual_seed(1)
    noise = torch.randn((n, 6), device=g.means.device, generator=gen)
    ws_bytes = abi.gs_densify_workspace_bytes(n)
    ws = torch.empty((ws_bytes,), device=g.means.device, dtype=torch.uint8)
    dec = torch.empty((n,), device=g.means.device, dtype=torch.uint8)
    num = torch.zeros((1,), device=g.means.device, dtype=torch.int64)
    mr = tr.densify_max_radius[:n]

    def plan():
        abi.gs_densify_plan(g.params(), pl._ptr(acc), pl._ptr(cnt), pl._ptr(mr), cfg, pl._ptr(ws), ws_bytes,
                            pl._ptr(dec), pl._ptr(num), s.cuda_stream)

    plan()
    n_out = int(num.item())
    out, om, ov = (pl.Gaussians(n_out, g.sh_degree, g.means.device) for _ in range(3))

    def apply():
        abi.gs_densify_apply(g.params(), tr.m.params(), tr.v.params(), pl._ptr(noise), pl._ptr(dec), pl._ptr(ws),
                             ws_bytes, n_out, out.grads(), om.grads(), ov.grads(), s.cuda_stream)

    def timed(fn):
        for _ in range(3):
            fn()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s)
        for _ in range(reps):
            fn()
        e1.record(s)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps

    plan_ms = timed(plan)
    apply_ms = timed(apply)
    d = torch.bincount(dec.long(), minlength=4).tolist()
    pb = 4 * (11 + 3 * (g.sh_degree + 1) ** 2)
    plan_bytes = n * (4 + 12 + 4 + 4 + 4 + 1)
    apply_bytes = (n + (d[1] + d[2]) * 3 * pb + d[3] * (pb + 24) + n_out * 3 * pb)
    hbm = peaks["hbm_gbs"]
    res = {"gaussians_in": n, "gaussians_out": n_out, "decisions": {"prune": d[0], "keep": d[1], "clone": d[2],
                                                                      "split": d[3]},
           "grad_threshold": thr, "plan_ms": plan_ms, "apply_ms": apply_ms,
           "roofline": {"kernel": "densify_apply", "bound": "hbm", "achieved": apply_bytes / apply_ms / 1e6,
                        "peak": hbm, "unit": "GB/s", "frac": apply_bytes / apply_ms / 1e6 / hbm,
                        "traffic": None, "algorithmic_bytes": apply_bytes, "peak_source": peaks["source"]},
           "plan_roofline_frac": plan_bytes / plan_ms / 1e6 / hbm}
    if with_oracle:
        import oracle
        from gaussian_splatting_differentiable_02_b200 import scenes
        p = g.to_numpy()
        sc = scenes.Scene(p["means"], p["quats"], p["log_scales"], p["opacity_logits"], p["sh"], g.sh_degree)
        a_h, c_h, r_h = acc.cpu().numpy(), cnt.cpu().numpy(), mr.cpu().numpy()
        z = noise.cpu().numpy().reshape(n, 2, 3)
        t0 = time.perf_counter()
        want = oracle.densify(sc, a_h, c_h, r_h, z, cfg.grad_threshold, cfg.scale_threshold, cfg.min_opacity,
                              cfg.max_screen_radius)
        res["cpu_oracle"] = {"ms": (time.perf_counter() - t0) * 1e3, "cores": 1, "kind": "oracle",
                             "sample": "all Gaussians, parameters only (no moments)",
                             "decisions_equal": bool(np.array_equal(want["decision"], dec.cpu().numpy()))}
    return res


def measure_alu_peaks(torch, local, target_ms: float = 60.0, reps: int = 5):
    """Measured instruction throughputs of this device (gs_alu_probe): float32 FMA
    scalar and paired (TFLOP/s, an FMA counting two) and ex2 / rcp.approx
    (T instructions x lanes per second); each op is calibrated to about
    `target_ms` per launch and the best of `reps` launches is kept (CUDA events)."""
    from gaussian_splatting_differentiable_02_b200 import abi
    out = torch.empty(abi.gs_alu_probe_slots(), device="cuda", dtype=torch.float32)
    s = torch.cuda.current_stream()
    names = {abi.GS_PROBE_FFMA: "ffma", abi.GS_PROBE_FFMA2: "ffma2", abi.GS_PROBE_EX2: "ex2",
             abi.GS_PROBE_RCP: "rcp"}
    res = {}
    clocks = ClockSampler(local)

    def once(op, iters):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s)
        ops = abi.gs_alu_probe(op, iters, out.data_ptr(), out.numel(), s.cuda_stream)
        e1.record(s)
        torch.cuda.synchronize()
        return ops, e0.elapsed_time(e1)

    for op, name in names.items():
        once(op, 256)
        ops, ms = once(op, 4096)
        iters = max(4096, int(4096 * target_ms / max(ms, 1e-3)))
        best = None
        for _ in range(reps):
            ops, ms = once(op, iters)
            rate = ops / (ms * 1e-3) / 1e12
            best = rate if best is None else max(best, rate)
        res[name] = best
    clk = clocks.stop()
    return {"ffma_tflops": res["ffma"], "ffma2_tflops": res["ffma2"], "ex2_tops": res["ex2"],
            "rcp_tops": res["rcp"], "fp32_tflops": max(res["ffma"], res["ffma2"]), "clocks": clk,
            "source": "measured: gs_alu_probe, 8 blocks x 256 threads per SM, best of %d launches of ~%.0f ms"
                      % (reps, target_ms)}


def raster_work_counts(tr, torch):
    """Work counters of the compositing kernels over the step's views, from the
    counted variants run once on the last step's lists (outside any timing):
    per view mean of the pairs the reverse pass's per-pixel loop visits (sum of
    n_contrib), of those the forward pass's loop visits (each pixel's list up to
    the entry it stops at, or all of it), the pairs it blends, the pairs the
    warps evaluate, and the list entries staged."""
    from gaussian_splatting_differentiable_02_b200 import pipeline as pl
    nv = len(tr.views)
    cf = torch.zeros(5, device="cuda", dtype=torch.int64)
    cb = torch.zeros(5, device="cuda", dtype=torch.int64)
    traversed = 0
    g2 = pl.Grad2D(tr.gauss.n)
    batched = getattr(tr, "depth_orders", None) is not None
    for k in range(nv):
        view, r = tr.views[k], tr._radius(k)
        if batched:
            proj = tr.projs[k]   # the view's projection, kept with its lists
        else:                    # the projections were reused across views: redo this view's
            proj = tr.proj
            pl.project(tr.gauss, view, proj, r)
            pl.bin_sort(proj, view, r)
        pl.raster_fwd_counted(proj, view, cf, tr.bg, r)
        traversed += int(view.n_contrib.sum().item())
        pl.raster_bwd_counted(proj, view, g2, cb, tr.bg, r)
    torch.cuda.synchronize()
    f, b = cf.cpu().tolist(), cb.cpu().tolist()
    return {"traversed_pairs": traversed / nv, "fwd_evaluated_pairs": f[0] / nv, "fwd_blended_pairs": f[1] / nv,
            "fwd_staged_entries": f[2] / nv, "fwd_visited_pairs": f[4] / nv, "bwd_evaluated_pairs": b[0] / nv,
            "bwd_gradient_pairs": b[1] / nv, "bwd_staged_entries": b[2] / nv}


def stage_breakdown(tr, pl, torch):
    """Milliseconds per step of each stage, from CUDA events around every call of
    one untimed step."""
    stream = torch.cuda.current_stream()
    acc = {}

    def timed(name, fn, *a, **kw):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        r = fn(*a, **kw)
        e1.record(stream)
        acc.setdefault(name, []).append((e0, e1))
        return r

    batched = getattr(tr, "depth_orders", None) is not None
    if batched:   # the Trainer's order: per view group the projections and one batched depth sort, then per view
        for ks, d in zip(tr.view_groups(), tr.depth_orders):
            timed("project", pl.project_views, tr.gauss, [tr.views[k] for k in ks], [tr.projs[k] for k in ks],
                  [tr.radii[k] for k in ks])
            timed("bin_sort", pl.depth_order_views, [tr.projs[k] for k in ks], [tr.radii[k] for k in ks], d)
            if tr.bin_views:
                timed("bin_sort", pl.bin_sort_ordered_views_async, [tr.projs[k] for k in ks],
                      [tr.views[k] for k in ks], d, tr.kcount[ks[0]:ks[-1] + 1], [tr.radii[k] for k in ks])
    for k, (view, tgt) in enumerate(zip(tr.views, tr.targets)):
        r = tr.radii[k]
        g2 = tr.grad2ds[k]
        proj = tr.projs[k] if batched else tr.proj
        if batched:
            if not tr.bin_views:
                timed("bin_sort", pl.bin_sort_ordered_async, proj, view, tr.order_row(k), tr.kcount[k:k + 1], r)
        else:
            timed("project", pl.project, tr.gauss, view, proj, r)
            timed("bin_sort", pl.bin_sort, proj, view, r)
        if tr.ssim_weight > 0.0:
            timed("raster_fwd", pl.raster_fwd, proj, view, tr.bg, r)
            timed("l1", pl.l1_dssim_loss_grad, view, tgt, tr.loss, 1.0, tr.ssim_weight)
        else:   # the Trainer's L1 step: the loss and dL/dimage come out of the forward kernel
            timed("raster_fwd", pl.raster_fwd_l1, proj, view, tgt, tr.loss, tr.bg, r)
        g2.zero_()
        timed("raster_bwd", pl.raster_bwd, proj, view, g2, tr.bg, None, r)
    tr.step_count += 1
    timed("project_bwd_adam", pl.project_bwd_views_adam, tr.gauss, tr.views, tr.proj, tr.radii, tr.grad2ds, tr.m,
          tr.v, tr.lrs, tr.step_count, tr.grads, tr.densify_accum, tr.densify_count,
          densify_max_radius=tr.densify_max_radius)
    torch.cuda.synchronize()
    return {k: sum(a.elapsed_time(b) for a, b in v) for k, v in acc.items()}


# Source file of each stage's kernels: a DRAM traffic figure taken by ncu is
# reported only while this file is unchanged since the capture.
STAGE_SOURCES = {
    "raster_bwd": ["csrc/raster.cu"],
    "raster_fwd": ["csrc/raster.cu"],
    "project_bwd_adam": ["csrc/project_bwd.cu"],
}


def profile_key(wl):
    """File-name key of a workload's ncu summaries: the scene and the image size
    (one launch of a stage does the same work whatever the number of views)."""
    cam = wl.cameras[0]
    scene = wl.name.split("-")[0] + wl.name.split("-")[1]
    return f"{scene}_{cam['width']}x{cam['height']}"


def stage_source_digest(stage):
    import hashlib
    pkg = os.path.join(ROOT, "gaussian_splatting_differentiable_02_b200")
    h = hashlib.sha256()
    for rel in STAGE_SOURCES[stage]:
        with open(os.path.normpath(os.path.join(pkg, rel)), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def profiled_traffic(stage, workload):
    """DRAM bytes per launch (read + write) of the stage's kernel from the ncu
    summary under profiles/, or None when there is none for this workload or the
    kernel's sources changed since it was taken."""
    if stage not in STAGE_SOURCES:
        return None
    path = os.path.join(ROOT, "profiles", f"{stage}_{workload}.md")
    if not os.path.exists(path):
        return None
    fields = {}
    with open(path) as f:
        for line in f:
            if ":" in line and line.startswith("- `"):
                k, v = line[3:].split("`", 1)[0], line.split(":", 1)[1].strip().strip("`")
                fields[k] = v
    try:
        if fields.get("source_sha256") != stage_source_digest(stage):
            return None
        return float(fields["traffic_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


def raster_roofline(stage, ms, work, alu, workload=""):
    """Roofline object of a compositing kernel against the measured float32 FMA
    peak: achieved = the method's flops per launch (FLOPS_ALPHA per pair its
    per-pixel loop visits: in the forward pass each pixel's list up to the entry
    at which it stops, in the reverse pass up to its n_contrib; plus the blend or
    gradient flops per blended pair) / the mean launch time.  The
    special-function unit (ex2, rcp per evaluated pair) is reported beside it
    against its own measured rate."""
    fwd = stage == "raster_fwd"
    blended = work["fwd_blended_pairs"] if fwd else work["bwd_gradient_pairs"]
    evaluated = work["fwd_evaluated_pairs"] if fwd else work["bwd_evaluated_pairs"]
    visited = work.get("fwd_visited_pairs", work["traversed_pairs"]) if fwd else work["traversed_pairs"]
    flops = FLOPS_ALPHA * visited + (FLOPS_FWD_BLEND if fwd else FLOPS_BWD_GRAD) * blended
    achieved = flops / (ms * 1e-3) / 1e12
    peak = alu["fp32_tflops"]
    sfu_ops = evaluated * (SFU_FWD if fwd else SFU_BWD)
    sfu_rate = sfu_ops / (ms * 1e-3) / 1e12
    return {"kernel": stage, "bound": "alu", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
            "frac": achieved / peak, "traffic": profiled_traffic(stage, workload),
            "work": (f"{visited:.4g} visited pairs x {FLOPS_ALPHA} + {blended:.4g} blended pairs x "
                     f"{FLOPS_FWD_BLEND if fwd else FLOPS_BWD_GRAD} flops per launch (mean over views)"),
            "peak_source": f"measured float32 FMA throughput ({alu['source']})",
            "sfu": {"achieved_tops": sfu_rate, "peak_tops": alu["ex2_tops"], "frac": sfu_rate / alu["ex2_tops"],
                    "ops": f"{evaluated:.4g} evaluated pairs x {SFU_FWD if fwd else SFU_BWD} (ex2{'' if fwd else ' + rcp'})"},
            "evaluated_over_visited": evaluated / max(visited, 1.0),
            "nominal_fp32_tflops": NUM_SMS * FP32_LANES_PER_SM * 2 * 1965.0 * 1e6 / 1e12}


def roofline_for(stage, ms, stats, scene, P, peaks, workload="", work=None, alu=None):
    """Roofline object of the dominant kernel: the raster kernels against the
    measured float32 FMA peak (raster_roofline), the streaming kernels against
    the measured HBM copy bandwidth."""
    K = float(np.mean([s[0] for s in stats]))
    pb = 4 * (11 + 3 * (scene.sh_degree + 1) ** 2)
    if stage in ("raster_bwd", "raster_fwd"):
        return raster_roofline(stage, ms, work, alu, workload)
    n = scene.n
    nv = len(stats)
    per_launch = {"project_bwd_adam": n * (6 * pb + 44 * nv + 8), "project": n * (pb + 52 * nv),
                  "bin_sort": n * 24 + K * 12 + K * (8 + 24 * stats[0][2]) + K * 8,
                  "adam": n * pb // 4 * 28, "l1": P * 36}.get(stage, 0)
    achieved = per_launch / (ms * 1e-3) / 1e9
    return {"kernel": stage, "bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / peaks["hbm_gbs"], "traffic": profiled_traffic(stage, workload),
            "peak_source": peaks["source"]}


def run_e2e(tr, targets_host, targets, args, world, torch):
    """Steps whose target images arrive from pinned host memory (copied on a side
    stream a few views ahead, overlapping the kernels of the views before) and
    whose loss is read back every step; the views run through the Trainer's own
    view loop."""
    if targets_host is None:
        return None
    stream = torch.cuda.current_stream()
    copy_stream = torch.cuda.Stream()
    nv = len(tr.views)
    side = tr.side_streams()
    nbuf = min(nv, 2 * len(side))   # targets in flight: the views running plus the next ones
    loss_host = torch.zeros(1, dtype=torch.float64).pin_memory()
    bufs = [torch.empty_like(targets[0]) for _ in range(nbuf)]

    # the view loop mirrors Trainer.step with the target taken from the copy buffers
    from gaussian_splatting_differentiable_02_b200 import pipeline as pl
    from gaussian_splatting_differentiable_02_b200 import abi

    def step():
        abi.gs_zero(tr.loss.data_ptr(), 8, stream.cuda_stream)
        begin = stream.record_event()
        copy_events = {}
        with torch.cuda.stream(copy_stream):
            copy_stream.wait_event(begin)   # the previous step's views are done with the buffers
            for v in range(nbuf):
                bufs[v].copy_(targets_host[v], non_blocking=True)
                copy_events[v] = copy_stream.record_event()

        class Ready:   # the copy event of view v exists by the time the Trainer asks for it
            def __getitem__(self, v):
                return copy_events[v]

        def after_view(v, ev):
            if v + nbuf < nv:
                with torch.cuda.stream(copy_stream):
                    copy_stream.wait_event(ev)
                    bufs[v % nbuf].copy_(targets_host[v + nbuf], non_blocking=True)
                    copy_events[v + nbuf] = copy_stream.record_event()

        tr._all_views(targets=[bufs[v % nbuf] for v in range(nv)], ready=Ready(), after_view=after_view)
        # the step's one wait: the instance counts (buffers were sized in the warm-up)
        if any(K > vw.capacity for K, vw in zip(tr.kcount.cpu().tolist(), tr.views)):
            raise RuntimeError("instance buffers overflowed after the warm-up")
        tr.step_count += 1
        pl.project_bwd_views_adam(tr.gauss, tr.views, tr.proj, tr.radii, tr.grad2ds, tr.m, tr.v, tr.lrs,
                                  tr.step_count, tr.grads, tr.densify_accum, tr.densify_count,
                                  densify_max_radius=tr.densify_max_radius)
        loss_host.copy_(tr.loss, non_blocking=True)

    for _ in range(max(1, args.warmup // 2)):
        step()
    torch.cuda.synchronize()
    barrier(world)
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(args.steps):
        step()
    end.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(start.elapsed_time(end), world)
    h2d = int(targets_host.numel() * 4)
    return {"value": world * args.steps / (ms / 1e3), "unit": "iterations/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": 8, "ms_per_step": ms / args.steps}


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["multiview", "mixture", "box", "city", "tiny"], default="multiview")
    ap.add_argument("--cpu-fraction", type=float, default=1.0 / 256)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-rows", action="store_true",
                    help="skip the rows of the other options (densification, D-SSIM, absgrad, packed, FP16 SH): "
                         "for short profiler captures, not a bench line")
    ap.add_argument("--streams", type=int, default=3,
                    help="CUDA streams the views of a step alternate over (1 = serial)")
    ap.add_argument("--groups", type=int, default=1,
                    help="view groups of the batched path (projection and depth sort of a group overlap "
                         "the compositing of the groups before it)")
    ap.add_argument("--per-view-bin", action="store_true",
                    help="bin each view with its own launches instead of one launch per kernel for a view group")
    ap.add_argument("--no-tile-cull", action="store_true",
                    help="bin each Gaussian into every tile of its 3-sigma rectangle instead of only the tiles "
                         "where its alpha can reach 1/255")
    ap.add_argument("--per-view-sort", action="store_true",
                    help="sort each view on its own stream instead of one batched depth sort of all views")
    ap.add_argument("--views", type=int, default=16,
                    help="views per step of the multiview workload (fewer: the first poses of the 16; "
                         "for small profiler captures, not a bench line)")
    args = ap.parse_args(argv)
    if not 1 <= args.views <= 16:
        ap.error("--views must be in 1..16")
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world, rank, local = dist_setup()
    try:
        if args.impl == "reference":
            return run_reference(args, world, rank)
        if args.workload in ("box", "city"):
            return run_render(args, world, rank, local)
        return run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
