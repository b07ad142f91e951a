"""Host-side checks of the C ABI (no GPU needed): libgs.so loads, exports every
function include/gs.h declares, and rejects bad arguments before it touches
the device."""
import ctypes as C
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gs.h")


@pytest.fixture(scope="module")
def gs():
    from gaussian_splatting_differentiable_02_b200 import build
    build.build()
    from gaussian_splatting_differentiable_02_b200 import abi
    abi.lib()
    return abi


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gs_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_hot_path_calls():
    names = declared_functions()
    for f in ("gs_project", "gs_bin_sort", "gs_raster_fwd", "gs_raster_bwd", "gs_project_bwd", "gs_adam"):
        assert f in names


def test_library_exports_every_declared_function(gs):
    out = subprocess.run(["nm", "-D", "--defined-only", gs.LIB_PATH], capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\bT (gs_[a-z0-9_]+)$", out, flags=re.M))
    missing = [f for f in declared_functions() if f not in exported]
    assert not missing, missing
    # the binding covers every declared function with the same name
    assert set(declared_functions()) == set(gs.SIGNATURES)
    for f in declared_functions():
        assert hasattr(gs, f)


def test_status_strings(gs):
    for code in range(5):
        assert gs.gs_status_string(code).startswith("GS_")
    assert "unknown" in gs.gs_status_string(99)


def test_sh_planes(gs):
    assert [gs.gs_sh_planes(d) for d in range(5)] == [1, 3, 7, 12, 0]


def cam(**kw):
    from gaussian_splatting_differentiable_02_b200 import scenes
    c = dict(scenes.tiny().cameras[0])
    c.update(kw)
    return c


def test_tile_grid_and_camera_checks(gs):
    assert gs.gs_tile_grid(gs.make_camera(cam())) == (8, 8)
    assert gs.gs_tile_grid(gs.make_camera(cam(width=100, height=37))) == (7, 3)
    with pytest.raises(gs.GsError) as e:
        gs.gs_tile_grid(gs.make_camera(cam(width=0)))
    assert e.value.status == gs.GS_ERR_UNSUPPORTED
    with pytest.raises(gs.GsError) as e:
        gs.gs_tile_grid(gs.make_camera(cam(width=20000)))
    assert e.value.status == gs.GS_ERR_UNSUPPORTED
    with pytest.raises(gs.GsError) as e:
        gs.gs_tile_grid(gs.make_camera(cam(fx=-1.0)))
    assert e.value.status == gs.GS_ERR_INVALID_ARG
    with pytest.raises(gs.GsError) as e:
        gs.gs_tile_grid(gs.make_camera(cam(near=0.0)))
    assert e.value.status == gs.GS_ERR_INVALID_ARG
    assert gs.gs_tile_grid(gs.make_camera(cam(), tile_cull=True)) == (8, 8)
    c = gs.make_camera(cam())
    c.tile_cull = 2
    with pytest.raises(gs.GsError) as e:
        gs.gs_tile_grid(c)
    assert e.value.status == gs.GS_ERR_INVALID_ARG


def test_camera_struct_layout(gs):
    import ctypes
    # float R[9], t[3], fx, fy, cx, cy; int32 width, height; float near_plane, eps2d; int32 tile_cull
    assert ctypes.sizeof(gs.gs_camera) == 4 * (9 + 3 + 4 + 2 + 2 + 1)
    assert gs.gs_camera.tile_cull.offset == 4 * 20


def test_invalid_arguments_rejected_before_launch(gs):
    L = gs.lib()
    c = gs.make_camera(cam())
    out = gs.gs_projected()
    # NULL params
    assert L.gs_project(None, C.byref(c), C.byref(out), None) == gs.GS_ERR_INVALID_ARG
    # unsupported SH degree
    p = gs.gs_params(16, 16, 16, 16, 16, 4, 10)
    assert L.gs_project(C.byref(p), C.byref(c), C.byref(out), None) == gs.GS_ERR_UNSUPPORTED
    assert "SH degree" in gs.gs_last_error_detail()
    # misaligned means
    p = gs.gs_params(16 + 4, 16, 16, 16, 16, 0, 10)
    assert L.gs_project(C.byref(p), C.byref(c), C.byref(out), None) == gs.GS_ERR_INVALID_ARG
    assert "aligned" in gs.gs_last_error_detail()
    # negative n
    p = gs.gs_params(16, 16, 16, 16, 16, 0, -1)
    assert L.gs_project(C.byref(p), C.byref(c), C.byref(out), None) == gs.GS_ERR_INVALID_ARG
    # NULL outputs of the projection
    p = gs.gs_params(16, 16, 16, 16, 16, 0, 10)
    assert L.gs_project(C.byref(p), C.byref(c), C.byref(out), None) == gs.GS_ERR_INVALID_ARG
    # Adam: step 0, misaligned buffers
    assert L.gs_adam(16, 16, 16, 16, 8, 1e-3, 0.9, 0.99, 1e-15, 0, None) == gs.GS_ERR_INVALID_ARG
    assert L.gs_adam(18, 16, 16, 16, 8, 1e-3, 0.9, 0.99, 1e-15, 1, None) == gs.GS_ERR_INVALID_ARG
    # bin sort: workspace too small, capacity out of range
    K = C.c_int64()
    proj = gs.gs_projected(16, 16, 16, 16, 16, 16, 16)
    assert L.gs_bin_sort(C.byref(proj), 10, C.byref(c), 256, 16, 256, 256, 100, C.byref(K), 256, None) == \
        gs.GS_ERR_INVALID_ARG
    assert "workspace" in gs.gs_last_error_detail()
    assert L.gs_bin_sort(C.byref(proj), 10, C.byref(c), 256, 1 << 30, 256, 256, -5, C.byref(K), 256, None) == \
        gs.GS_ERR_INVALID_ARG
    # densify buffers must come in pairs
    g2 = gs.gs_grad2d(16, 16, 16)
    gr = gs.gs_param_grads(16, 16, 16, 16, 16)
    p = gs.gs_params(16, 16, 16, 16, 16, 0, 10)
    assert L.gs_project_bwd(C.byref(p), C.byref(c), C.byref(proj), C.byref(g2), C.byref(gr), 256, None, None,
                            None) == gs.GS_ERR_INVALID_ARG
    # densify: no config, non-finite threshold, small workspace, moments not all given, n_out out of range
    cfg = gs.gs_densify_config(2e-4, 0.01, 0.005, 38)
    ws = gs.gs_densify_workspace_bytes(10)
    assert L.gs_densify_plan(C.byref(p), 256, 256, None, None, 256, ws, 256, 256, None) == gs.GS_ERR_INVALID_ARG
    bad = gs.gs_densify_config(float("nan"), 0.01, 0.005, 38)
    assert L.gs_densify_plan(C.byref(p), 256, 256, None, C.byref(bad), 256, ws, 256, 256, None) == \
        gs.GS_ERR_INVALID_ARG
    assert L.gs_densify_plan(C.byref(p), 256, 256, None, C.byref(cfg), 256, 8, 256, 256, None) == \
        gs.GS_ERR_INVALID_ARG
    assert "workspace" in gs.gs_last_error_detail()
    assert L.gs_densify_apply(C.byref(p), C.byref(p), None, 256, 256, 256, ws, 12, C.byref(gr), None, None,
                              None) == gs.GS_ERR_INVALID_ARG
    assert L.gs_densify_apply(C.byref(p), None, None, 256, 256, 256, ws, 21, C.byref(gr), None, None, None) == \
        gs.GS_ERR_INVALID_ARG
    assert "n_out" in gs.gs_last_error_detail()
    # batched depth order: view count bounds, small workspace, NULL order
    projs = (gs.gs_projected * 2)(proj, proj)
    wsd = gs.gs_depth_order_workspace_bytes(10, 2)
    assert wsd >= 4 * 4 * 10 * 2
    assert L.gs_depth_order_views(projs, 0, 10, 256, wsd, 256, None) == gs.GS_ERR_INVALID_ARG
    assert L.gs_depth_order_views(projs, 17, 10, 256, wsd, 256, None) == gs.GS_ERR_INVALID_ARG
    assert L.gs_depth_order_views(projs, 2, 10, 256, 16, 256, None) == gs.GS_ERR_INVALID_ARG
    assert "workspace" in gs.gs_last_error_detail()
    assert L.gs_depth_order_views(projs, 2, 10, 256, wsd, None, None) == gs.GS_ERR_INVALID_ARG
    # binning from an order: the order is required
    cnt = C.c_uint64()
    assert L.gs_bin_sort_ordered_async(C.byref(proj), 10, None, C.byref(c), 256, 1 << 30, 256, 256, 100, 256, 256,
                                       None) == gs.GS_ERR_INVALID_ARG
    assert "order" in gs.gs_last_error_detail()
    # the sparse Adam flag is 0 or 1
    lr = (C.c_float * 5)(1e-3, 1e-3, 1e-3, 1e-3, 1e-3)
    assert L.gs_project_bwd_views_adam(C.byref(p), 1, C.byref(c), C.byref(proj), C.byref(g2), C.byref(gr),
                                       C.byref(gr), C.byref(gr), lr, 0.9, 0.99, 1e-15, 1, None, None, None, None, 2,
                                       None) == gs.GS_ERR_INVALID_ARG
    # more views than the one-kernel form takes: the gradient buffer is required
    assert L.gs_project_bwd_views_adam(C.byref(p), gs.GS_ADAM_ONE_PASS_MAX_VIEWS + 1, C.byref(c), C.byref(proj),
                                       C.byref(g2), C.byref(gr), C.byref(gr), C.byref(gr), lr, 0.9, 0.99, 1e-15, 1,
                                       None, None, None, None, 0, None) == gs.GS_ERR_INVALID_ARG
    assert "grads" in gs.gs_last_error_detail()
    # packed projection: workspace size, capacity, the visible counter and the slot map
    wsp = gs.gs_project_packed_workspace_bytes(10)
    assert wsp >= 60 * 10
    packed = gs.gs_projected(16, 16, 16, 16, 16, 16, 16)
    cntp = 256
    assert L.gs_project_packed(C.byref(p), C.byref(c), 256, 8, C.byref(packed), 10, 256, 256, cntp, None) == \
        gs.GS_ERR_INVALID_ARG
    assert "workspace" in gs.gs_last_error_detail()
    assert L.gs_project_packed(C.byref(p), C.byref(c), 256, wsp, C.byref(packed), -1, 256, 256, cntp, None) == \
        gs.GS_ERR_INVALID_ARG
    assert L.gs_project_packed(C.byref(p), C.byref(c), 256, wsp, C.byref(packed), 10, 256, 256, None, None) == \
        gs.GS_ERR_INVALID_ARG
    assert L.gs_project_packed(C.byref(p), C.byref(c), 256, wsp, C.byref(packed), 10, 256, None, cntp, None) == \
        gs.GS_ERR_INVALID_ARG
    assert "slot_of" in gs.gs_last_error_detail()
    assert L.gs_project_packed(C.byref(p), C.byref(c), 256, wsp, C.byref(packed), 10, None, 256, cntp, None) == \
        gs.GS_ERR_INVALID_ARG
    # packed backward: the slot maps are required
    assert L.gs_project_bwd_views_packed(C.byref(p), 1, C.byref(c), C.byref(proj), None, C.byref(g2), C.byref(gr),
                                         None, None, None, None) == gs.GS_ERR_INVALID_ARG
    assert "slot_of" in gs.gs_last_error_detail()
    bad_slots = (C.c_void_p * 1)(258)
    assert L.gs_project_bwd_views_adam_packed(C.byref(p), 1, C.byref(c), C.byref(proj), bad_slots, C.byref(g2),
                                              C.byref(gr), C.byref(gr), C.byref(gr), lr, 0.9, 0.99, 1e-15, 1, None,
                                              None, None, None, 0, None) == gs.GS_ERR_INVALID_ARG
    assert "aligned" in gs.gs_last_error_detail()
    # 16-bit SH: negative count, misaligned input, missing half copy
    assert L.gs_to_half(256, -1, 256, None) == gs.GS_ERR_INVALID_ARG
    assert L.gs_to_half(260, 8, 256, None) == gs.GS_ERR_INVALID_ARG
    assert "aligned" in gs.gs_last_error_detail()
    assert L.gs_to_half(None, 0, None, None) == gs.GS_OK
    p_nosh = gs.gs_params(16, 16, 16, 16, None, 3, 10)
    assert L.gs_project_sh16(C.byref(p_nosh), None, C.byref(c), C.byref(packed), None) == gs.GS_ERR_INVALID_ARG
    assert "sh_half" in gs.gs_last_error_detail()
    assert L.gs_project_bwd_views_adam_sh16(C.byref(p), 1, C.byref(c), C.byref(proj), C.byref(g2), None, 256,
                                            C.byref(gr), C.byref(gr), C.byref(gr), lr, 0.9, 0.99, 1e-15, 1, None,
                                            None, None, None, 0, None) == gs.GS_ERR_INVALID_ARG
    # D-SSIM: image size limits and workspace
    assert L.gs_l1_dssim_loss_grad(256, 256, 0, 10, 1.0, 0.2, 256, 1 << 20, 256, 256, None) == gs.GS_ERR_UNSUPPORTED
    assert L.gs_l1_dssim_loss_grad(256, 256, 10, 10, 1.0, 0.2, 256, 8, 256, 256, None) == gs.GS_ERR_INVALID_ARG
    assert gs.gs_l1_dssim_workspace_bytes(10, 10) >= 72 * 100
    # zero-size work needs no pointers and launches nothing
    assert L.gs_adam(None, None, None, None, 0, 1e-3, 0.9, 0.99, 1e-15, 1, None) == gs.GS_OK
    assert L.gs_l1_loss_grad(None, None, 0, None, None, None) == gs.GS_OK
    assert L.gs_zero(None, 0, None) == gs.GS_OK


def test_workspace_grows_with_capacity(gs):
    c = gs.make_camera(cam())
    a = gs.gs_bin_sort_workspace_bytes(1000, 10_000, c)
    b = gs.gs_bin_sort_workspace_bytes(1000, 1_000_000, c)
    assert 0 < a < b
    assert b >= 12 * 1_000_000          # the ping-pong key/value copy


def test_culled_binning_workspace(gs):
    """The culled binning keeps, per Gaussian, the runs of its first 8 rows (32 bytes)
    and its count (4 bytes): exactly that much more workspace, each region aligned to
    256 bytes; a NULL camera means no culling."""
    for n in (1, 1000, 1_000_000):
        plain = gs.gs_bin_sort_workspace_bytes(n, 10 * n, gs.make_camera(cam()))
        culled = gs.gs_bin_sort_workspace_bytes(n, 10 * n, gs.make_camera(cam(), tile_cull=True))
        up = lambda x: (x + 255) // 256 * 256
        assert culled - plain == up(32 * n) + up(4 * n), n
        assert gs.lib().gs_bin_sort_workspace_bytes(n, 10 * n, None) == plain


def test_binding_argument_counts_match_the_header(gs):
    """Every prototype of include/gs.h takes as many parameters as the ctypes binding
    passes (a missing or extra argument would be undefined behaviour at the call)."""
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    decls = re.findall(r"\b(?:gs_status|size_t|int32_t|int64_t|uint64_t|const char\s*\*)\s+(gs_[a-z0-9_]+)\s*\(([^;]*?)\)\s*;",
                       text, flags=re.S)
    assert {name for name, _ in decls} == set(declared_functions())
    for name, params in decls:
        p = params.strip()
        n = 0 if p in ("", "void") else p.count(",") + 1
        assert n == len(gs.SIGNATURES[name][1]), (name, n, len(gs.SIGNATURES[name][1]))


def test_static_scratch_size_matches_the_header(gs):
    """The binding's GS_STATIC_SCRATCH_BYTES is the header's #define, not a stale copy."""
    text = open(HEADER).read()
    m = re.search(r"#define\s+GS_STATIC_SCRATCH_BYTES\s+\(\(size_t\)\s*(\d+)\s*<<\s*(\d+)\)", text)
    assert m, "GS_STATIC_SCRATCH_BYTES not found in gs.h"
    assert int(m.group(1)) << int(m.group(2)) == gs.GS_STATIC_SCRATCH_BYTES


def test_static_scratch_limit_is_checked_at_the_boundary(gs):
    """gs_bin_sort_static rejects, before it touches a device, the smallest capacity whose
    workspace exceeds the static scratch, and lets the largest one that fits through to
    its next checks (here the missing device or the NULL buffers, never the size)."""
    c = gs.make_camera(cam())
    n = 1000
    lo, hi = 1, 1 << 26   # workspace(lo) fits, workspace(hi) does not
    assert gs.gs_bin_sort_workspace_bytes(n, lo, c) <= gs.GS_STATIC_SCRATCH_BYTES
    assert gs.gs_bin_sort_workspace_bytes(n, hi, c) > gs.GS_STATIC_SCRATCH_BYTES
    while hi - lo > 1:
        mid = (lo + hi) // 2
        if gs.gs_bin_sort_workspace_bytes(n, mid, c) <= gs.GS_STATIC_SCRATCH_BYTES:
            lo = mid
        else:
            hi = mid
    proj = gs.gs_projected()
    K = C.c_int64(0)
    L = gs.lib()
    st = L.gs_bin_sort_static(C.byref(proj), n, C.byref(c), None, None, hi, C.byref(K), None, None)
    assert st == gs.GS_ERR_UNSUPPORTED
    assert "static scratch" in L.gs_last_error_detail().decode()
    st = L.gs_bin_sort_static(C.byref(proj), n, C.byref(c), None, None, lo, C.byref(K), None, None)
    assert st not in (gs.GS_OK, gs.GS_ERR_UNSUPPORTED)


def test_alu_probe_argument_checks(gs):
    L = gs.lib()
    ops = C.c_double(0.0)
    slots = gs.gs_alu_probe_slots()
    assert slots == 148 * 8 * 256
    assert L.gs_alu_probe(7, 10, C.c_void_p(256), slots, C.byref(ops), None) == gs.GS_ERR_INVALID_ARG
    assert L.gs_alu_probe(gs.GS_PROBE_EX2, 0, C.c_void_p(256), slots, C.byref(ops), None) == gs.GS_ERR_INVALID_ARG
    assert L.gs_alu_probe(gs.GS_PROBE_EX2, 10, None, slots, C.byref(ops), None) == gs.GS_ERR_INVALID_ARG
    assert L.gs_alu_probe(gs.GS_PROBE_FFMA, 10, C.c_void_p(256), slots - 1, C.byref(ops), None) == \
        gs.GS_ERR_INVALID_ARG
    assert "needed" in L.gs_last_error_detail().decode()


def test_counted_raster_calls_check_their_counter(gs):
    L = gs.lib()
    c = gs.make_camera(cam())
    proj = gs.gs_projected()
    bg = (C.c_float * 3)(0, 0, 0)
    st = L.gs_raster_fwd_counted(C.byref(proj), None, None, None, C.byref(c), bg, None, None, None, None, None)
    assert st == gs.GS_ERR_INVALID_ARG and "counts" in L.gs_last_error_detail().decode()
    st = L.gs_raster_bwd_counted(C.byref(proj), None, None, None, C.byref(c), bg, None, None, None, None, None, None)
    assert st == gs.GS_ERR_INVALID_ARG and "counts" in L.gs_last_error_detail().decode()


@pytest.mark.parametrize("name", ["GS_MAX_VIEWS", "GS_ADAM_ONE_PASS_MAX_VIEWS"])
def test_view_limits_match_the_header(gs, name):
    """The binding's view limits are the header's #defines, not stale copies."""
    m = re.search(r"#define\s+%s\s+(\d+)\b" % name, open(HEADER).read())
    assert m, f"{name} not found in gs.h"
    assert int(m.group(1)) == getattr(gs, name)
