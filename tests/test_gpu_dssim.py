"""Parity of the L1 + D-SSIM loss (gs_l1_dssim_loss_grad) with the oracle: the loss
to 1e-12 relative, dL/dimage (computed in double on both sides, rounded once to
float32 on the device) within one float32 ulp of the oracle's value plus 1e-13 of
the largest gradient; ragged and tiny images, identical images, the Trainer with
the D-SSIM term."""
import numpy as np
import pytest
import torch

from gaussian_splatting_differentiable_02_b200 import abi, scenes
from gaussian_splatting_differentiable_02_b200 import pipeline as pl

pytestmark = pytest.mark.gpu


def _gpu(img, tgt, l1w=1.0, sw=0.2):
    H, W, _ = img.shape
    x = torch.from_numpy(np.ascontiguousarray(img, np.float32)).cuda()
    y = torch.from_numpy(np.ascontiguousarray(tgt, np.float32)).cuda()
    g = torch.empty_like(x)
    loss = torch.zeros((1,), device="cuda", dtype=torch.float64)
    nb = abi.gs_l1_dssim_workspace_bytes(W, H)
    ws = torch.empty((nb,), device="cuda", dtype=torch.uint8)
    abi.gs_l1_dssim_loss_grad(x.data_ptr(), y.data_ptr(), W, H, l1w, sw, ws.data_ptr(), nb, g.data_ptr(),
                              loss.data_ptr(), torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    return float(loss.item()), g.cpu().numpy()


def _compare(orc, img, tgt, l1w=1.0, sw=0.2):
    loss, g = _gpu(img, tgt, l1w, sw)
    # the weights cross the C boundary as float32
    want_loss, want_g = orc.l1_dssim(img.astype(np.float32).astype(np.float64),
                                     tgt.astype(np.float32).astype(np.float64), float(np.float32(l1w)),
                                     float(np.float32(sw)))
    assert abs(loss - want_loss) <= 1e-12 * max(1.0, abs(want_loss)), (loss, want_loss)
    w32 = want_g.astype(np.float32)
    ulp = np.spacing(np.abs(w32)).astype(np.float64)
    err = np.abs(g.astype(np.float64) - want_g)
    bound = ulp + 1e-13 * np.max(np.abs(want_g))
    assert np.all(err <= bound), float(np.max(err / bound))
    return loss


@pytest.mark.parametrize("shape", [(37, 53), (8, 32), (1, 1), (3, 200), (130, 7)])
def test_random_images(orc, shape):
    rng = np.random.default_rng(shape[0] * 1000 + shape[1])
    img = rng.random((*shape, 3)).astype(np.float32)
    tgt = np.clip(img + 0.2 * rng.standard_normal(img.shape), 0, 1).astype(np.float32)
    _compare(orc, img, tgt)


def test_weights_and_dark_regions(orc):
    """Dark, nearly flat regions make the SSIM partial derivatives large (1/C1)."""
    rng = np.random.default_rng(3)
    img = (0.002 * rng.random((64, 96, 3))).astype(np.float32)
    img[20:40, 30:70] += 0.8
    tgt = (0.002 * rng.random((64, 96, 3))).astype(np.float32)
    _compare(orc, img, tgt, 0.8, 0.2)
    _compare(orc, img, tgt, 0.0, 1.0)


def test_identical_images_give_zero():
    rng = np.random.default_rng(4)
    img = rng.random((45, 61, 3)).astype(np.float32)
    loss, g = _gpu(img, img)
    assert loss == 0.0
    # the partial derivative with respect to the windowed mean cancels to rounding
    # (four terms summed in order), so the gradient is zero up to that
    assert np.max(np.abs(g)) < 1e-15


def test_full_hd_rendered_image(orc):
    """A rendered 1920x1080 view of the 1M mixture against a U[0, 1] target."""
    wl = scenes.multiview1m(views=1)
    g = pl.Gaussians.from_scene(wl.scene)
    view = pl.View(wl.scene.n, wl.cameras[0])
    proj = pl.Projected(wl.scene.n)
    pl.project(g, view, proj)
    pl.bin_sort(proj, view)
    pl.raster_fwd(proj, view)
    torch.cuda.synchronize()
    img = view.image.cpu().numpy()
    _compare(orc, img, wl.targets[0])


def test_trainer_with_dssim():
    rng = np.random.default_rng(5)
    scene = scenes.random_scene(rng, 700, 1, mean_box=1.0, log_scale=(-4.0, -2.5))
    R, t = scenes.look_at((0.0, 0.0, -4.0))
    cam = scenes.camera(R, t, 128.0, 128.0, 64.0, 64.0, 128, 128)
    target = torch.from_numpy(rng.random((128, 128, 3)).astype(np.float32)).cuda()
    lrs = {"means": 1.6e-4, "log_scales": 5e-3, "quats": 1e-3, "opacity_logits": 5e-2, "sh": 2.5e-3}
    tr = pl.Trainer(pl.Gaussians.from_scene(scene), [pl.View(scene.n, cam)], [target], lrs, ssim_weight=0.2)
    losses = []
    for _ in range(5):
        tr.step()
        losses.append(tr.loss.item())
    assert all(np.isfinite(losses)) and losses[-1] < losses[0]
