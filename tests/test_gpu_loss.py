"""The fused L1 + D-SSIM loss kernel (through the C ABI) against the float64
oracle on seeded image pairs: whole images at sizes that span several 32 x 32
tiles with ragged edges, images smaller than the window, and the benchmark's
1080p frame on sampled crops plus its full-image loss terms.

Tolerances: the loss terms within 2e-6 absolute (float32 window sums, double
accumulation); the gradient within 1e-4 relative L2 and each value within
1e-3 of the largest magnitude (the gradient bar is 1e-3 relative L2).
"""

import numpy as np
import pytest
import torch

from gaussian_splatting_differentiable_ewa_b200 import api
from gaussian_splatting_differentiable_ewa_b200 import scenes as S
from gaussian_splatting_differentiable_ewa_b200.pipeline import Splatter
from oracle import oracle as O

pytestmark = pytest.mark.gpu


def _run(img, tgt, lam=0.2, grad=True):
    V, _, H, W = img.shape
    x = torch.from_numpy(img).cuda()
    y = torch.from_numpy(tgt).cuda()
    terms = torch.full((V, 3), float("nan"), dtype=torch.float64, device="cuda")
    g = torch.full_like(x, float("nan")) if grad else None
    nb = api.gs_l1_dssim_workspace_size(V)
    ws = torch.full(((nb + 7) // 8,), 123.0, dtype=torch.float64, device="cuda")
    api.gs_l1_dssim(x, y, V, H, W, lam, terms, g, ws)
    torch.cuda.synchronize()
    return terms.cpu().numpy(), (g.cpu().numpy() if grad else None)


def _check_grad(got, want):
    rel = np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-300)
    assert rel < 1e-4, rel
    assert np.abs(got - want).max() <= 1e-3 * np.abs(want).max()


@pytest.mark.parametrize("V,H,W", [(2, 70, 100), (1, 33, 65), (1, 5, 7), (1, 1, 1),
                                   (3, 64, 96), (1, 200, 40)])
def test_loss_matches_oracle(V, H, W):
    img, tgt = S.make_image_pair(V, H, W, seed=H * 1000 + W)
    terms, g = _run(img, tgt)
    want_t, want_g = O.l1_dssim_loss(img, tgt)
    np.testing.assert_allclose(terms, want_t, rtol=0, atol=2e-6)
    _check_grad(g, want_g)


@pytest.mark.parametrize("lam", [0.0, 1.0, 0.5])
def test_loss_weights_and_forward_only(lam):
    img, tgt = S.make_image_pair(2, 48, 80, seed=11)
    terms, g = _run(img, tgt, lam)
    want_t, want_g = O.l1_dssim_loss(img, tgt, lam)
    np.testing.assert_allclose(terms, want_t, rtol=0, atol=2e-6)
    _check_grad(g, want_g)
    t2, none = _run(img, tgt, lam, grad=False)
    assert none is None
    # the same sums in another instantiation and atomic order: float32 noise only
    np.testing.assert_allclose(t2, terms, rtol=0, atol=2e-6)


def test_loss_of_identical_images():
    img, _ = S.make_image_pair(1, 40, 50, seed=12)
    terms, g = _run(img, img.copy())
    np.testing.assert_allclose(terms, [[0.0, 0.0, 1.0]], atol=2e-6)
    # the SSIM gradient vanishes at x == y up to float32 rounding, small
    # against the gradient's scale 1/N, and the L1 subgradient there is 0
    assert np.abs(g).max() < 1e-3 / img.size


def test_loss_rejects_bad_arguments_and_accepts_no_views():
    x = torch.zeros((1, 3, 8, 8), device="cuda")
    terms = torch.zeros((1, 3), dtype=torch.float64, device="cuda")
    ws = torch.zeros(8, dtype=torch.float64, device="cuda")
    for args in [(1, 0, 8, 0.2), (1, 8, 0, 0.2), (1, 8, 8, 1.5), (1, 8, 8, -0.1),
                 (21846, 8, 8, 0.2)]:
        with pytest.raises(api.GsError):
            api.gs_l1_dssim(x, x, args[0], args[1], args[2], args[3], terms, None, ws)
    small = torch.zeros(1, dtype=torch.float64, device="cuda")
    with pytest.raises(api.GsError):
        api.gs_l1_dssim(x, x, 1, 8, 8, 0.2, terms, None, small)
    api.gs_l1_dssim(x, x, 0, 8, 8, 0.2, terms, None, ws)


def test_loss_full_1080p_terms_and_sampled_crops():
    """The benchmark's frame size: the full-image loss terms against the
    oracle's, and the gradient on crops: SSIM is local (radius 5 window,
    radius 10 for the gradient), so a crop grown by 10 pixels, or reaching the
    image border, gives the oracle's values inside it, scaled from the
    crop's pixel count to the frame's."""
    H, W = 1080, 1920
    img, tgt = S.make_image_pair(1, H, W, seed=5)
    terms, g = _run(img, tgt)
    ssim = O.ssim_map(img, tgt).mean()
    l1 = np.abs(img.astype(np.float64) - tgt).mean()
    np.testing.assert_allclose(terms[0], [0.8 * l1 + 0.2 * (1 - ssim), l1, ssim],
                               rtol=0, atol=2e-6)
    rng = np.random.default_rng(9)
    crops = [(0, 0), (H - 64, W - 64), (0, W - 64), (H - 64, 0)]
    crops += [(int(rng.integers(0, H - 64)), int(rng.integers(0, W - 64))) for _ in range(4)]
    N = 3.0 * H * W
    for (y0, x0) in crops:
        ya, yb = max(0, y0 - 10), min(H, y0 + 64 + 10)
        xa, xb = max(0, x0 - 10), min(W, x0 + 64 + 10)
        _, gc = O.l1_dssim_loss(img[:, :, ya:yb, xa:xb], tgt[:, :, ya:yb, xa:xb])
        gc *= 3.0 * (yb - ya) * (xb - xa) / N
        want = gc[:, :, y0 - ya:y0 - ya + 64, x0 - xa:x0 - xa + 64]
        _check_grad(g[:, :, y0:y0 + 64, x0:x0 + 64], want)


def test_training_on_a_rendered_target_lowers_the_loss():
    """A real training step: targets rendered by the oracle from one scene,
    the Splatter starting from the same scene with its colours and opacities
    disturbed; thirty steps of render, loss, backward and Adam must lower the
    loss well below its start."""
    sc = S.make_scene("fwd_1k_128")
    outs = O.render_all(sc)
    V = len(sc.cameras)
    H, W = sc.cameras[0].height, sc.cameras[0].width
    tgt = np.stack([o[1]["color"].reshape(H, W, 3).transpose(2, 0, 1) for o in outs])
    tgt = torch.from_numpy(np.ascontiguousarray(tgt, np.float32)).cuda()
    rng = np.random.default_rng(1)
    sc2 = S.make_scene("fwd_1k_128")
    sc2.sh[:, 0, :] += rng.normal(0, 0.2, size=sc2.sh[:, 0, :].shape).astype(np.float32)
    sc2.opacity_logit[:] += rng.normal(0, 0.5, size=sc2.opacity_logit.shape).astype(np.float32)
    sp = Splatter(sc2, lr=dict(means=1.6e-4, sh=1e-2, opacity_logit=5e-2, log_scales=5e-3,
                               quats=1e-3))
    sp.ensure_capacity()
    first = None
    for _ in range(30):
        sp.train_step_target(tgt)
        if first is None:
            first = sp.loss_terms.cpu().numpy()[:, 0].copy()
    sp.forward()
    last = sp.loss(tgt, grad=False).cpu().numpy()[:, 0]
    assert sp.status() == api.GS_OK
    assert np.all(last < 0.85 * first), (first, last)
