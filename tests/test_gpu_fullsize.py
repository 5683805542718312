"""The two largest workloads at their stated sizes, through the C ABI, against
the float64 oracle on sampled outputs (`-m gpu`):

* 6,000,000 Gaussians seen by 8 views of 1920x1080 with 64-bit
  (tile << 32 | depth) sort keys, about 1e9 Gaussian x tile pairs: the pair
  count, the per-tile lists of sampled tiles bit for bit, sampled pixels, the
  screen-space and parameter gradients of an upstream gradient on those
  pixels, and the densify statistics summed over the views;
* 10,000,000 Gaussians at 3840x2160 with the fused Adam step: the same, plus
  the Adam state of every Gaussian after one step.

The oracle works one view at a time (a view's float64 projection of every
Gaussian, then the sampled tiles and pixels of that view) and differentiates
the projection only for the Gaussians the sampled pixels reach. The
comparator is the parity tests' (tests/parity.py).
"""

import numpy as np
import pytest
import torch

from gaussian_splatting_differentiable_ewa_b200 import api
from gaussian_splatting_differentiable_ewa_b200 import scenes as S
from gaussian_splatting_differentiable_ewa_b200.pipeline import Splatter
from oracle import oracle as O

import parity as P

pytestmark = pytest.mark.gpu


def _sample(W, H, v, n_random, rng):
    xs = rng.integers(0, W, n_random)
    ys = rng.integers(0, H, n_random)
    r = int(rng.integers(0, (H + 15) // 16))
    yy, xx = np.meshgrid(np.arange(r * 16, min(H, r * 16 + 16)), np.arange(W), indexing="ij")
    pix = np.concatenate([np.stack([np.full(n_random, v), xs, ys], 1),
                          np.stack([np.full(xx.size, v), xx.ravel(), yy.ravel()], 1)])
    _, idx = np.unique(pix, axis=0, return_index=True)
    return pix[np.sort(idx)].astype(np.int32)


def _check_view(sc, sp, v, proj, ids, ranges, rng, n_pix):
    """Binning, render and render-backward checks of view v; returns the
    sampled pixels, the oracle's screen-space gradient rows of the Gaussians
    they reach, and those Gaussians' indices."""
    cam = sc.cameras[v]
    tx, ty = (cam.width + 15) // 16, (cam.height + 15) // 16
    tpv = tx * ty
    amb = proj["ambiguous"] != 0
    assert amb.mean() < 1e-4
    # per-tile lists: random tiles plus the 16 longest of the view
    lens = ranges[v * tpv:(v + 1) * tpv, 1] - ranges[v * tpv:(v + 1) * tpv, 0]
    tiles = np.unique(np.concatenate([rng.integers(0, tpv, 48), np.argsort(lens)[-16:]]))
    req = np.stack([np.zeros(len(tiles), np.int32), tiles.astype(np.int32)], 1)
    counts, oids = O.tile_lists(proj["rect"][None], proj["key"][None], [(tx, ty)], req)
    off = 0
    for k, t in enumerate(tiles):
        want = oids[off:off + counts[k]]
        off += counts[k]
        s, e = ranges[v * tpv + t]
        got = ids[int(s):int(e)].cpu().numpy()  # the tile's slice only (ids can be GBs)
        assert np.array_equal(got.astype(np.int64), want.astype(np.int64)), (v, t)
    # sampled pixels of this view
    pix = _sample(cam.width, cam.height, 0, n_pix, rng)
    bound = P.alpha_error_bound([proj])
    ref = O.render([proj], [cam], sc.background, pix, alpha_err=bound)
    img = sp.image[v].cpu().numpy()[None]
    fT = sp.final_T[v].cpu().numpy()[None]
    nc = sp.n_contrib[v].cpu().numpy()[None]
    st = P.compare_render(img, fT, nc, ref, pix, P.colour_max([proj], sc.background))
    print("view", v, st, "evaluations per pixel %.1f" % ref["n_exp"].mean())
    assert st["flagged"] <= P.FLAG_RATE * ref["n_exp"].sum()
    assert st["max_abs"] <= P.MAX_ABS and st["mean_abs"] <= P.MEAN_ABS
    assert st["nc_mismatch"] == 0 and st["T_max_rel"] < 1e-3
    assert st["flagged_excess"] <= 0.0 and st["flagged_T_excess"] <= 0.0
    return pix


def _upstream(sc, pix_by_view):
    c = sc.cameras[0]
    dL = S.make_upstream_grad(sc.n_views, c.height, c.width, seed=1)
    mask = np.zeros_like(dL)
    for v, pix in enumerate(pix_by_view):
        mask[v, :, pix[:, 2], pix[:, 1]] = 1.0
    return dL * mask


def _run_case(name, mode, n_pix, adam):
    sc = S.make_scene(name)
    sp = Splatter(sc, sort_mode=mode)
    need = sp.ensure_capacity()
    sp.rasterize_fwd()
    torch.cuda.synchronize()
    assert sp.status() == api.GS_OK
    n_pairs = int(sp.n_pairs.item())
    assert n_pairs == need
    print(name, "pairs", n_pairs)
    ids = sp.ids
    ranges = sp.ranges.cpu().numpy()
    rng = np.random.default_rng(17)
    total = 0
    pix_by_view, valid = [], []
    for v, cam in enumerate(sc.cameras):
        proj = O.project(sc, cam)
        valid.append(proj["valid"].astype(np.int32))
        r = proj["rect"].astype(np.int64)
        total += int(((r[:, 1] - r[:, 0] + 1) * (r[:, 3] - r[:, 2] + 1))[proj["valid"] != 0].sum())
        pix_by_view.append(_check_view(sc, sp, v, proj, ids, ranges, rng, n_pix))
        del proj
    assert n_pairs == total
    # backward of an upstream gradient on the sampled pixels
    dL = _upstream(sc, pix_by_view)
    sp.rasterize_bwd(torch.as_tensor(dL).cuda())
    sp.densify_stats()
    p0 = {k: t.clone() for k, t in sp.param_list} if adam else None
    if adam:
        sp.adam_step()
    torch.cuda.synchronize()
    assert sp.status() == api.GS_OK
    sparse = []  # per view: (indices of the Gaussians reached, their rows)
    for v, cam in enumerate(sc.cameras):
        proj = O.project(sc, cam)
        pix = pix_by_view[v]
        g = O.render_bwd([proj], [cam], sc.background, pix,
                         dL[v][:, pix[:, 2], pix[:, 1]].T)[0]
        nz = np.nonzero(np.any(g != 0, axis=1))[0]
        sparse.append((nz, g[nz]))
        del proj, g
    touched = np.unique(np.concatenate([nz for nz, _ in sparse]))
    assert len(touched) > 1000
    g2_ref = np.zeros((sc.n_views, len(touched), 10))       # [V, m, 10]
    for v, (nz, rws) in enumerate(sparse):
        g2_ref[v, np.searchsorted(touched, nz)] = rws
    del sparse
    g2_gpu = sp.grad2d[:, torch.as_tensor(touched).cuda()].cpu().numpy()
    for f in range(10):
        e = P.rel_l2(g2_gpu[..., f], g2_ref[..., f])
        assert e < P.REL_L2, ("grad2d field", f, e)
    # parameter gradients of the touched Gaussians (every other one is 0)
    import copy
    sub = copy.copy(sc)
    for k in ("means", "log_scales", "quats", "opacity_logit", "sh"):
        setattr(sub, k, np.ascontiguousarray(getattr(sc, k)[touched]))
    projs_sub = O.project_views(sub)
    gr = O.project_bwd(sub, projs_sub, g2_ref)
    tt = torch.as_tensor(touched).cuda()
    for k, t in sp.grads.items():
        gpu = t[tt].cpu().numpy()
        if k in ("means", "log_scales"):
            gpu = gpu[:, :3]
        e = P.rel_l2(gpu.reshape(gr[k].shape), gr[k])
        assert e < P.REL_L2, (k, e)
        keep = torch.ones(t.shape[0], dtype=torch.bool, device="cuda")
        keep[tt] = False
        assert not t[keep].any(), k
    # densify statistics summed over the views
    plain, absg, _ = O.densify_stats(g2_ref, np.stack(valid)[:, touched])
    assert P.rel_l2(sp.accum_plain[tt].cpu().numpy(), plain) < P.REL_L2
    assert P.rel_l2(sp.accum_abs[tt].cpu().numpy(), absg) < P.REL_L2
    assert np.array_equal(sp.denom.cpu().numpy(), np.stack(valid).sum(0))
    if adam:
        # one Adam step from zero moments: the touched Gaussians against the
        # oracle's Adam on the oracle's gradient; every other parameter keeps
        # its value and zero moments (g = 0)
        for k, t in sp.param_list:
            g = gr[k].reshape(len(touched), -1)
            p = p0[k][tt].cpu().numpy().astype(np.float64).reshape(len(touched), -1)[:, :g.shape[1]]
            rp, rm, rv = O.adam(p, g, np.zeros_like(g), np.zeros_like(g), sp.lr[k], 1)
            m_gpu = sp.exp_avg[k][tt].cpu().numpy().reshape(len(touched), -1)[:, :g.shape[1]]
            v_gpu = sp.exp_avg_sq[k][tt].cpu().numpy().reshape(len(touched), -1)[:, :g.shape[1]]
            p_gpu = t[tt].cpu().numpy().reshape(len(touched), -1)[:, :g.shape[1]]
            assert P.rel_l2(m_gpu, rm) < P.REL_L2, k
            assert P.rel_l2(v_gpu, rv) < P.REL_L2, k
            big = np.abs(g) > 1e-3 * np.sqrt(np.mean(g * g) + 1e-300)
            assert P.rel_l2((p_gpu - p)[big], (rp - p)[big]) < P.REL_L2, k
            keep = torch.ones(t.shape[0], dtype=torch.bool, device="cuda")
            keep[tt] = False
            assert torch.equal(t[keep], p0[k][keep]), k
            assert not sp.exp_avg[k][keep].any() and not sp.exp_avg_sq[k][keep].any(), k


def test_six_million_gaussians_eight_views_64bit_keys():
    _run_case("train_6m_8x1080p", api.GS_SORT_FULL64, n_pix=1024, adam=False)


def test_ten_million_gaussians_4k_with_adam():
    _run_case("train_10m_4k", api.GS_SORT_PRESORT, n_pix=2048, adam=True)
