"""Python face of the float64 CPU oracle (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this module. It loads ``liboracle.so`` built from
``gs_oracle.cpp`` (see ``build.py``) and adds the two steps whose definitions
are one line each -- the view-space gradient statistics and Adam -- written in
numpy float64.

Every array crossing this interface is float64 (inputs are the float32 scene
arrays widened exactly), except the float32 depth keys and the int32 flags.
"""

from __future__ import annotations

import ctypes
import os
from typing import Dict, List, Optional, Sequence

import numpy as np

from . import build as _build

_LIB = None

_D = ctypes.POINTER(ctypes.c_double)
_F = ctypes.POINTER(ctypes.c_float)
_I32 = ctypes.POINTER(ctypes.c_int32)
_I64 = ctypes.POINTER(ctypes.c_int64)
_U64 = ctypes.POINTER(ctypes.c_uint64)


def lib():
    """Load (building first if needed) the oracle shared library."""
    global _LIB
    if _LIB is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        L.orc_sh_basis.argtypes = [ctypes.c_int64, _D, ctypes.c_int, _D]
        L.orc_project.argtypes = [ctypes.c_int64, _D, _D, _D, _D, _D, ctypes.c_int, _D,
                                  ctypes.c_double, _D, _I32, _F]
        L.orc_tile_lists.argtypes = [ctypes.c_int, ctypes.c_int64, _I32, _F, _I32, _I32,
                                     ctypes.c_int64, _I32, _I64, _I32]
        L.orc_render.argtypes = [ctypes.c_int, ctypes.c_int64, _D, _F, _I32, _I32, ctypes.c_int64,
                                 _I32, _D, ctypes.c_double, ctypes.c_double, _D, _D, _D, _I32,
                                 _I32, _I64, _I32, _U64, _D, _D]
        L.orc_render_bwd.argtypes = [ctypes.c_int, ctypes.c_int64, _D, _F, _I32, _I32,
                                     ctypes.c_int64, _I32, _D, _D, _D]
        L.orc_project_bwd.argtypes = [ctypes.c_int64, _D, _D, _D, _D, _D, ctypes.c_int,
                                      ctypes.c_int, _D, _I32, _D, _D, _D, _D, _D, _D]
        L.orc_num_threads.restype = ctypes.c_int
        _LIB = L
    return _LIB


def num_threads() -> int:
    return int(lib().orc_num_threads())


def _p(a: np.ndarray, t):
    return a.ctypes.data_as(t)


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def pack_camera(cam) -> np.ndarray:
    """22 doubles: viewmat (3x4 row-major), fx, fy, cx, cy, W, H, campos, 0."""
    c = cam if isinstance(cam, dict) else cam.as_dict()
    out = np.zeros(22, np.float64)
    out[:12] = np.asarray(c["viewmat"], np.float32).astype(np.float64).reshape(12)
    out[12:16] = [np.float32(c["fx"]), np.float32(c["fy"]), np.float32(c["cx"]), np.float32(c["cy"])]
    out[16:18] = [c["width"], c["height"]]
    out[18:21] = np.asarray(c["campos"], np.float32).astype(np.float64)
    return out


def sh_basis(dirs: np.ndarray, deg: int) -> np.ndarray:
    """Real SH basis [n, 16] (Legendre recursion) for unit directions [n, 3]."""
    d = _f64(dirs)
    n = d.shape[0]
    out = np.zeros((n, 16), np.float64)
    lib().orc_sh_basis(n, _p(d, _D), int(deg), _p(out, _D))
    return out


def _raw(scene):
    n = scene.n
    k = (scene.sh_degree + 1) ** 2
    return (_f64(scene.means[:, :3]), _f64(scene.log_scales[:, :3]), _f64(scene.quats),
            _f64(scene.opacity_logit), _f64(scene.sh.reshape(n, k, 3)))


def project(scene, cam, tol: float = 1e-12) -> Dict[str, np.ndarray]:
    """Project every Gaussian of ``scene`` into ``cam`` (float64)."""
    m, s, q, lg, sh = _raw(scene)
    n = scene.n
    geom = np.zeros((n, 16), np.float64)
    ints = np.zeros((n, 8), np.int32)
    key = np.zeros(n, np.float32)
    lib().orc_project(n, _p(m, _D), _p(s, _D), _p(q, _D), _p(lg, _D), _p(sh, _D),
                      int(scene.sh_degree), _p(pack_camera(cam), _D), float(tol),
                      _p(geom, _D), _p(ints, _I32), _p(key, _F))
    return dict(
        xy=geom[:, 0:2].copy(), depth=geom[:, 2].copy(), cov=geom[:, 3:6].copy(),
        conic=geom[:, 6:9].copy(), opacity=geom[:, 9].copy(), rgb=geom[:, 10:13].copy(),
        lam=geom[:, 13].copy(), radius_arg=geom[:, 14].copy(),
        valid=ints[:, 0].copy(), radius=ints[:, 1].copy(), rect=ints[:, 2:6].copy(),
        clamp=ints[:, 6].copy(), ambiguous=ints[:, 7].copy(), key=key)


def project_views(scene, tol: float = 1e-12) -> List[Dict[str, np.ndarray]]:
    return [project(scene, c, tol) for c in scene.cameras]


def _stack_views(projs: Sequence[dict]):
    g2d = np.ascontiguousarray(np.stack([np.concatenate(
        [p["xy"], p["conic"], p["opacity"][:, None], p["rgb"]], axis=1) for p in projs]))
    keys = np.ascontiguousarray(np.stack([p["key"] for p in projs]).astype(np.float32))
    rects = np.ascontiguousarray(np.stack([p["rect"] for p in projs]).astype(np.int32))
    return g2d, keys, rects


def _dims(cams) -> np.ndarray:
    out = []
    for c in cams:
        c = c if isinstance(c, dict) else c.as_dict()
        out.append([c["width"], c["height"]])
    return np.ascontiguousarray(np.asarray(out, np.int32))


def tile_lists(rects: np.ndarray, keys: np.ndarray, tiles_xy: Sequence, requests: np.ndarray):
    """Sorted Gaussian ids of the requested (view, tile) pairs.

    ``rects`` int32 [V, n, 4]; ``keys`` float32 [V, n]; ``tiles_xy`` [(tx, ty)]
    per view; ``requests`` int32 [R, 2]. Returns (counts [R], ids concatenated).
    """
    rects = np.ascontiguousarray(rects, np.int32)
    keys = np.ascontiguousarray(keys, np.float32)
    V, n = keys.shape
    tx = np.ascontiguousarray([t[0] for t in tiles_xy], np.int32)
    ty = np.ascontiguousarray([t[1] for t in tiles_xy], np.int32)
    req = np.ascontiguousarray(requests, np.int32)
    R = req.shape[0]
    counts = np.zeros(R, np.int64)
    lib().orc_tile_lists(V, n, _p(rects, _I32), _p(keys, _F), _p(tx, _I32), _p(ty, _I32), R,
                         _p(req, _I32), _p(counts, _I64), None)
    ids = np.zeros(max(int(counts.sum()), 1), np.int32)
    lib().orc_tile_lists(V, n, _p(rects, _I32), _p(keys, _F), _p(tx, _I32), _p(ty, _I32), R,
                         _p(req, _I32), _p(counts, _I64), _p(ids, _I32))
    return counts, ids[: int(counts.sum())]


def render(projs: Sequence[dict], cams, bg, pixels: np.ndarray,
           win_alpha: float = 0.0, win_T: float = 0.0,
           alpha_err: Optional[np.ndarray] = None) -> Dict[str, np.ndarray]:
    """Render the listed pixels ``[(view, x, y)]`` from projected Gaussians.

    ``win_alpha`` / ``win_T`` flag evaluations whose alpha (trial
    transmittance) lies within that relative distance of 1/255 (1e-4);
    ``alpha_err`` [V, n, 2], if given, bounds the relative alpha error of the
    implementation being compared by alpha_err[..., 0] + alpha_err[..., 1] q
    (q the pixel's quadratic form), which flags by that bound and by the
    transmittance error bound it implies (see orc_render); ``flag_dev`` /
    ``flag_T`` receive what the flagged decisions can change."""
    g2d, keys, rects = _stack_views(projs)
    V, n = keys.shape
    pix = np.ascontiguousarray(pixels, np.int32).reshape(-1, 3)
    P = pix.shape[0]
    color = np.zeros((P, 3)); T = np.zeros(P); nc = np.zeros(P, np.int32)
    flags = np.zeros(P, np.int32); nexp = np.zeros(P, np.int64); used = np.zeros(P, np.int32)
    sig = np.zeros(P, np.uint64)
    fdev = np.zeros(P); fT = np.zeros(P)
    bgd = _f64(bg)
    ae = None if alpha_err is None else np.ascontiguousarray(alpha_err,
                                                             np.float64).reshape(V, n, 2)
    lib().orc_render(V, n, _p(g2d, _D), _p(keys, _F), _p(rects, _I32), _p(_dims(cams), _I32),
                     P, _p(pix, _I32), _p(bgd, _D), float(win_alpha), float(win_T),
                     None if ae is None else _p(ae, _D),
                     _p(color, _D), _p(T, _D), _p(nc, _I32), _p(flags, _I32), _p(nexp, _I64),
                     _p(used, _I32), _p(sig, _U64), _p(fdev, _D), _p(fT, _D))
    return dict(color=color, T=T, n_contrib=nc, flags=flags, n_exp=nexp, n_used=used, sig=sig,
                flag_dev=fdev, flag_T=fT)


def render_bwd(projs: Sequence[dict], cams, bg, pixels: np.ndarray, dL_dC: np.ndarray) -> np.ndarray:
    """Screen-space gradients [V, n, 10] for the listed pixels and upstream dL/dC [P, 3]."""
    g2d, keys, rects = _stack_views(projs)
    V, n = keys.shape
    pix = np.ascontiguousarray(pixels, np.int32).reshape(-1, 3)
    P = pix.shape[0]
    gC = _f64(dL_dC).reshape(P, 3)
    out = np.zeros((V, n, 10), np.float64)
    lib().orc_render_bwd(V, n, _p(g2d, _D), _p(keys, _F), _p(rects, _I32), _p(_dims(cams), _I32),
                         P, _p(pix, _I32), _p(_f64(bg), _D), _p(gC, _D), _p(out, _D))
    return out


def project_bwd(scene, projs: Sequence[dict], grad2d: np.ndarray) -> Dict[str, np.ndarray]:
    """Gradients of the raw parameters from screen-space gradients [V, n, 10]."""
    m, s, q, lg, sh = _raw(scene)
    n = scene.n
    V = len(scene.cameras)
    K = (scene.sh_degree + 1) ** 2
    cams = np.ascontiguousarray(np.stack([pack_camera(c) for c in scene.cameras]))
    valid = np.ascontiguousarray(np.stack([p["valid"] for p in projs]).astype(np.int32))
    g = _f64(grad2d)
    gm = np.zeros((n, 3)); gs = np.zeros((n, 3)); gq = np.zeros((n, 4)); gl = np.zeros(n)
    gsh = np.zeros((n, K, 3))
    lib().orc_project_bwd(n, _p(m, _D), _p(s, _D), _p(q, _D), _p(lg, _D), _p(sh, _D),
                          int(scene.sh_degree), V, _p(cams, _D), _p(valid, _I32), _p(g, _D),
                          _p(gm, _D), _p(gs, _D), _p(gq, _D), _p(gl, _D), _p(gsh, _D))
    return dict(means=gm, log_scales=gs, quats=gq, opacity_logit=gl, sh=gsh)


def densify_stats(grad2d: np.ndarray, valid: np.ndarray, accum_plain=None, accum_abs=None,
                  denom=None):
    """View-space gradient statistics for densification, summed over views.

    Per view v and visible Gaussian i (the "plain" and "absolute" gradients of
    the absolute-gradient densification page, sec. 2 table):
      plain_i += || sum_p g_{i,p} ||_2   (the view's dL/dmean2D)
      abs_i   += sum_p || g_{i,p} ||_2
      denom_i += 1
    """
    g = np.asarray(grad2d, np.float64)
    vis = np.asarray(valid) != 0
    n = g.shape[1]
    plain = np.zeros(n) if accum_plain is None else np.array(accum_plain, np.float64)
    absg = np.zeros(n) if accum_abs is None else np.array(accum_abs, np.float64)
    den = np.zeros(n, np.int64) if denom is None else np.array(denom, np.int64)
    for v in range(g.shape[0]):
        plain += np.where(vis[v], np.hypot(g[v, :, 0], g[v, :, 1]), 0.0)
        absg += np.where(vis[v], g[v, :, 9], 0.0)
        den += vis[v].astype(np.int64)
    return plain, absg, den


def adam(param, grad, m, v, lr: float, step: int, beta1=0.9, beta2=0.999, eps=1e-15):
    """One Adam step (Kingma and Ba, with bias correction), float64.

    m <- b1 m + (1-b1) g;  v <- b2 v + (1-b2) g^2;
    p <- p - lr * (m / (1-b1^t)) / (sqrt(v / (1-b2^t)) + eps).
    """
    p = np.array(param, np.float64)
    g = np.asarray(grad, np.float64)
    m = beta1 * np.asarray(m, np.float64) + (1.0 - beta1) * g
    v = beta2 * np.asarray(v, np.float64) + (1.0 - beta2) * g * g
    mhat = m / (1.0 - beta1 ** step)
    vhat = v / (1.0 - beta2 ** step)
    p = p - lr * mhat / (np.sqrt(vhat) + eps)
    return p, m, v


def render_all(scene, projs=None, bg=None, tol_alpha=0.0, tol_T=0.0):
    """Full-image forward render of every view; returns [V,3,H,W] colour etc."""
    projs = project_views(scene) if projs is None else projs
    outs = []
    for v, c in enumerate(scene.cameras):
        ys, xs = np.meshgrid(np.arange(c.height), np.arange(c.width), indexing="ij")
        pix = np.stack([np.full(xs.size, v), xs.ravel(), ys.ravel()], axis=1)
        outs.append((pix, render(projs, scene.cameras, scene.background if bg is None else bg,
                                 pix, tol_alpha, tol_T)))
    return outs


# --------------------------------------------------------------- densify_and_prune

DP_PRUNE, DP_KEEP, DP_CLONE, DP_SPLIT = 0, 1, 2, 3
PARAM_NAMES = ("means", "log_scales", "quats", "opacity_logit", "sh")


def _rotate(q, u):
    """u rotated by the unit quaternion q = (w, x, y, z): the sandwich product
    q (0, u) q*, written as u + 2w (v x u) + 2 v x (v x u) with v = (x, y, z)."""
    w = q[..., :1]
    v = q[..., 1:]
    t = 2.0 * np.cross(v, u)
    return u + w * t + np.cross(v, t)


def densify_decisions(log_scales, opacity_logit, accum, denom, grad_threshold, log_scale_split,
                      logit_min_opacity, log_max_scale):
    """Per-Gaussian decision of densify_and_prune (absolute-gradient
    densification page, sec. 1 and 3.3: the average gradient accum / denom
    against a threshold; clone a small Gaussian, split a large one, prune a
    faint or oversized one). Taken in float32 like the kernel: the gradient
    test as accum > threshold * denom (denom > 0), the scale and opacity tests
    on the raw log-scale and logit against float32 thresholds. Pruning wins.
    Returns the codes DP_PRUNE / DP_KEEP / DP_CLONE / DP_SPLIT."""
    f = np.float32
    ls = np.asarray(log_scales, f)
    lg = np.asarray(opacity_logit, f).reshape(-1)
    acc = np.asarray(accum, f).reshape(-1)
    den = np.asarray(denom).reshape(-1)
    max_ls = ls.max(axis=1)
    hot = (den > 0) & (acc > f(grad_threshold) * den.astype(f))
    large = max_ls > f(log_scale_split)
    prune = (lg < f(logit_min_opacity)) | (max_ls > f(log_max_scale))
    code = np.full(len(lg), DP_KEEP, np.int32)
    code[hot & ~large] = DP_CLONE
    code[hot & large] = DP_SPLIT
    code[prune] = DP_PRUNE
    return code


def densify_and_prune(params: dict, moments: dict, accum, denom, z, grad_threshold,
                      log_scale_split, logit_min_opacity, log_max_scale,
                      split_shrink: float = 1.6):
    """densify_and_prune in float64, Gaussian by Gaussian in index order:
      prune -> nothing;  keep -> the Gaussian (its Adam moments kept);
      clone -> the Gaussian, then an exact copy (moments zero);
      split -> two children c = 0, 1 (moments zero): mean + R (s * z[i, c]),
               log-scale - ln(split_shrink), everything else copied;
    R the rotation of the normalised quaternion, s = exp(log-scale), z the
    caller's standard normal draws [N][2][3].
    params: name -> array [N, ...]; moments: name -> (m, v) of the same shapes.
    Returns (params_out, moments_out, codes)."""
    code = densify_decisions(params["log_scales"], params["opacity_logit"], accum, denom,
                             grad_threshold, log_scale_split, logit_min_opacity, log_max_scale)
    P = {k: np.asarray(params[k], np.float64) for k in PARAM_NAMES}
    Mo = {k: (np.asarray(moments[k][0], np.float64), np.asarray(moments[k][1], np.float64))
          for k in PARAM_NAMES}
    n = len(code)
    z = np.asarray(z, np.float64).reshape(n, 2, 3)
    q = P["quats"] / np.linalg.norm(P["quats"], axis=1, keepdims=True)
    s = np.exp(P["log_scales"])
    out = {k: [] for k in PARAM_NAMES}
    mom = {k: ([], []) for k in PARAM_NAMES}
    for i in range(n):
        c = code[i]
        if c == DP_PRUNE:
            continue
        if c in (DP_KEEP, DP_CLONE):
            for k in PARAM_NAMES:
                out[k].append(P[k][i])
                mom[k][0].append(Mo[k][0][i])
                mom[k][1].append(Mo[k][1][i])
        if c == DP_CLONE:
            for k in PARAM_NAMES:
                out[k].append(P[k][i])
                mom[k][0].append(np.zeros_like(P[k][i]))
                mom[k][1].append(np.zeros_like(P[k][i]))
        if c == DP_SPLIT:
            for ch in range(2):
                child = {k: P[k][i].copy() for k in PARAM_NAMES}
                child["means"] = P["means"][i] + _rotate(q[i], s[i] * z[i, ch])
                child["log_scales"] = P["log_scales"][i] - np.log(split_shrink)
                for k in PARAM_NAMES:
                    out[k].append(child[k])
                    mom[k][0].append(np.zeros_like(P[k][i]))
                    mom[k][1].append(np.zeros_like(P[k][i]))
    shapes = {k: P[k].shape[1:] for k in PARAM_NAMES}
    params_out = {k: (np.array(out[k]).reshape((-1,) + shapes[k])) for k in PARAM_NAMES}
    moments_out = {k: (np.array(mom[k][0]).reshape((-1,) + shapes[k]),
                       np.array(mom[k][1]).reshape((-1,) + shapes[k])) for k in PARAM_NAMES}
    return params_out, moments_out, code


# --------------------------------------------------------------- photometric loss

# The training objective of the second Julia page (lshu.cn, sec. 3.3): a blend
# of the L1 error and the structural dissimilarity 1 - SSIM with weight
# lambda about 0.2. The page fixes nothing else about SSIM, so the constants
# are those of the SSIM definition itself (Wang, Bovik, Sheikh, Simoncelli
# 2004): an 11 x 11 Gaussian window of standard deviation 1.5 normalised to
# sum 1, C1 = (0.01 L)^2 and C2 = (0.03 L)^2 with dynamic range L = 1. The map
# is taken at every pixel with the image zero-padded outside its border, and
# both terms are means over the pixels and colour channels of one view.
SSIM_WINDOW = 11
SSIM_SIGMA = 1.5
SSIM_C1 = 0.01 ** 2
SSIM_C2 = 0.03 ** 2
LOSS_LAMBDA = 0.2


def ssim_window(size: int = SSIM_WINDOW, sigma: float = SSIM_SIGMA) -> np.ndarray:
    """The 2-D Gaussian window w[i, j] ~ exp(-(di^2 + dj^2) / (2 sigma^2)),
    di, dj the offsets from the centre, normalised to sum 1."""
    r = np.arange(size, dtype=np.float64) - (size - 1) / 2.0
    w = np.exp(-(r[:, None] ** 2 + r[None, :] ** 2) / (2.0 * sigma * sigma))
    return w / w.sum()


def window_filter(img: np.ndarray, w: np.ndarray) -> np.ndarray:
    """Same-size correlation of the last two axes with the window w, zero
    outside the image: out[y, x] = sum_ij w[i, j] img[y + i - h, x + j - h]."""
    img = np.asarray(img, np.float64)
    s = w.shape[0]
    h = s // 2
    H, W = img.shape[-2:]
    pad = np.zeros(img.shape[:-2] + (H + 2 * h, W + 2 * h))
    pad[..., h:h + H, h:h + W] = img
    out = np.zeros(img.shape)
    for i in range(s):
        for j in range(s):
            out += w[i, j] * pad[..., i:i + H, j:j + W]
    return out


def ssim_map(x: np.ndarray, y: np.ndarray, w: Optional[np.ndarray] = None) -> np.ndarray:
    """SSIM at every pixel of the planes x, y (last two axes): local means,
    variances and covariance under the window, then
    S = (2 mx my + C1)(2 sxy + C2) / ((mx^2 + my^2 + C1)(sx^2 + sy^2 + C2))."""
    w = ssim_window() if w is None else w
    x = np.asarray(x, np.float64)
    y = np.asarray(y, np.float64)
    mx, my = window_filter(x, w), window_filter(y, w)
    sxx = window_filter(x * x, w) - mx * mx
    syy = window_filter(y * y, w) - my * my
    sxy = window_filter(x * y, w) - mx * my
    return ((2 * mx * my + SSIM_C1) * (2 * sxy + SSIM_C2)
            / ((mx * mx + my * my + SSIM_C1) * (sxx + syy + SSIM_C2)))


def l1_dssim_loss(image: np.ndarray, target: np.ndarray, lam: float = LOSS_LAMBDA):
    """Loss and its gradient for images [V, 3, H, W] against targets of the
    same shape, view by view:
      L_v = (1 - lam) mean|x - y| + lam (1 - mean SSIM(x, y)).
    The gradient dL_v / dx is the chain rule through the window statistics:
    with the SSIM map written as S(mx, Exx, Exy) of the windowed moments
    mx = w*x, Exx = w*(x x), Exy = w*(x y), each pixel q receives
      dS_mean/dx_q = (1/N) [w'*(dS/dmx) + 2 x_q w'*(dS/dExx) + y_q w'*(dS/dExy)]_q
    where w'* is the adjoint of the zero-padded correlation (correlation with
    the flipped window, zero outside). The L1 term contributes
    sign(x_q - y_q) / N with sign(0) = 0. Returns (terms [V, 3] = loss, mean
    L1, mean SSIM per view; grad [V, 3, H, W])."""
    x = np.asarray(image, np.float64)
    y = np.asarray(target, np.float64)
    w = ssim_window()
    wf = w[::-1, ::-1]
    V = x.shape[0]
    N = float(np.prod(x.shape[1:]))
    mx, my = window_filter(x, w), window_filter(y, w)
    exx, eyy, exy = window_filter(x * x, w), window_filter(y * y, w), window_filter(x * y, w)
    a1 = 2 * mx * my + SSIM_C1
    a2 = 2 * (exy - mx * my) + SSIM_C2
    b1 = mx * mx + my * my + SSIM_C1
    b2 = (exx - mx * mx) + (eyy - my * my) + SSIM_C2
    num, den = a1 * a2, b1 * b2
    S = num / den
    # partial derivatives of S = num / den with respect to mx, Exx and Exy
    d_num_mx = 2 * my * a2 + a1 * (-2 * my)
    d_den_mx = 2 * mx * b2 + b1 * (-2 * mx)
    d_mx = (d_num_mx * den - num * d_den_mx) / (den * den)
    d_exx = -num * b1 / (den * den)
    d_exy = 2 * a1 / den
    g_ssim = (window_filter(d_mx, wf) + 2 * x * window_filter(d_exx, wf)
              + y * window_filter(d_exy, wf)) / N
    diff = x - y
    l1 = np.abs(diff).reshape(V, -1).mean(axis=1)
    ssim = S.reshape(V, -1).mean(axis=1)
    terms = np.stack([(1 - lam) * l1 + lam * (1 - ssim), l1, ssim], axis=1)
    grad = (1 - lam) * np.sign(diff) / N - lam * g_ssim
    return terms, grad


# --------------------------------------------------------------- quantised SH state

# The Spirula VRAM page (sec. 魔法一, quantised training): SH coefficients are
# stored as 8- or 16-bit fixed point, every 256 units sharing one (min, max)
# pair that decodes them; gradients stay float32; the Adam moments are 16-bit
# words in a transposed layout. Readings where the page is silent: a unit is
# one SH value; the layout is coefficient-major ([3K][N], N padded to a
# multiple of 256), so a group is one coefficient of 256 consecutive
# Gaussians; a code q decodes to min + q (max - min) / (2^b - 1); encoding
# takes the group's min and max and rounds (x - min) (2^b - 1) / (max - min),
# in float32 like the kernel, to nearest-even or stochastically (floor of
# t + u, u uniform from SplitMix64); the 16-bit Adam words are bfloat16,
# rounded to nearest-even from float32.
Q_GROUP = 256
_GAMMA = np.uint64(0x9E3779B97F4A7C15)


def splitmix64(seed: int, counter) -> np.ndarray:
    """Output number `counter` + 1 of SplitMix64 started at `seed` (Steele,
    Lea and Flood 2014): z = seed + (counter + 1) gamma, then the variant-13
    mix z ^= z >> 30; z *= 0xBF58476D1CE4E5B9; z ^= z >> 27;
    z *= 0x94D049BB133111EB; z ^= z >> 31 (all mod 2^64)."""
    with np.errstate(over="ignore"):
        c = np.asarray(counter, np.uint64)
        z = np.uint64(seed) + (c + np.uint64(1)) * _GAMMA
        z = (z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
        return z ^ (z >> np.uint64(31))


def sr_uniform(seed: int, step: int, coef, gauss) -> np.ndarray:
    """The stochastic-rounding draw of SH value (coefficient j, Gaussian n) at
    Adam step t: counter = t 2^37 + j 2^31 + n, u = (top 24 bits) / 2^24, a
    float32 in [0, 1)."""
    c = ((np.uint64(step) << np.uint64(37)) + (np.asarray(coef, np.uint64) << np.uint64(31))
         + np.asarray(gauss, np.uint64))
    return ((splitmix64(seed, c) >> np.uint64(40)).astype(np.float64) / 2.0 ** 24).astype(
        np.float32)


def to_bf16(x) -> np.ndarray:
    """bfloat16 bits (uint16) of float32(x), rounded to nearest-even."""
    b = np.asarray(np.asarray(x, np.float32)).view(np.uint32).astype(np.uint64)
    r = (b + np.uint64(0x7FFF) + ((b >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return r.astype(np.uint16)


def from_bf16(h) -> np.ndarray:
    return (np.asarray(h, np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32).astype(
        np.float64)


def _sh_transposed(sh: np.ndarray, n_pad: int) -> np.ndarray:
    """[N][K][3] -> [3K][n_pad] (value j = 3 k + channel), zero padding."""
    n = sh.shape[0]
    t = np.zeros((sh.shape[1] * 3, n_pad), np.asarray(sh).dtype)
    t[:, :n] = np.asarray(sh).reshape(n, -1).T
    return t


def quantize_groups(x: np.ndarray, n: int, bits: int, rounding: int = 0, seed: int = 0,
                    step: int = 0):
    """Codes and (min, max) bounds of float32 values x [3K][n_pad], groups of
    256 along the Gaussian axis over the first n Gaussians only. The decision
    is taken in float32: range = max - min, inv = (2^b - 1) / range,
    t = (x - min) inv, then rint(t) (rounding 0) or floor(t + u) (rounding 1),
    clamped to [0, 2^b - 1]; a group with max == min gets code 0."""
    f = np.float32
    x = np.asarray(x, f)
    k3, n_pad = x.shape
    qmax = (1 << bits) - 1
    codes = np.zeros((k3, n_pad), np.uint16 if bits == 16 else np.uint8)
    bounds = np.zeros((k3, n_pad // Q_GROUP, 2), f)
    for g in range(n_pad // Q_GROUP):
        a, b = g * Q_GROUP, min((g + 1) * Q_GROUP, n)
        if b <= a:
            continue
        blk = x[:, a:b]
        lo, hi = blk.min(axis=1), blk.max(axis=1)
        bounds[:, g, 0], bounds[:, g, 1] = lo, hi
        rng = (hi - lo).astype(f)
        flat = rng == 0
        inv = np.where(flat, f(0), f(qmax) / np.where(flat, f(1), rng)).astype(f)
        t = ((blk - lo[:, None]).astype(f) * inv[:, None]).astype(f)
        if rounding == 0:
            q = np.rint(t)
        else:
            u = sr_uniform(seed, step, np.arange(k3)[:, None], np.arange(a, b)[None, :])
            q = np.floor((t + u).astype(f))
        codes[:, a:b] = np.clip(q, 0, qmax).astype(codes.dtype)
    return codes, bounds


def dequantize_groups(codes: np.ndarray, bounds: np.ndarray, n: int, bits: int) -> np.ndarray:
    """x = min + q (max - min) / (2^b - 1) in float64 -> [3K][n]."""
    qmax = (1 << bits) - 1
    c = np.asarray(codes, np.float64)[:, :n]
    g = np.arange(n) // Q_GROUP
    lo = np.asarray(bounds, np.float64)[:, g, 0]
    hi = np.asarray(bounds, np.float64)[:, g, 1]
    return lo + c * (hi - lo) / qmax


def fma_f32(a, b, c) -> np.ndarray:
    """float32 fused multiply-add, correctly rounded (round to nearest-even),
    elementwise on float32 arrays: a*b is exact in float64 (24 + 24
    significant bits), p + c is taken with its exact error (Knuth's TwoSum),
    and the float64 sum is rounded to float32, except where it sits exactly
    halfway between two float32 values: there the error's sign decides."""
    f64 = np.float64
    a, b, c = (np.asarray(x, np.float32).astype(f64) for x in (a, b, c))
    p = a * b
    s = p + c
    bv = s - p
    e = (p - (s - bv)) + (c - bv)
    r = s.astype(np.float32)
    rd = r.astype(f64)
    up = np.nextafter(r, np.float32(np.inf))
    dn = np.nextafter(r, np.float32(-np.inf))
    tie_up = (s - rd) * 2 == up.astype(f64) - rd
    tie_dn = (rd - s) * 2 == rd - dn.astype(f64)
    r = np.where(tie_up & (e > 0), up, r)
    r = np.where(tie_dn & (e < 0), dn, r)
    return np.asarray(r, np.float32)


def dequantize_groups_f32(codes: np.ndarray, bounds: np.ndarray, n: int, bits: int) -> np.ndarray:
    """The float32 decoding of the codes, as the state's definition fixes
    it: step = (max - min) / (2^b - 1) with each operation rounded to
    float32, then x = fma(q, step, min) rounded once -> float32 [3K][n]."""
    f = np.float32
    g = np.arange(n) // Q_GROUP
    lo = np.asarray(bounds, f)[:, g, 0]
    hi = np.asarray(bounds, f)[:, g, 1]
    step = ((hi - lo).astype(f) / f((1 << bits) - 1)).astype(f)
    return fma_f32(np.asarray(codes)[:, :n].astype(f), step, lo)


def sh_quantize(sh: np.ndarray, bits: int):
    """Quantised SH state of float32 SH [N][K][3]: (codes [3K][n_pad], bounds
    [3K][n_pad / 256][2]) with round-to-nearest."""
    n = sh.shape[0]
    n_pad = -(-n // Q_GROUP) * Q_GROUP
    return quantize_groups(_sh_transposed(np.asarray(sh, np.float32), n_pad), n, bits)


def adam_sh_quant(codes, bounds, grad_sh, m16, v16, n: int, bits: int, lr: float, step: int,
                  beta1=0.9, beta2=0.999, eps=1e-15, rounding: int = 0, seed: int = 0):
    """One Adam step on quantised SH: decode the parameters, update the
    bfloat16 moments with the float32 gradient (grad_sh [N][K][3]), take the
    Adam step (as ``adam``), store the moments back as bfloat16 and re-encode
    the parameters with their groups' new min and max (the float32 value of
    the new parameter is quantised, like the kernel's). Returns (codes,
    bounds, m16, v16, p_new [3K][n] float64)."""
    n_pad = codes.shape[1]
    p = dequantize_groups(codes, bounds, n, bits)
    g = _sh_transposed(np.asarray(grad_sh, np.float64), n_pad)[:, :n]
    m = from_bf16(m16[:, :n])
    v = from_bf16(v16[:, :n])
    p, m, v = adam(p, g, m, v, lr, step, beta1, beta2, eps)
    m_out = np.array(m16, copy=True)
    v_out = np.array(v16, copy=True)
    m_out[:, :n] = to_bf16(m)
    v_out[:, :n] = to_bf16(v)
    x = np.zeros((codes.shape[0], n_pad), np.float32)
    x[:, :n] = p.astype(np.float32)
    c, b = quantize_groups(x, n, bits, rounding, seed, step)
    return c, b, m_out, v_out, p
