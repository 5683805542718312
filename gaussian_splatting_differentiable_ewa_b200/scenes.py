"""Seeded synthetic scenes and cameras for the differentiable EWA splatting path.

This module only draws random numbers and builds pinhole cameras. It holds none
of the splatting arithmetic (projection, binning, compositing, gradients,
Adam), so that the CUDA path and the float64 oracle can both be fed from it
without sharing any of the method's code.

Workloads (sizes and distributions as the task's workload table gives them;
every array is drawn in float64 from ``numpy.random.default_rng(seed)`` and
cast to float32, in the order means, log-scales, quaternions, opacity logits,
SH coefficients):

* ``fwd_1k_128``      1,000 Gaussians, SH degree 0, one 128x128 view, f=128.
* ``fwd_100k_800``    100,000 Gaussians, SH degree 3, one 800x800 view, f=900.
* ``train_1m_1080p``  1,000,000 Gaussians, SH3, one 1920x1080 view, f=1200.
* ``train_6m_8x1080p`` 6,000,000 Gaussians, SH3, 8 views of 1920x1080 on an
  orbit of radius 8, log-scales U(-6,-3) with 5 % outliers U(-2,-1).
* ``train_10m_4k``    10,000,000 Gaussians, SH3, one 3840x2160 view, f=2400.

Any workload can be drawn at a smaller Gaussian count (``n=``) or image size
(``width=``/``height=``, focal length scaled with the width) with the same
distributions; parity tests use that to keep the oracle fast.

Readings of the workload text:

* ``N(m, s)`` is read as mean m and variance s (the text writes the cluster as
  ``N(0, 0.5^2 I)``), so the higher-order SH draws have std sqrt(0.05) and the
  upstream image gradient has std 0.1.
* The "50/50 mixture of a box and clusters" draws one Bernoulli(1/2) per
  Gaussian; the cluster is N(0, 0.5^2 I) centred at the origin.
* The degree-0 workload gives colours as RGB U(0,1). It is stored as the DC
  coefficient k = (rgb - 0.5) * 2 sqrt(pi), the inverse of the degree-0 colour
  map rgb = k / (2 sqrt(pi)) + 0.5, so that the rendered colour is that RGB.
* Cameras follow the OpenCV convention (x right, y down, z forward); the
  look-at uses world up = -y. Views at "distance 8 on a sphere" sit at
  (0, 0, -8); the 8-view orbit puts view k at 8 (sin 2pi k/8, 0, -cos 2pi k/8).
"""

from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional

import numpy as np

__all__ = [
    "Camera",
    "Scene",
    "WORKLOADS",
    "look_at",
    "make_scene",
    "make_upstream_grad",
    "make_projected_2d",
    "make_isolated_scene",
]


@dataclasses.dataclass
class Camera:
    """Pinhole camera; ``viewmat`` is the row-major 3x4 world-to-camera [R|t]."""

    viewmat: np.ndarray  # (3, 4) float32
    fx: float
    fy: float
    cx: float
    cy: float
    width: int
    height: int
    campos: np.ndarray  # (3,) float32, camera centre in world coordinates

    def as_dict(self) -> dict:
        return dict(viewmat=self.viewmat, fx=self.fx, fy=self.fy, cx=self.cx,
                    cy=self.cy, width=self.width, height=self.height,
                    campos=self.campos)


@dataclasses.dataclass
class Scene:
    """Raw (un-activated) Gaussian parameters plus cameras.

    Layout: ``means``, ``log_scales`` and ``quats`` are float32 [N, 4]; the
    fourth lane of means / log-scales is zero padding; quats are (w, x, y, z).
    ``opacity_logit`` is float32 [N]; ``sh`` is float32 [N, (deg+1)^2, 3].
    """

    name: str
    means: np.ndarray
    log_scales: np.ndarray
    quats: np.ndarray
    opacity_logit: np.ndarray
    sh: np.ndarray
    sh_degree: int
    cameras: List[Camera]
    background: np.ndarray  # (3,) float32

    @property
    def n(self) -> int:
        return int(self.means.shape[0])

    @property
    def n_views(self) -> int:
        return len(self.cameras)


def look_at(centre, target=(0.0, 0.0, 0.0), up=(0.0, -1.0, 0.0)) -> np.ndarray:
    """World-to-camera [R|t] (float64, 3x4) for a camera at ``centre``.

    Rows of R are the camera axes in world coordinates: z looks from the
    centre to the target, x = normalize(z cross up), y = z cross x.
    """
    c = np.asarray(centre, np.float64)
    z = np.asarray(target, np.float64) - c
    z /= np.linalg.norm(z)
    x = np.cross(z, np.asarray(up, np.float64))
    x /= np.linalg.norm(x)
    y = np.cross(z, x)
    r = np.stack([x, y, z])
    t = -r @ c
    return np.concatenate([r, t[:, None]], axis=1)


def _camera(viewmat64: np.ndarray, centre, f: float, width: int, height: int) -> Camera:
    return Camera(viewmat=viewmat64.astype(np.float32), fx=float(f), fy=float(f),
                  cx=width / 2.0, cy=height / 2.0, width=int(width),
                  height=int(height),
                  campos=np.asarray(centre, np.float64).astype(np.float32))


# name -> workload description
WORKLOADS: Dict[str, dict] = {
    "fwd_1k_128": dict(n=1000, sh_degree=0, width=128, height=128, f=128.0,
                       views="origin", means="box_near", log_scale=(-4.0, -2.0),
                       opacity="uniform", colour="rgb", backward=False),
    "fwd_100k_800": dict(n=100_000, sh_degree=3, width=800, height=800, f=900.0,
                         views="front", means="mixture", log_scale=(-5.0, -2.0),
                         opacity="normal", colour="sh", backward=False),
    "train_1m_1080p": dict(n=1_000_000, sh_degree=3, width=1920, height=1080, f=1200.0,
                           views="front", means="mixture", log_scale=(-5.0, -2.0),
                           opacity="normal", colour="sh", backward=True),
    "train_6m_8x1080p": dict(n=6_000_000, sh_degree=3, width=1920, height=1080, f=1200.0,
                             views="orbit8", means="mixture", log_scale=(-6.0, -3.0),
                             outliers=(0.05, -2.0, -1.0), opacity="normal",
                             colour="sh", backward=True),
    "train_10m_4k": dict(n=10_000_000, sh_degree=3, width=3840, height=2160, f=2400.0,
                         views="front", means="mixture", log_scale=(-5.0, -2.0),
                         opacity="normal", colour="sh", backward=True),
}


def _cameras(kind: str, f: float, width: int, height: int) -> List[Camera]:
    if kind == "origin":
        vm = np.concatenate([np.eye(3), np.zeros((3, 1))], axis=1)
        return [_camera(vm, (0.0, 0.0, 0.0), f, width, height)]
    if kind == "front":
        c = (0.0, 0.0, -8.0)
        return [_camera(look_at(c), c, f, width, height)]
    if kind == "orbit8":
        cams = []
        for k in range(8):
            a = 2.0 * math.pi * k / 8.0
            c = (8.0 * math.sin(a), 0.0, -8.0 * math.cos(a))
            cams.append(_camera(look_at(c), c, f, width, height))
        return cams
    raise ValueError(kind)


def make_scene(name: str, seed: int = 0, n: Optional[int] = None,
               width: Optional[int] = None, height: Optional[int] = None,
               n_views: Optional[int] = None) -> Scene:
    """Draw a seeded synthetic scene for workload ``name``.

    ``n`` overrides the Gaussian count; ``width``/``height`` override the image
    size, with the focal length scaled by width / nominal width so the field of
    view is kept; ``n_views`` keeps only the first views of a multi-view rig.
    """
    w = WORKLOADS[name]
    n = int(w["n"] if n is None else n)
    width = int(w["width"] if width is None else width)
    height = int(w["height"] if height is None else height)
    f = float(w["f"]) * width / float(w["width"])
    rng = np.random.default_rng(seed)

    # 1. means
    if w["means"] == "box_near":
        xy = rng.uniform(-1.0, 1.0, size=(n, 2))
        z = rng.uniform(2.0, 6.0, size=(n, 1))
        m3 = np.concatenate([xy, z], axis=1)
    else:
        pick_box = rng.random(n) < 0.5
        box = rng.uniform(-3.0, 3.0, size=(n, 3))
        cluster = rng.normal(0.0, 0.5, size=(n, 3))
        m3 = np.where(pick_box[:, None], box, cluster)

    # 2. log-scales (per axis), with optional large outliers
    lo, hi = w["log_scale"]
    s3 = rng.uniform(lo, hi, size=(n, 3))
    if "outliers" in w:
        frac, olo, ohi = w["outliers"]
        is_out = rng.random(n) < frac
        big = rng.uniform(olo, ohi, size=(n, 3))
        s3 = np.where(is_out[:, None], big, s3)

    # 3. rotations: normalised 4-D standard normal draws (uniform on S^3)
    q = rng.normal(0.0, 1.0, size=(n, 4))
    q /= np.linalg.norm(q, axis=1, keepdims=True)

    # 4. opacity logits
    if w["opacity"] == "uniform":
        logit = rng.uniform(-2.0, 2.0, size=n)
    else:
        logit = rng.normal(0.0, 1.0, size=n)

    # 5. colour / SH coefficients, [N, K, 3]
    deg = int(w["sh_degree"])
    k = (deg + 1) ** 2
    sh = np.zeros((n, k, 3), np.float64)
    if w["colour"] == "rgb":
        rgb = rng.uniform(0.0, 1.0, size=(n, 3))
        sh[:, 0, :] = (rgb - 0.5) * (2.0 * math.sqrt(math.pi))
    else:
        sh[:, 0, :] = rng.uniform(0.0, 1.0, size=(n, 3))
        if k > 1:
            sh[:, 1:, :] = rng.normal(0.0, math.sqrt(0.05), size=(n, k - 1, 3))

    means = np.zeros((n, 4), np.float32)
    means[:, :3] = m3
    log_scales = np.zeros((n, 4), np.float32)
    log_scales[:, :3] = s3
    cams = _cameras(w["views"], f, width, height)
    if n_views is not None:
        cams = cams[:n_views]
    return Scene(name=name, means=means, log_scales=log_scales,
                 quats=q.astype(np.float32), opacity_logit=logit.astype(np.float32),
                 sh=sh.astype(np.float32), sh_degree=deg, cameras=cams,
                 background=np.zeros(3, np.float32))


def make_upstream_grad(n_views: int, height: int, width: int, seed: int = 1,
                       std: float = 0.1) -> np.ndarray:
    """dL/d(image), float32 [V, 3, H, W], drawn N(0, std^2) (std 0.1 = var 1e-2)."""
    rng = np.random.default_rng(seed)
    g = rng.normal(0.0, std, size=(n_views, 3, height, width))
    return g.astype(np.float32)


def make_projected_2d(n: int, width: int, height: int, seed: int = 2,
                      radius_range=(1, 40), n_views: int = 1) -> dict:
    """Random screen-space Gaussians for testing the binning and sort alone.

    Returns float32 centres ``xy`` [V, n, 2] spread a little beyond the image,
    integer radii [V, n] (0 marks a culled Gaussian, about 5 %), and float32
    depths [V, n] drawn from a small set of values so that equal sort keys
    (ties broken by index) are common.
    """
    rng = np.random.default_rng(seed)
    xy = np.stack([rng.uniform(-0.1 * width, 1.1 * width, size=(n_views, n)),
                   rng.uniform(-0.1 * height, 1.1 * height, size=(n_views, n))], axis=-1)
    radius = rng.integers(radius_range[0], radius_range[1] + 1, size=(n_views, n))
    radius = np.where(rng.random((n_views, n)) < 0.05, 0, radius)
    depth = rng.choice(np.linspace(0.5, 30.0, 257), size=(n_views, n))
    depth = depth + rng.integers(0, 4, size=(n_views, n)) * 1e-3
    return dict(xy=xy.astype(np.float32), radius=radius.astype(np.int32),
                depth=depth.astype(np.float32))


def make_image_pair(n_views: int, height: int, width: int, seed: int = 3,
                    noise: float = 0.05, tie_frac: float = 0.05):
    """A rendered-like image and a target for the photometric loss, float32
    [V, 3, H, W] each, values in [0, 1].

    The target is a smooth field (a few random low-frequency sinusoids per
    channel) with sharp-edged discs on top, like a render of a few large
    splats over a background; the image is the target shifted by a slowly
    varying offset plus white noise of standard deviation `noise`, clipped to
    [0, 1]. A fraction `tie_frac` of the image's values equals the target's
    exactly, so that |x - y| has zeros.
    """
    rng = np.random.default_rng(seed)
    yy, xx = np.meshgrid(np.linspace(0, 1, height), np.linspace(0, 1, width), indexing="ij")
    tgt = np.empty((n_views, 3, height, width))
    img = np.empty_like(tgt)
    for v in range(n_views):
        for c in range(3):
            f = 0.5 + np.zeros((height, width))
            for _ in range(4):
                kx, ky = rng.uniform(0.5, 6.0, 2)
                f += 0.12 * np.sin(2 * np.pi * (kx * xx + ky * yy) + rng.uniform(0, 2 * np.pi))
            for _ in range(6):
                cx, cy, r = rng.uniform(0, 1), rng.uniform(0, 1), rng.uniform(0.03, 0.2)
                f = np.where((xx - cx) ** 2 + (yy - cy) ** 2 < r * r, rng.uniform(0, 1), f)
            tgt[v, c] = f
            off = 0.05 * np.sin(2 * np.pi * (rng.uniform(0.2, 2) * xx + rng.uniform(0, 1)))
            img[v, c] = f + off + rng.normal(0.0, noise, size=(height, width))
    tgt = np.clip(tgt, 0.0, 1.0).astype(np.float32)
    img = np.clip(img, 0.0, 1.0).astype(np.float32)
    tie = rng.random(img.shape) < tie_frac
    img[tie] = tgt[tie]
    return img, tgt


def make_isolated_scene(side: int = 16, spacing: int = 128, seed: int = 9,
                        f: float = 600.0, depth: float = 8.0) -> Scene:
    """side x side Gaussians, one per spacing x spacing pixel cell of a single
    view (camera at the origin looking down +z), far enough apart that no tile
    holds two of them, so every pixel sees at most one splat. Log-scales
    U(-5, -2.3) per axis (2D anisotropy up to ~15), uniform rotations, opacity
    logits U(-5, 7) (so both the alpha clamp at 0.99 and splats too faint to
    count occur), a random sub-pixel offset of each mean, and an image of
    side * spacing pixels squared (means far from the origin, where a float
    keeps only ~1e-4 px of the mean). Degree-0 colour, DC U(0, 1)."""
    rng = np.random.default_rng(seed)
    n = side * side
    width = height = side * spacing
    cx = cy = width / 2.0
    gx, gy = np.meshgrid(np.arange(side), np.arange(side), indexing="xy")
    px = (gx.ravel() + 0.5) * spacing + rng.uniform(-0.5, 0.5, n)
    py = (gy.ravel() + 0.5) * spacing + rng.uniform(-0.5, 0.5, n)
    m3 = np.stack([(px - cx) / f * depth, (py - cy) / f * depth, np.full(n, depth)], 1)
    s3 = rng.uniform(-5.0, -2.3, size=(n, 3))
    q = rng.normal(0.0, 1.0, size=(n, 4))
    q /= np.linalg.norm(q, axis=1, keepdims=True)
    logit = rng.uniform(-5.0, 7.0, size=n)
    sh = np.zeros((n, 1, 3))
    sh[:, 0, :] = rng.uniform(0.0, 1.0, size=(n, 3))
    means = np.zeros((n, 4), np.float32)
    means[:, :3] = m3
    log_scales = np.zeros((n, 4), np.float32)
    log_scales[:, :3] = s3
    vm = np.concatenate([np.eye(3), np.zeros((3, 1))], axis=1)
    return Scene(name="isolated", means=means, log_scales=log_scales,
                 quats=q.astype(np.float32), opacity_logit=logit.astype(np.float32),
                 sh=sh.astype(np.float32), sh_degree=0,
                 cameras=[_camera(vm, (0.0, 0.0, 0.0), f, width, height)],
                 background=np.zeros(3, np.float32))
