"""Shared helpers for the GPU parity tests: run the CUDA path and the oracle on
the same seeded scene and compare them under the stated tolerances.

Tolerances (the task's acceptance criteria):
  * binning: per-tile sorted id lists bit-exact;
  * rendered colours: max |d| <= 2e-3 and mean |d| <= 1e-5, over pixels whose
    float64 decisions are not within the flag windows of a threshold
    (alpha vs 1/255, trial transmittance vs 1e-4); flagged pixels are counted;
  * gradients, densify statistics and Adam state: relative L2 <= 1e-3.
"""

from __future__ import annotations

import numpy as np

from oracle import oracle as O

# Flag windows: relative distance of alpha from 1/255 and of the trial
# transmittance from 1e-4 below which float32 and float64 may decide apart.
# With cancellation in the quadratic form of an elongated Gaussian the
# kernel's alpha can sit 2e-5 relative from the float64 value (a flip seen at
# a distance between 2e-5 and 2e-4); every near-opaque layer multiplies that
# by alpha / (1 - alpha) in the trial T.
WIN_ALPHA = 2e-4
WIN_T = 2e-3

MAX_ABS = 2e-3
MEAN_ABS = 1e-5
REL_L2 = 1e-3


def rel_l2(a, b) -> float:
    a = np.asarray(a, np.float64).ravel()
    b = np.asarray(b, np.float64).ravel()
    den = np.linalg.norm(b)
    if den == 0:
        return float(np.linalg.norm(a))
    return float(np.linalg.norm(a - b) / den)


def oracle_projs(scene):
    return O.project_views(scene)


def unpack_records(rec: np.ndarray, bins: np.ndarray) -> dict:
    """GPU records [V, n, 12] and binning records [V, n, 4] -> named fields."""
    tx = bins[..., 1].view(np.uint32)
    ty = bins[..., 2].view(np.uint32)
    rect = np.stack([tx & 0xFFFF, tx >> 16, ty & 0xFFFF, ty >> 16], -1).astype(np.int32)
    return dict(xy=rec[..., 0:2], conic=rec[..., 2:5], opacity=rec[..., 5], rgb=rec[..., 6:9],
                hx=rec[..., 9], hy=rec[..., 10], depth=bins[..., 0], rect=rect)


def pack_bins(projs) -> np.ndarray:
    """Oracle projections -> float32 binning records in the library's layout
    [V, n, 4]: depth key, packed tile ranges."""
    V = len(projs)
    n = projs[0]["xy"].shape[0]
    out = np.zeros((V, n, 4), np.float32)
    for v, p in enumerate(projs):
        out[v, :, 0] = p["key"]
        r = p["rect"].astype(np.int64)
        tx = (r[:, 0] & 0xFFFF) | ((r[:, 1] & 0xFFFF) << 16)
        ty = (r[:, 2] & 0xFFFF) | ((r[:, 3] & 0xFFFF) << 16)
        out[v, :, 1] = tx.astype(np.uint32).view(np.float32)
        out[v, :, 2] = ty.astype(np.uint32).view(np.float32)
        bad = p["valid"] == 0
        out[v, bad, 0] = 0
        out[v, bad, 1] = np.uint32(1).view(np.float32)
        out[v, bad, 2] = np.uint32(1).view(np.float32)
    return out


def ambiguous_tiles(scene, projs) -> np.ndarray:
    """Global tiles whose list may legitimately differ: those within one tile
    of the rectangle of a Gaussian whose radius / rectangle decision the oracle
    flags as too close to its threshold to be decided the same way by a double
    computation in another order (expected: none or a handful)."""
    tx, ty = tiles_of(scene)
    out = np.zeros((scene.n_views, ty, tx), bool)
    for v, p in enumerate(projs):
        for i in np.nonzero(p["ambiguous"])[0]:
            r = p["rect"][i]
            u, w, rr = p["xy"][i, 0], p["xy"][i, 1], p["radius"][i]
            x0 = max(0, int(np.floor((u - rr) / 16)) - 1)
            x1 = min(tx - 1, int(np.floor((u + rr) / 16)) + 1)
            y0 = max(0, int(np.floor((w - rr) / 16)) - 1)
            y1 = min(ty - 1, int(np.floor((w + rr) / 16)) + 1)
            if x0 <= x1 and y0 <= y1:
                out[v, y0:y1 + 1, x0:x1 + 1] = True
    return out.reshape(-1)


def ambiguous_pixels(scene, projs, pix) -> np.ndarray:
    tx, ty = tiles_of(scene)
    t = pix[:, 0] * tx * ty + (pix[:, 2] // 16) * tx + pix[:, 1] // 16
    return ambiguous_tiles(scene, projs)[t]


def tiles_of(scene):
    c = scene.cameras[0]
    return (c.width + 15) // 16, (c.height + 15) // 16


def gpu_tile_lists(ids: np.ndarray, ranges: np.ndarray, tiles: np.ndarray):
    return [ids[ranges[t, 0]:ranges[t, 1]] for t in tiles]


def compare_lists(gpu_ids, gpu_ranges, rects, keys, scene, tiles_global):
    """Bit-exact comparison of the GPU per-tile lists with the oracle's.
    ``tiles_global`` indexes view * tiles_per_view + tile."""
    tx, ty = tiles_of(scene)
    tpv = tx * ty
    req = np.stack([tiles_global // tpv, tiles_global % tpv], 1).astype(np.int32)
    counts, ids = O.tile_lists(rects, keys, [(tx, ty)] * scene.n_views, req)
    off = 0
    mism = 0
    for k, t in enumerate(tiles_global):
        want = ids[off:off + counts[k]]
        off += counts[k]
        got = gpu_ids[gpu_ranges[t, 0]:gpu_ranges[t, 1]]
        if got.shape != want.shape or not np.array_equal(got.astype(np.int64), want.astype(np.int64)):
            mism += 1
    return mism


def pixel_sample(scene, n_random=4096, rows=2, seed=5):
    """Seeded random pixels plus `rows` full tile rows of every view."""
    rng = np.random.default_rng(seed)
    out = []
    c = scene.cameras[0]
    for v in range(scene.n_views):
        xs = rng.integers(0, c.width, n_random)
        ys = rng.integers(0, c.height, n_random)
        out.append(np.stack([np.full(n_random, v), xs, ys], 1))
        tyn = (c.height + 15) // 16
        for r in rng.choice(tyn, size=min(rows, tyn), replace=False):
            y0, y1 = r * 16, min(c.height, r * 16 + 16)
            yy, xx = np.meshgrid(np.arange(y0, y1), np.arange(c.width), indexing="ij")
            out.append(np.stack([np.full(xx.size, v), xx.ravel(), yy.ravel()], 1))
    pix = np.concatenate(out).astype(np.int32)
    # unique, keep order
    _, idx = np.unique(pix, axis=0, return_index=True)
    return pix[np.sort(idx)]


def full_pixels(scene):
    c = scene.cameras[0]
    out = []
    for v in range(scene.n_views):
        yy, xx = np.meshgrid(np.arange(c.height), np.arange(c.width), indexing="ij")
        out.append(np.stack([np.full(xx.size, v), xx.ravel(), yy.ravel()], 1))
    return np.concatenate(out).astype(np.int32)


def compare_render(gpu_image, gpu_T, gpu_nc, ref, pix):
    """Colour / transmittance / contributor comparison on listed pixels.
    Returns a dict of statistics; asserts nothing."""
    v, x, y = pix[:, 0], pix[:, 1], pix[:, 2]
    g = gpu_image[v, :, y, x].astype(np.float64)           # [P, 3]
    d = np.abs(g - ref["color"])
    flagged = ref["flags"] != 0
    ok = ~flagged
    stats = dict(
        n=len(pix), flagged=int(flagged.sum()),
        max_abs=float(d[ok].max()) if ok.any() else 0.0,
        mean_abs=float(d[ok].mean()) if ok.any() else 0.0,
        max_abs_all=float(d.max()),
        nc_mismatch=int((gpu_nc[v, y, x].astype(np.int64) != ref["n_contrib"])[ok].sum()),
        T_max_rel=float((np.abs(gpu_T[v, y, x] - ref["T"]) / np.maximum(ref["T"], 1e-4))[ok].max())
        if ok.any() else 0.0,
    )
    return stats
