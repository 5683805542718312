"""Pins of the float64 oracle against facts fixed outside the oracle itself.

Each test checks the oracle against a closed form, an invariant, a textbook
table, a numerical derivative or a brute force written independently here, so
that a dropped term, a wrong sign or index, or a transposed operand in the
oracle fails at least one of them. No GPU is needed.
"""

import copy
import math

import numpy as np
import pytest

from gaussian_splatting_differentiable_ewa_b200 import scenes as S
from oracle import oracle as O


def _cam(f=100.0, W=64, H=64, viewmat=None, campos=(0, 0, 0), cx=None, cy=None):
    vm = np.concatenate([np.eye(3), np.zeros((3, 1))], 1) if viewmat is None else viewmat
    return S.Camera(viewmat=np.asarray(vm, np.float32), fx=f, fy=f,
                    cx=W / 2.0 if cx is None else cx, cy=H / 2.0 if cy is None else cy,
                    width=W, height=H, campos=np.asarray(campos, np.float32))


def _scene(means, log_scales, quats, logits, sh, deg, cams):
    n = len(means)
    m = np.zeros((n, 4)); m[:, :3] = means
    s = np.zeros((n, 4)); s[:, :3] = log_scales
    return S.Scene("t", means=m, log_scales=s, quats=np.asarray(quats, np.float64),
                   opacity_logit=np.asarray(logits, np.float64),
                   sh=np.asarray(sh, np.float64).reshape(n, (deg + 1) ** 2, 3),
                   sh_degree=deg, cameras=cams, background=np.zeros(3))


# ---------------------------------------------------------------- SH basis

def _sh_textbook(d):
    """Real SH to degree 3 from the standard table of real spherical harmonics
    (e.g. the 'table of spherical harmonics', real form), with the
    Condon-Shortley phase carried into the real form, i.e. the table's entries
    times (-1)^m for odd |m|. Index l*l + l + m."""
    x, y, z = d[:, 0], d[:, 1], d[:, 2]
    pi = math.pi
    Y = np.zeros((d.shape[0], 16))
    Y[:, 0] = 0.5 * math.sqrt(1 / pi)
    Y[:, 1] = -math.sqrt(3 / (4 * pi)) * y
    Y[:, 2] = math.sqrt(3 / (4 * pi)) * z
    Y[:, 3] = -math.sqrt(3 / (4 * pi)) * x
    Y[:, 4] = 0.5 * math.sqrt(15 / pi) * x * y
    Y[:, 5] = -0.5 * math.sqrt(15 / pi) * y * z
    Y[:, 6] = 0.25 * math.sqrt(5 / pi) * (3 * z * z - 1)
    Y[:, 7] = -0.5 * math.sqrt(15 / pi) * x * z
    Y[:, 8] = 0.25 * math.sqrt(15 / pi) * (x * x - y * y)
    Y[:, 9] = -0.25 * math.sqrt(35 / (2 * pi)) * y * (3 * x * x - y * y)
    Y[:, 10] = 0.5 * math.sqrt(105 / pi) * x * y * z
    Y[:, 11] = -0.25 * math.sqrt(21 / (2 * pi)) * y * (5 * z * z - 1)
    Y[:, 12] = 0.25 * math.sqrt(7 / pi) * z * (5 * z * z - 3)
    Y[:, 13] = -0.25 * math.sqrt(21 / (2 * pi)) * x * (5 * z * z - 1)
    Y[:, 14] = 0.25 * math.sqrt(105 / pi) * z * (x * x - y * y)
    Y[:, 15] = -0.25 * math.sqrt(35 / (2 * pi)) * x * (x * x - 3 * y * y)
    return Y


def _unit(rng, n):
    d = rng.normal(size=(n, 3))
    return d / np.linalg.norm(d, axis=1, keepdims=True)


def test_sh_matches_textbook_table():
    d = _unit(np.random.default_rng(0), 500)
    np.testing.assert_allclose(O.sh_basis(d, 3), _sh_textbook(d), rtol=0, atol=1e-12)


def test_sh_lower_degree_is_prefix():
    d = _unit(np.random.default_rng(1), 50)
    full = O.sh_basis(d, 3)
    for deg in range(3):
        k = (deg + 1) ** 2
        Y = O.sh_basis(d, deg)
        np.testing.assert_allclose(Y[:, :k], full[:, :k], atol=1e-14)
        assert np.all(Y[:, k:] == 0)


def test_sh_orthonormal_by_quadrature():
    # Gauss-Legendre in cos(theta) (16 nodes) x 32 uniform phi nodes integrates
    # products of degree-3 harmonics exactly.
    ct, w = np.polynomial.legendre.leggauss(16)
    phi = (np.arange(32) + 0.5) * 2 * math.pi / 32
    CT, PH = np.meshgrid(ct, phi, indexing="ij")
    W = np.repeat(w, 32) * (2 * math.pi / 32)
    st = np.sqrt(1 - CT.ravel() ** 2)
    d = np.stack([st * np.cos(PH.ravel()), st * np.sin(PH.ravel()), CT.ravel()], 1)
    Y = O.sh_basis(d, 3)
    G = (Y * W[:, None]).T @ Y
    np.testing.assert_allclose(G, np.eye(16), atol=1e-12)


# ---------------------------------------------------------------- projection

def test_point_projection_front_and_side_cameras():
    # camera at (0,0,-8) looking at the origin: world point (1, 0.5, 0) sits
    # at camera coordinates (1, 0.5, 8)
    c = (0.0, 0.0, -8.0)
    cam = _cam(f=1200.0, W=1920, H=1080, viewmat=S.look_at(c), campos=c)
    sc = _scene([[1.0, 0.5, 0.0]], [[-3, -3, -3]], [[1, 0, 0, 0]], [0.0], np.zeros(3), 0, [cam])
    p = O.project(sc, cam)
    np.testing.assert_allclose(p["xy"][0], [960 + 1200 / 8, 540 + 1200 * 0.5 / 8], atol=1e-9)
    assert abs(p["depth"][0] - 8.0) < 1e-12
    # camera at (8, 0, 0) looking at the origin: camera x axis is world +z
    c = (8.0, 0.0, 0.0)
    cam = _cam(f=1200.0, W=1920, H=1080, viewmat=S.look_at(c), campos=c)
    sc = _scene([[0.0, 0.5, 1.0]], [[-3, -3, -3]], [[1, 0, 0, 0]], [0.0], np.zeros(3), 0, [cam])
    p = O.project(sc, cam)
    np.testing.assert_allclose(p["xy"][0], [960 + 1200 / 8, 540 + 1200 * 0.5 / 8], atol=1e-9)
    assert abs(p["depth"][0] - 8.0) < 1e-12


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_isotropic_on_axis_closed_form_and_rotation_invariance(seed):
    rng = np.random.default_rng(seed)
    f, z = 150.0, 3.7
    ls = float(np.float32(rng.uniform(-3, -1)))
    q = rng.normal(size=(5, 4))
    q /= np.linalg.norm(q, axis=1, keepdims=True)
    cam = _cam(f=f, W=96, H=80)
    sc = _scene([[0, 0, z]] * 5, [[ls] * 3] * 5, q, [0.3] * 5, np.zeros((5, 3)), 0, [cam])
    p = O.project(sc, cam)
    s = math.exp(ls)
    var = (f * s / z) ** 2 + 0.3
    np.testing.assert_allclose(p["cov"], np.tile([var, 0, var], (5, 1)), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(p["conic"], np.tile([1 / var, 0, 1 / var], (5, 1)), rtol=1e-12, atol=1e-12)
    assert np.all(p["radius"] == math.ceil(3 * math.sqrt(var)))
    np.testing.assert_allclose(p["xy"], np.tile([48.0, 40.0], (5, 1)), atol=1e-12)


def test_anisotropic_rotation_about_z():
    # 45 degrees about z, quaternion (w, x, y, z) = (cos 22.5, 0, 0, sin 22.5):
    # Sigma_xy = (sx^2 - sy^2) / 2 (a transposed rotation flips its sign)
    f, z = 200.0, 5.0
    sx, sy, sz = 0.3, 0.1, 0.05
    h = math.radians(22.5)
    cam = _cam(f=f, W=64, H=64)
    sc = _scene([[0, 0, z]], [[math.log(sx), math.log(sy), math.log(sz)]],
                [[math.cos(h), 0, 0, math.sin(h)]], [0.0], np.zeros(3), 0, [cam])
    p = O.project(sc, cam)
    k = (f / z) ** 2
    A = k * (sx * sx + sy * sy) / 2 + 0.3
    B = k * (sx * sx - sy * sy) / 2
    np.testing.assert_allclose(p["cov"][0], [A, B, A], rtol=1e-12)
    # 90 degrees about z swaps the screen axes
    h = math.radians(45)
    sc = _scene([[0, 0, z]], [[math.log(sx), math.log(sy), math.log(sz)]],
                [[math.cos(h), 0, 0, math.sin(h)]], [0.0], np.zeros(3), 0, [cam])
    p = O.project(sc, cam)
    np.testing.assert_allclose(p["cov"][0], [k * sy * sy + 0.3, 0, k * sx * sx + 0.3], rtol=1e-12, atol=1e-12)


def test_ewa_covariance_matches_numerical_jacobian():
    # off-axis Gaussians seen by a rotated camera: the 2D covariance must be
    # J W Sigma W^T J^T + 0.3 I with J the Jacobian of the perspective map,
    # here taken by central differences of the pixel coordinates
    sc = S.make_scene("train_6m_8x1080p", seed=4, n=40, n_views=3)
    cam = sc.cameras[2]
    p = O.project(sc, cam)
    Wm = cam.viewmat.astype(np.float64)
    for i in range(sc.n):
        mu = sc.means[i, :3].astype(np.float64)
        t = Wm[:, :3] @ mu + Wm[:, 3]

        def uv(tt):
            return np.array([cam.fx * tt[0] / tt[2] + cam.cx, cam.fy * tt[1] / tt[2] + cam.cy])
        J = np.zeros((2, 3))
        for k in range(3):
            e = np.zeros(3); e[k] = 1e-6
            J[:, k] = (uv(t + e) - uv(t - e)) / 2e-6
        w, x, y, z = sc.quats[i].astype(np.float64) / np.linalg.norm(sc.quats[i].astype(np.float64))
        # rotation of a unit quaternion applied to basis vectors via q v q*
        def rot(v):
            qv = np.array([x, y, z])
            return v + 2 * w * np.cross(qv, v) + 2 * np.cross(qv, np.cross(qv, v))
        R = np.stack([rot(e) for e in np.eye(3)], 1)
        s = np.exp(sc.log_scales[i, :3].astype(np.float64))
        Sig = R @ np.diag(s * s) @ R.T
        M = J @ Wm[:, :3]
        cov = M @ Sig @ M.T + 0.3 * np.eye(2)
        np.testing.assert_allclose(p["cov"][i], [cov[0, 0], cov[0, 1], cov[1, 1]], rtol=1e-6)
        np.testing.assert_allclose(p["xy"][i], uv(t), rtol=1e-12)


def test_sh_colour_uses_direction_from_camera_centre():
    c = np.array([0.5, -1.0, -6.0])
    cam = _cam(f=100.0, W=64, H=64, viewmat=S.look_at(c), campos=c)
    mu = np.array([0.2, 0.3, 0.1])
    sh = np.zeros((1, 16, 3)); sh[0, 2, :] = [0.4, -0.4, 2.0]      # Y_1,0 only
    sc = _scene([mu], [[-3] * 3], [[1, 0, 0, 0]], [0.0], sh, 3, [cam])
    p = O.project(sc, cam)
    d = (mu - c) / np.linalg.norm(mu - c)
    y10 = math.sqrt(3 / (4 * math.pi)) * d[2]
    raw = 0.5 + y10 * np.array([0.4, -0.4, 2.0])
    np.testing.assert_allclose(p["rgb"][0], np.maximum(raw, 0), atol=1e-12)
    assert p["clamp"][0] == sum(1 << c for c in range(3) if raw[c] <= 0)


def test_culling_near_plane_and_outside_image():
    cam = _cam(f=100.0, W=64, H=64)
    sc = _scene([[0, 0, 0.19], [0, 0, 0.21], [50, 0, 2.0], [0, 0, 3]], [[-5] * 3] * 4,
                [[1, 0, 0, 0]] * 4, [0.0] * 4, np.zeros((4, 3)), 0, [cam])
    p = O.project(sc, cam)
    assert list(p["valid"]) == [0, 1, 0, 1]
    assert p["radius"][0] == 0 and p["radius"][2] == 0
    assert p["rect"][0][0] > p["rect"][0][1]


def test_tile_rect_floor_semantics():
    # the rectangle is floor((u -+ r)/16) clamped to the grid: a Gaussian whose
    # extent ends exactly on a tile edge touches the next tile
    cam = _cam(f=1.0, W=64, H=48, cx=0.0, cy=0.0)
    # make u = 32 exactly (t = (32, 24, 1) with f = 1), radius from the covariance
    # flat along z so that the third column of the Jacobian adds nothing
    sc = _scene([[32.0, 24.0, 1.0]], [[math.log(2.0), math.log(2.0), -20.0]], [[1, 0, 0, 0]],
                [0.0], np.zeros(3), 0, [cam])
    p = O.project(sc, cam)
    r = p["radius"][0]
    assert r == math.ceil(3 * math.sqrt(4.0 + 0.3))
    tx0, tx1, ty0, ty1 = p["rect"][0]
    assert (tx0, tx1) == (max(0, math.floor((32 - r) / 16)), min(3, math.floor((32 + r) / 16)))
    assert (ty0, ty1) == (max(0, math.floor((24 - r) / 16)), min(2, math.floor((24 + r) / 16)))


# ---------------------------------------------------------------- binning

def test_tile_lists_match_python_brute_force():
    rng = np.random.default_rng(7)
    V, n = 2, 300
    tiles = [(5, 4), (5, 4)]
    rects = np.zeros((V, n, 4), np.int32)
    for v in range(V):
        for i in range(n):
            if rng.random() < 0.1:
                rects[v, i] = [1, 0, 1, 0]
                continue
            x0 = rng.integers(0, 5); x1 = rng.integers(x0, 5)
            y0 = rng.integers(0, 4); y1 = rng.integers(y0, 4)
            rects[v, i] = [x0, x1, y0, y1]
    keys = rng.choice(np.float32([1.0, 1.5, 2.25, 7.0]), size=(V, n)).astype(np.float32)
    req = np.array([[v, t] for v in range(V) for t in range(20)], np.int32)
    counts, ids = O.tile_lists(rects, keys, tiles, req)
    off = 0
    for (v, t), c in zip(req, counts):
        tx, ty = t % 5, t // 5
        expect = [i for i in range(n)
                  if rects[v, i, 0] <= tx <= rects[v, i, 1] and rects[v, i, 2] <= ty <= rects[v, i, 3]]
        expect.sort(key=lambda i: (keys[v, i], i))
        assert list(ids[off:off + c]) == expect
        off += c


# ---------------------------------------------------------------- compositing

def _proj2d(xy, conic, opac, rgb, keys, W, H):
    n = len(xy)
    tx, ty = (W + 15) // 16, (H + 15) // 16
    return dict(xy=np.asarray(xy, float), conic=np.asarray(conic, float),
                opacity=np.asarray(opac, float), rgb=np.asarray(rgb, float),
                key=np.asarray(keys, np.float32),
                rect=np.tile([0, tx - 1, 0, ty - 1], (n, 1)).astype(np.int32),
                valid=np.ones(n, np.int32))


def _alpha(p, i, px, py):
    d0 = px + 0.5 - p["xy"][i][0]; d1 = py + 0.5 - p["xy"][i][1]
    a, b, c = p["conic"][i]
    return min(0.99, p["opacity"][i] * math.exp(-0.5 * (a * d0 * d0 + 2 * b * d0 * d1 + c * d1 * d1)))


def test_single_gaussian_centred_on_pixel_gives_o_c():
    cam = _cam(W=32, H=32)
    bg = np.array([0.1, 0.2, 0.3])
    p = _proj2d([[10.5, 7.5]], [[0.3, 0.1, 0.2]], [0.7], [[0.2, 0.6, 0.9]], [1.0], 32, 32)
    r = O.render([p], [cam], bg, np.array([[0, 10, 7]]))
    np.testing.assert_allclose(r["color"][0], 0.7 * np.array([0.2, 0.6, 0.9]) + 0.3 * bg, atol=1e-15)
    assert abs(r["T"][0] - 0.3) < 1e-15 and r["n_contrib"][0] == 1


def test_render_flags_follow_the_given_error_bound():
    """The comparator inputs of orc_render: with a per-splat relative alpha
    error bound e, an evaluation whose alpha lies within e of 1/255 is
    flagged and one outside is not; a trial transmittance is flagged within
    the transmittance bound the alphas in front imply; flag_dev / flag_T add
    up what a flagged decision can change (2.02 T a and T a / (1 - a) for a
    skip, 2.02 T and T for a stop)."""
    cam = _cam(W=32, H=32)
    bg = np.zeros(3)
    pix = np.array([[0, 10, 7]])
    # one splat centred on the pixel: alpha = o exactly
    for rel, flagged in ((3e-6, True), (-3e-6, True), (2e-5, False), (-2e-5, False)):
        o = (1.0 / 255.0) * (1.0 + rel)
        p = _proj2d([[10.5, 7.5]], [[0.3, 0.1, 0.2]], [o], [[1.0, 1.0, 1.0]], [1.0], 32, 32)
        err = np.array([[[1e-5, 0.0]]])
        r = O.render([p], [cam], bg, pix, alpha_err=err)
        assert bool(r["flags"][0] & 1) == flagged, rel
        assert (r["flags"][0] & 2) == 0
        if flagged:
            np.testing.assert_allclose(r["flag_dev"][0], 2.02 * max(o, 1 / 255.0), rtol=1e-12)
            a = max(o, 1 / 255.0)
            np.testing.assert_allclose(r["flag_T"][0], a / (1 - a), rtol=1e-12)
        else:
            assert r["flag_dev"][0] == 0.0 and r["flag_T"][0] == 0.0
        # without a bound nothing is flagged
        assert O.render([p], [cam], bg, pix)["flags"][0] == 0
    # the bound grows with q: one pixel away from the centre (q = 0.3),
    # alpha 4e-6 above 1/255 is inside e1 q for e1 = 2e-5, outside for 1e-5
    a = 0.3
    q = a * 1.0 * 1.0
    o_edge = (1.0 / 255.0) * (1 + 4e-6) / math.exp(-0.5 * q)
    p = _proj2d([[11.5, 7.5]], [[a, 0.0, a]], [o_edge], [[1.0, 1.0, 1.0]], [1.0], 32, 32)
    assert O.render([p], [cam], bg, pix, alpha_err=np.array([[[0.0, 2e-5]]]))["flags"][0] & 1
    assert not O.render([p], [cam], bg, pix, alpha_err=np.array([[[0.0, 1e-5]]]))["flags"][0]
    # a layer of alpha 0.99 leaves T = 0.01 in front of a second of alpha
    # 0.99 - 1e-9, whose trial T is a hair (1e-7 relative) above 1e-4: flagged
    # with a bound, not without
    xy = [[10.5, 7.5]] * 3
    opac = [0.99, 0.99 - 1e-9, 0.5]
    p = _proj2d(xy, [[0.3, 0.0, 0.3]] * 3, opac, [[1.0, 0.0, 0.0]] * 3, [1.0, 2.0, 3.0], 32, 32)
    r0 = O.render([p], [cam], bg, pix)
    assert r0["flags"][0] == 0 and r0["n_contrib"][0] == 2
    r1 = O.render([p], [cam], bg, pix, alpha_err=np.full((1, 3, 2), [1e-6, 0.0]))
    assert r1["flags"][0] & 2
    # the stop taken the other way at the second splat, with T = 0.01 in front
    np.testing.assert_allclose(r1["flag_T"][0], 0.01, rtol=1e-9)
    np.testing.assert_allclose(r1["flag_dev"][0], 2.02 * 0.01, rtol=1e-9)


def test_two_gaussians_front_to_back():
    cam = _cam(W=32, H=32)
    p = _proj2d([[10.2, 7.9], [11.0, 6.5]], [[0.3, 0.1, 0.2], [0.1, -0.02, 0.15]], [0.6, 0.8],
                [[0.2, 0.6, 0.9], [0.9, 0.1, 0.4]], [2.0, 1.0], 32, 32)
    r = O.render([p], [cam], np.zeros(3), np.array([[0, 10, 7]]))
    a0, a1 = _alpha(p, 0, 10, 7), _alpha(p, 1, 10, 7)      # Gaussian 1 is in front
    expect = p["rgb"][1] * a1 + p["rgb"][0] * a0 * (1 - a1)
    np.testing.assert_allclose(r["color"][0], expect, atol=1e-14)
    np.testing.assert_allclose(r["T"][0], (1 - a0) * (1 - a1), atol=1e-15)


def test_opaque_front_layers_hide_everything_behind():
    cam = _cam(W=32, H=32)
    xy = [[8.5, 8.5]] * 3 + [[8.0, 9.0], [9.0, 8.0]]
    conic = [[1e-4, 0, 1e-4]] * 5
    base = _proj2d(xy, conic, [1.0, 1.0, 1.0, 0.5, 0.9], [[1, 0, 0], [0, 1, 0], [0, 0, 1],
                   [0.3, 0.3, 0.3], [0.7, 0.2, 0.1]], [1.0, 2.0, 3.0, 4.0, 5.0], 32, 32)
    pix = np.array([[0, 8, 8]])
    r0 = O.render([base], [cam], np.array([0.5, 0.5, 0.5]), pix)
    other = copy.deepcopy(base)
    other["rgb"][3:] = [[0.0, 1.0, 0.5], [1.0, 1.0, 1.0]]
    other["opacity"][3:] = [0.95, 0.05]
    r1 = O.render([other], [cam], np.array([0.5, 0.5, 0.5]), pix)
    assert np.array_equal(r0["color"], r1["color"])
    # two 0.99 layers leave T = 1e-4 (just above the limit); the third would
    # take it below 1e-4 and stops the pixel before being added
    assert r0["n_used"][0] == 2 and r0["n_contrib"][0] == 2
    g = O.render_bwd([base], [cam], np.zeros(3), pix, np.ones((1, 3)))
    assert np.all(g[0, 2:] == 0)


def test_alpha_below_threshold_is_skipped():
    cam = _cam(W=32, H=32)
    o = (1.0 / 255.0) * 0.999
    p = _proj2d([[5.5, 5.5]], [[0.1, 0, 0.1]], [o], [[1, 1, 1]], [1.0], 32, 32)
    r = O.render([p], [cam], np.zeros(3), np.array([[0, 5, 5]]))
    assert np.all(r["color"][0] == 0) and r["T"][0] == 1.0 and r["n_exp"][0] == 0


def test_permutation_invariance_and_transmittance_bounds():
    sc = S.make_scene("fwd_1k_128", seed=3, n=300)
    cam = sc.cameras[0]
    p = O.project(sc, cam)
    H, W = 128, 128
    ys, xs = np.meshgrid(np.arange(0, H, 3), np.arange(0, W, 3), indexing="ij")
    pix = np.stack([np.zeros(xs.size, int), xs.ravel(), ys.ravel()], 1)
    r0 = O.render([p], [cam], np.zeros(3), pix)
    perm = np.random.default_rng(0).permutation(sc.n)
    sc2 = copy.deepcopy(sc)
    for k in ("means", "log_scales", "quats", "opacity_logit", "sh"):
        setattr(sc2, k, getattr(sc, k)[perm])
    p2 = O.project(sc2, cam)
    assert len(np.unique(p["key"][p["valid"] == 1])) == int(p["valid"].sum())
    r2 = O.render([p2], [cam], np.zeros(3), pix)
    np.testing.assert_allclose(r2["color"], r0["color"], atol=1e-13)
    assert np.all((r0["T"] >= 1e-4) & (r0["T"] <= 1.0))
    assert np.all(r0["color"] >= 0)


# ---------------------------------------------------------------- gradients

def _fd_case(seed, deg):
    sc = S.make_scene("fwd_100k_800" if deg else "fwd_1k_128", seed=seed, n=10, width=48, height=40)
    if deg:
        sc.log_scales[:, :3] += 2.5
        sc.means[:, :3] *= 0.5
    for k in ("means", "log_scales", "quats", "opacity_logit", "sh"):
        setattr(sc, k, getattr(sc, k).astype(np.float64))
    return sc


@pytest.mark.parametrize("seed,deg", [(3, 3), (11, 3), (5, 0)])
def test_gradients_match_central_differences(seed, deg):
    _check_central_differences(_fd_case(seed, deg), seed)


def _clamp_case():
    """The finite-difference scene with both clamps reached: Gaussian 0 is an
    opaque (logit 8, opacity 0.99966), round, front-most splat over the image
    centre, so alpha = min(0.99, o exp(-q/2)) clamps on the pixels within
    ~0.14 sigma of its mean; Gaussians 1 and 2 have a colour channel (red,
    blue) whose SH sum is far below 0, so max(0, .) clamps it."""
    sc = _fd_case(3, 3)
    sc.means[0, :3] = (0.05, -0.03, -3.0)       # depth 5, in front of the rest
    sc.log_scales[0, :3] = 0.2
    sc.opacity_logit[0] = 8.0
    sc.sh[1, 0, 0] = -4.0
    sc.sh[2, 0, 2] = -4.0
    return sc


def test_clamp_branches_are_reached_and_match_central_differences():
    sc = _clamp_case()
    cam = sc.cameras[0]
    pr = O.project_views(sc)[0]
    # the colour clamp holds for red of Gaussian 1 and blue of Gaussian 2
    assert pr["clamp"][1] & 1 and pr["clamp"][2] & 4
    assert pr["rgb"][1, 0] == 0.0 and pr["rgb"][2, 2] == 0.0
    # the alpha clamp holds on a few pixels of Gaussian 0
    ys, xs = np.meshgrid(np.arange(cam.height) + 0.5, np.arange(cam.width) + 0.5, indexing="ij")
    d0, d1 = xs - pr["xy"][0, 0], ys - pr["xy"][0, 1]
    a, b, c = pr["conic"][0]
    araw = pr["opacity"][0] * np.exp(-0.5 * (a * d0 * d0 + 2 * b * d0 * d1 + c * d1 * d1))
    assert (araw >= 0.99).sum() >= 3
    # every gradient, the clamped ones included, against central differences
    _check_central_differences(sc, 3)


def test_clamped_alpha_passes_colour_gradient_only():
    """On a pixel where the front-most splat's alpha is clamped at 0.99, the
    pixel's gradient reaches that splat's colour (d C / d c = alpha T = 0.99)
    and nothing else: its opacity, its conic and its screen-space mean do not
    move the pixel (the 3D mean still moves it through the view-dependent
    colour, so the central differences below perturb the logit, the scales
    and the rotation)."""
    sc = _clamp_case()
    cam = sc.cameras[0]
    pr = O.project_views(sc)
    x, y = int(pr[0]["xy"][0, 0]), int(pr[0]["xy"][0, 1])
    pix = np.array([[0, x, y]])
    d0, d1 = x + 0.5 - pr[0]["xy"][0, 0], y + 0.5 - pr[0]["xy"][0, 1]
    a, b, c = pr[0]["conic"][0]
    assert pr[0]["opacity"][0] * np.exp(-0.5 * (a * d0 * d0 + 2 * b * d0 * d1 + c * d1 * d1)) \
        >= 0.99
    gC = np.array([[0.3, -0.2, 0.5]])
    bg = np.array([0.2, 0.5, 0.1])
    g = O.render_bwd(pr, sc.cameras, bg, pix, gC)[0, 0]
    assert np.all(g[[0, 1, 2, 3, 4, 5, 9]] == 0.0)
    np.testing.assert_allclose(g[6:9], 0.99 * gC[0], rtol=1e-12)
    # the same by central differences of that pixel's colour
    for k in ("opacity_logit", "log_scales", "quats"):
        for j in range(getattr(sc, k).reshape(sc.n, -1).shape[1]):
            vals = []
            for sgn in (1, -1):
                s2 = copy.deepcopy(sc)
                getattr(s2, k).reshape(sc.n, -1)[0, j] += sgn * 1e-5
                p2 = O.project_views(s2)
                vals.append((O.render(p2, s2.cameras, bg, pix)["color"] * gC).sum())
            assert abs(vals[0] - vals[1]) < 1e-12, (k, j)


def _check_central_differences(sc, seed):
    cam = sc.cameras[0]
    ys, xs = np.meshgrid(np.arange(cam.height), np.arange(cam.width), indexing="ij")
    pix = np.stack([np.zeros(xs.size, int), xs.ravel(), ys.ravel()], 1)
    gC = np.random.default_rng(seed + 100).normal(0, 0.1, (pix.shape[0], 3))
    bg = np.array([0.2, 0.5, 0.1])

    def evaluate(scene):
        pr = O.project_views(scene)
        r = O.render(pr, scene.cameras, bg, pix)
        return float((r["color"] * gC).sum()), (r["sig"], r["n_contrib"], pr[0]["radius"],
                                                pr[0]["rect"], pr[0]["clamp"])

    pr = O.project_views(sc)
    g2 = O.render_bwd(pr, sc.cameras, bg, pix, gC)
    an = O.project_bwd(sc, pr, g2)
    h = 1e-5
    checked = 0
    for field in ("means", "log_scales", "quats", "opacity_logit", "sh"):
        a = an[field].reshape(sc.n, -1)
        num = np.zeros_like(a)
        keep = np.ones_like(a, bool)
        width = a.shape[1]
        for i in range(sc.n):
            for k in range(width):
                vals, sigs = [], []
                for sgn in (1, -1):
                    s2 = copy.deepcopy(sc)
                    getattr(s2, field).reshape(sc.n, -1)[i, k] += sgn * h
                    L, sg = evaluate(s2)
                    vals.append(L); sigs.append(sg)
                # a discrete decision changed between the two evaluations:
                # the function is not differentiable there; drop the sample
                if not all(np.array_equal(x, y) for x, y in zip(*sigs)):
                    keep[i, k] = False
                num[i, k] = (vals[0] - vals[1]) / (2 * h)
        if np.linalg.norm(num[keep]) < 1e-12:
            continue
        err = np.linalg.norm((a - num)[keep]) / np.linalg.norm(num[keep])
        assert err < 1e-5, (field, err)
        assert keep.mean() > 0.8
        checked += 1
    assert checked >= 4


def test_screen_space_gradients_match_central_differences():
    # dL/d(u, v, conic, opacity, rgb) of the compositing alone
    cam = _cam(W=40, H=40)
    rng = np.random.default_rng(2)
    n = 8
    xy = rng.uniform(5, 35, (n, 2))
    L = rng.normal(size=(n, 2, 2)) * 0.3
    cov = np.einsum("nij,nkj->nik", L, L) + 4 * np.eye(2)
    inv = np.linalg.inv(cov)
    conic = np.stack([inv[:, 0, 0], inv[:, 0, 1], inv[:, 1, 1]], 1)
    p = _proj2d(xy, conic, rng.uniform(0.3, 0.95, n), rng.uniform(0, 1, (n, 3)),
                rng.permutation(n).astype(np.float32) + 1, 40, 40)
    ys, xs = np.meshgrid(np.arange(40), np.arange(40), indexing="ij")
    pix = np.stack([np.zeros(xs.size, int), xs.ravel(), ys.ravel()], 1)
    gC = rng.normal(0, 0.1, (pix.shape[0], 3))
    bg = np.array([0.3, 0.1, 0.7])
    g = O.render_bwd([p], [cam], bg, pix, gC)[0]
    fields = [("xy", 0), ("xy", 1), ("conic", 0), ("conic", 1), ("conic", 2), ("opacity", None),
              ("rgb", 0), ("rgb", 1), ("rgb", 2)]
    h = 1e-6
    for j, (f, c) in enumerate(fields):
        num = np.zeros(n)
        for i in range(n):
            vals = []
            for sgn in (1, -1):
                q = copy.deepcopy(p)
                if c is None:
                    q[f][i] += sgn * h
                else:
                    q[f][i, c] += sgn * h
                vals.append((O.render([q], [cam], bg, pix)["color"] * gC).sum())
            num[i] = (vals[0] - vals[1]) / (2 * h)
        np.testing.assert_allclose(g[:, j], num, rtol=1e-5, atol=1e-9)


def test_absolute_gradient_bounds_plain_gradient():
    sc = S.make_scene("fwd_1k_128", seed=9, n=200)
    cam = sc.cameras[0]
    p = O.project(sc, cam)
    ys, xs = np.meshgrid(np.arange(128), np.arange(128), indexing="ij")
    pix = np.stack([np.zeros(xs.size, int), xs.ravel(), ys.ravel()], 1)
    gC = np.random.default_rng(4).normal(0, 0.1, (pix.shape[0], 3))
    g = O.render_bwd([p], [cam], np.zeros(3), pix, gC)
    plain, absg, den = O.densify_stats(g, p["valid"][None])
    assert np.all(absg >= plain * (1 - 1e-12))
    assert np.sum(absg > plain * (1 + 1e-6)) > 10
    assert np.array_equal(den, p["valid"])
    # one pixel: plain equals absolute
    g1 = O.render_bwd([p], [cam], np.zeros(3), pix[5000:5001], gC[5000:5001])
    pl1, ab1, _ = O.densify_stats(g1, p["valid"][None])
    np.testing.assert_allclose(pl1, ab1, rtol=1e-12, atol=1e-300)


# ---------------------------------------------------------------- Adam

def test_adam_closed_forms():
    rng = np.random.default_rng(0)
    p0 = rng.normal(size=100); g1 = rng.normal(size=100); g2 = rng.normal(size=100)
    g1[:5] = 0
    lr, eps = 1e-3, 1e-15
    z = np.zeros(100)
    p1, m1, v1 = O.adam(p0, g1, z, z, lr, 1, eps=eps)
    # step 1: m_hat = g, v_hat = g^2, so p1 = p0 - lr g / (|g| + eps)
    np.testing.assert_allclose(p1, p0 - lr * g1 / (np.abs(g1) + eps), rtol=0, atol=1e-15)
    assert np.array_equal(p1[:5], p0[:5])
    p2, m2, v2 = O.adam(p1, g2, m1, v1, lr, 2, eps=eps)
    m_hat = (0.9 * 0.1 * g1 + 0.1 * g2) / (1 - 0.81)
    v_hat = (0.999 * 0.001 * g1 ** 2 + 0.001 * g2 ** 2) / (1 - 0.999 ** 2)
    np.testing.assert_allclose(p2, p1 - lr * m_hat / (np.sqrt(v_hat) + eps), rtol=1e-12)
    p3, _, _ = O.adam(p0, np.zeros(100), z, z, lr, 1)
    assert np.array_equal(p3, p0)


# ------------------------------------------------------------ densify_and_prune

def _dp_set(n, K=1, seed=0):
    rng = np.random.default_rng(seed)
    params = dict(means=rng.normal(size=(n, 3)), log_scales=rng.uniform(-4, -1, (n, 3)),
                  quats=rng.normal(size=(n, 4)), opacity_logit=rng.normal(size=n),
                  sh=rng.normal(size=(n, K, 3)))
    params = {k: v.astype(np.float32).astype(np.float64) for k, v in params.items()}
    moments = {k: (rng.normal(size=v.shape), rng.random(v.shape)) for k, v in params.items()}
    return params, moments


def test_dp_rotation_is_the_axis_angle_rotation():
    # the sandwich product agrees with Rodrigues' formula for angle t about a
    rng = np.random.default_rng(3)
    for _ in range(20):
        a = rng.normal(size=3)
        a /= np.linalg.norm(a)
        t = rng.uniform(-np.pi, np.pi)
        q = np.concatenate([[np.cos(t / 2)], np.sin(t / 2) * a])
        u = rng.normal(size=3)
        rod = u * np.cos(t) + np.cross(a, u) * np.sin(t) + a * np.dot(a, u) * (1 - np.cos(t))
        np.testing.assert_allclose(O._rotate(q, u), rod, atol=1e-12)


def test_dp_split_child_closed_form():
    params, moments = _dp_set(1)
    params["quats"][0] = [3.0, 0.0, 0.0, 0.0]          # identity after normalisation
    params["log_scales"][0] = np.log([2.0, 1.0, 0.5])
    params["opacity_logit"][0] = 2.0
    z = np.array([[[1.0, -1.0, 2.0], [0.0, 0.5, 0.0]]])
    out, mom, code = O.densify_and_prune(params, moments, [1.0], [1], z, 0.5,
                                         np.log(1.5), -10.0, 10.0)
    assert code.tolist() == [O.DP_SPLIT]
    mu = params["means"][0]
    np.testing.assert_allclose(out["means"], [mu + [2.0, -1.0, 1.0], mu + [0.0, 0.5, 0.0]],
                               atol=1e-12)
    np.testing.assert_allclose(out["log_scales"],
                               np.log([[1.25, 0.625, 0.3125]] * 2), atol=1e-12)
    for k in ("quats", "opacity_logit", "sh"):
        assert np.array_equal(out[k], np.stack([params[k][0]] * 2))
        assert not mom[k][0].any() and not mom[k][1].any()


def test_dp_decisions_order_copies_and_moments():
    # 0 keep (cold), 1 clone (hot, small), 2 split (hot, large), 3 prune (faint),
    # 4 prune beats split (hot, large, faint), 5 keep (never seen: denom 0),
    # 6 prune (oversized)
    params, moments = _dp_set(7, K=4)
    small, large = np.log(0.01), np.log(0.2)
    params["log_scales"][:] = small
    params["log_scales"][[2, 4], 1] = large
    params["log_scales"][6, 2] = np.log(5.0)
    params["opacity_logit"][:] = 1.0
    params["opacity_logit"][[3, 4]] = -8.0
    accum = np.array([0.1, 3.0, 3.0, 3.0, 3.0, 3.0, 0.1])
    denom = np.array([1, 2, 2, 2, 2, 0, 1])
    z = np.random.default_rng(1).normal(size=(7, 2, 3))
    out, mom, code = O.densify_and_prune(params, moments, accum, denom, z, 1.0, np.log(0.1),
                                         -5.0, np.log(1.0))
    assert code.tolist() == [O.DP_KEEP, O.DP_CLONE, O.DP_SPLIT, O.DP_PRUNE, O.DP_PRUNE,
                             O.DP_KEEP, O.DP_PRUNE]
    # layout: g0, g1, g1 (clone), child 2a, child 2b, g5
    assert len(out["means"]) == 6
    for k in O.PARAM_NAMES:
        for row, src in ((0, 0), (1, 1), (2, 1), (5, 5)):
            assert np.array_equal(out[k][row], params[k][src]), (k, row)
        for row, src in ((0, 0), (1, 1), (5, 5)):                 # kept: moments kept
            assert np.array_equal(mom[k][0][row], moments[k][0][src])
            assert np.array_equal(mom[k][1][row], moments[k][1][src])
        for row in (2, 3, 4):                                       # new: moments zero
            assert not mom[k][0][row].any() and not mom[k][1][row].any()
    # children: the scales shrink by 1.6, the offsets are R (s * z)
    assert np.allclose(out["log_scales"][3], params["log_scales"][2] - np.log(1.6))
    d = out["means"][3:5] - params["means"][2]
    assert np.allclose(np.linalg.norm(d, axis=1),
                       np.linalg.norm(np.exp(params["log_scales"][2]) * z[2], axis=1))


def test_dp_threshold_is_strict_and_exact_in_float32():
    # accum == threshold * denom exactly is not above it; one ulp more is
    params, moments = _dp_set(2)
    params["log_scales"][:] = -5.0
    params["opacity_logit"][:] = 0.0
    thr = np.float32(0.0002)
    acc = np.array([np.float32(thr * np.float32(3)),
                    np.nextafter(np.float32(thr * np.float32(3)), np.float32(1))])
    code = O.densify_decisions(params["log_scales"], params["opacity_logit"], acc, [3, 3],
                               thr, np.log(0.1), -10.0, 10.0)
    assert code.tolist() == [O.DP_KEEP, O.DP_CLONE]


# ---------------------------------------------------------------- L1 + D-SSIM loss

def _gauss1d(size=11, sigma=1.5):
    """Normalised 1-D Gaussian taps; the 2-D SSIM window is their outer product."""
    g = np.array([math.exp(-((k - size // 2) ** 2) / (2 * sigma * sigma)) for k in range(size)])
    return g / g.sum()


def test_ssim_window_is_the_normalised_gaussian():
    w = O.ssim_window()
    assert w.shape == (11, 11)
    assert abs(w.sum() - 1.0) < 1e-15
    c = 5
    assert w[c, c + 1] / w[c, c] == pytest.approx(math.exp(-1 / 4.5), rel=1e-14)
    assert w[c + 2, c - 1] / w[c, c] == pytest.approx(math.exp(-5 / 4.5), rel=1e-14)
    g = _gauss1d()
    np.testing.assert_allclose(w, np.outer(g, g), rtol=1e-13, atol=0)


def test_ssim_of_an_image_with_itself_is_one_and_loss_zero():
    rng = np.random.default_rng(3)
    x = rng.random((2, 3, 17, 21))
    S = O.ssim_map(x, x)
    np.testing.assert_allclose(S, 1.0, rtol=0, atol=1e-12)
    terms, grad = O.l1_dssim_loss(x, x)
    np.testing.assert_allclose(terms, [[0.0, 0.0, 1.0]] * 2, atol=1e-12)
    assert np.abs(grad).max() < 1e-14


def _window_mass(H, W, y, x):
    """Weight of the 11 x 11 window that falls inside an H x W image at (y, x)."""
    g = _gauss1d()
    rows = sum(g[i] for i in range(11) if 0 <= y + i - 5 < H)
    cols = sum(g[j] for j in range(11) if 0 <= x + j - 5 < W)
    return rows * cols


def test_ssim_of_constant_planes_closed_form():
    """x = a, y = b everywhere: inside, S = (2ab + C1) / (a^2 + b^2 + C1) (no
    variance, the contrast-structure factor is C2 / C2); at the border the
    zero padding leaves window mass m < 1, so mx = a m, var x = a^2 m (1 - m),
    cov = a b m (1 - m)."""
    a, b, H, W = 0.5, 0.25, 20, 24
    S = O.ssim_map(np.full((H, W), a), np.full((H, W), b))
    assert S[10, 12] == pytest.approx((0.25 + 1e-4) / (0.3125 + 1e-4), rel=1e-13)
    C1, C2 = 1e-4, 9e-4
    for (yy, xx) in [(0, 0), (0, 7), (3, 23), (19, 2), (10, 12)]:
        m = _window_mass(H, W, yy, xx)
        v = m * (1 - m)
        want = ((2 * a * b * m * m + C1) * (2 * a * b * v + C2)
                / (((a * a + b * b) * m * m + C1) * ((a * a + b * b) * v + C2)))
        assert S[yy, xx] == pytest.approx(want, rel=1e-12), (yy, xx)


def test_ssim_of_a_checkerboard_against_its_mean():
    """x = 0.5 + 0.25 (-1)^(i+j) against y = 0.5: the window's alternating sum
    A = (sum_k g_k (-1)^k)^2 gives mx = 0.5 + 0.25 s A (s the pixel's parity
    sign) and var x = 0.0625 (1 - A^2); y has no variance and no covariance."""
    H, W = 24, 24
    ii, jj = np.meshgrid(np.arange(H), np.arange(W), indexing="ij")
    x = 0.5 + 0.25 * (-1.0) ** (ii + jj)
    y = np.full((H, W), 0.5)
    S = O.ssim_map(x, y)
    g = _gauss1d()
    A = sum(g[k] * (-1) ** (k - 5) for k in range(11)) ** 2
    C1, C2 = 1e-4, 9e-4
    for (yy, xx) in [(11, 11), (11, 12), (8, 15)]:
        s = (-1.0) ** (yy + xx)
        mx = 0.5 + 0.25 * s * A
        vx = 0.0625 * (1 - A * A)
        want = (2 * mx * 0.5 + C1) * C2 / ((mx * mx + 0.25 + C1) * (vx + C2))
        assert S[yy, xx] == pytest.approx(want, rel=1e-12)


def test_ssim_against_brute_force_patch_statistics():
    """Each pixel's statistics taken directly from its zero-padded 11 x 11
    patch in centred form, sum w (x - mx)(y - my), instead of the moment maps."""
    rng = np.random.default_rng(5)
    H, W = 23, 29
    x, y = rng.random((H, W)), rng.random((H, W))
    S = O.ssim_map(x, y)
    w = np.outer(_gauss1d(), _gauss1d())
    px = np.pad(x, 5)
    py = np.pad(y, 5)
    C1, C2 = 1e-4, 9e-4
    for (yy, xx) in [(0, 0), (0, 28), (22, 0), (22, 28), (11, 14), (4, 9), (17, 3)]:
        P = px[yy:yy + 11, xx:xx + 11]
        Q = py[yy:yy + 11, xx:xx + 11]
        mx, my = (w * P).sum(), (w * Q).sum()
        vx, vy = (w * (P - mx) ** 2).sum(), (w * (Q - my) ** 2).sum()
        cxy = (w * (P - mx) * (Q - my)).sum()
        lum = (2 * mx * my + C1) / (mx * mx + my * my + C1)
        cs = (2 * cxy + C2) / (vx + vy + C2)
        assert S[yy, xx] == pytest.approx(lum * cs, rel=1e-12), (yy, xx)


def test_loss_terms_weights_and_symmetry():
    rng = np.random.default_rng(6)
    x, y = rng.random((2, 3, 14, 19)), rng.random((2, 3, 14, 19))
    t0, _ = O.l1_dssim_loss(x, y, lam=0.0)
    t1, _ = O.l1_dssim_loss(x, y, lam=1.0)
    t, _ = O.l1_dssim_loss(x, y)
    np.testing.assert_allclose(t0[:, 0], np.abs(x - y).reshape(2, -1).mean(1), rtol=1e-14)
    S = O.ssim_map(x, y)
    np.testing.assert_allclose(t1[:, 0], 1 - S.reshape(2, -1).mean(1), rtol=1e-14)
    np.testing.assert_allclose(t[:, 0], 0.8 * t0[:, 0] + 0.2 * t1[:, 0], rtol=1e-14)
    np.testing.assert_allclose(S, O.ssim_map(y, x), rtol=1e-14)
    assert S.max() <= 1.0 + 1e-12


@pytest.mark.parametrize("lam", [0.2, 1.0])
def test_loss_gradient_matches_central_differences(lam):
    rng = np.random.default_rng(7)
    x, y = rng.random((2, 3, 12, 15)), rng.random((2, 3, 12, 15))
    keep = np.abs(x - y) < 1e-3          # stay off the L1 kink
    x[keep] += 2e-3
    _, g = O.l1_dssim_loss(x, y, lam)
    eps = 1e-6
    for _ in range(24):
        idx = tuple(int(rng.integers(0, s)) for s in x.shape)
        xp, xm = x.copy(), x.copy()
        xp[idx] += eps
        xm[idx] -= eps
        v = idx[0]
        fd = (O.l1_dssim_loss(xp, y, lam)[0][v, 0] - O.l1_dssim_loss(xm, y, lam)[0][v, 0]) / (2 * eps)
        assert g[idx] == pytest.approx(fd, rel=1e-6, abs=1e-11), idx
        # another view's loss does not depend on this pixel
        o = 1 - v
        assert O.l1_dssim_loss(xp, y, lam)[0][o, 0] == O.l1_dssim_loss(x, y, lam)[0][o, 0]


def test_loss_l1_subgradient_is_zero_where_equal():
    rng = np.random.default_rng(8)
    x, y = rng.random((1, 3, 13, 13)), rng.random((1, 3, 13, 13))
    x[0, 1, 6, 6] = y[0, 1, 6, 6]
    _, g = O.l1_dssim_loss(x, y, 0.2)
    _, g1 = O.l1_dssim_loss(x, y, 1.0)
    assert g[0, 1, 6, 6] == pytest.approx(0.2 * g1[0, 1, 6, 6], rel=1e-13)


# ---------------------------------------------------------------- quantised SH state

def test_splitmix64_published_sequence():
    """The first three outputs of SplitMix64 seeded with 0, as published with
    the generator (and used to seed the xoshiro family)."""
    out = [int(v) for v in O.splitmix64(0, np.arange(3))]
    assert out == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_bf16_rounding_closed_forms():
    assert int(O.to_bf16(1.0)) == 0x3F80
    assert int(O.to_bf16(-2.0)) == 0xC000
    assert int(O.to_bf16(1 + 2 ** -8)) == 0x3F80          # tie -> even
    assert int(O.to_bf16(1 + 3 * 2 ** -8)) == 0x3F82      # tie -> even (up)
    assert int(O.to_bf16(1 + 2 ** -8 + 2 ** -20)) == 0x3F81  # above the tie
    assert int(O.to_bf16(0.0)) == 0 and int(O.to_bf16(-0.0)) == 0x8000
    rng = np.random.default_rng(1)
    x = rng.normal(0, 1, 10000) * 10.0 ** rng.integers(-20, 20, 10000)
    back = O.from_bf16(O.to_bf16(x))
    assert np.all(np.abs(back - x) <= np.abs(x) * 2.0 ** -8)


def _round_f32_exact(x) -> np.float32:
    """float32 nearest to the rational x (ties to even), by brute force over
    the candidates around float(x)."""
    from fractions import Fraction
    r0 = np.float32(float(x))
    cands = [r0, np.nextafter(r0, np.float32(np.inf)), np.nextafter(r0, np.float32(-np.inf))]
    best = min(abs(Fraction(float(c)) - x) for c in cands)
    ties = [c for c in cands if abs(Fraction(float(c)) - x) == best]
    if len(ties) > 1:
        ties = [c for c in ties if int(np.float32(c).view(np.uint32)) % 2 == 0]
    return np.float32(ties[0])


def test_fma_f32_is_the_correctly_rounded_fused_multiply_add():
    """Against exact rational arithmetic: random triples (with cancellation),
    and sums that sit on a float32 halfway point in float64 while the exact
    value does not (97 * 257 * 673 = 2^24 + 1, so 24929 * (673 * 2^-24) is
    the midpoint 1 + 2^-24 exactly)."""
    from fractions import Fraction
    rng = np.random.default_rng(11)
    a = rng.normal(0, 1, 400).astype(np.float32)
    b = rng.normal(0, 1, 400).astype(np.float32) * np.float32(2.0) ** rng.integers(-30, 30, 400)
    c = (-(a.astype(np.float64) * b) * (1 + rng.normal(0, 1e-6, 400))).astype(np.float32)
    c[::3] = rng.normal(0, 1, 134).astype(np.float32)
    mid_a, mid_b = np.float32(24929.0), np.float32(673.0 * 2.0 ** -24)
    tiny = np.float32(2.0 ** -80)
    a = np.concatenate([a, [mid_a] * 3])
    b = np.concatenate([b, [mid_b] * 3])
    c = np.concatenate([c, [tiny, np.float32(0), -tiny]])
    got = O.fma_f32(a, b, c)
    for k in range(len(a)):
        exact = Fraction(float(a[k])) * Fraction(float(b[k])) + Fraction(float(c[k]))
        assert got[k] == _round_f32_exact(exact), k
    assert got[-3] == np.float32(1 + 2.0 ** -23)      # just above the midpoint: up
    assert got[-2] == np.float32(1.0) and got[-1] == np.float32(1.0)  # tie to even; below


def test_float32_decoding_of_the_codes():
    """Code 0 decodes to the group's min exactly, a constant group to its
    value, and every value within float32 rounding of the float64 decoding."""
    rng = np.random.default_rng(12)
    n, K = 600, 4
    sh = rng.normal(0, 1, (n, K, 3)).astype(np.float32)
    sh[256:512, 1, 2] = -0.75
    for bits in (8, 16):
        codes, bounds = O.sh_quantize(sh, bits)
        x32 = O.dequantize_groups_f32(codes, bounds, n, bits)
        x64 = O.dequantize_groups(codes, bounds, n, bits)
        assert x32.dtype == np.float32 and x32.shape == (12, n)
        g = np.arange(n) // 256
        lo, hi = bounds[:, g, 0], bounds[:, g, 1]
        zero = codes[:, :n] == 0
        assert np.array_equal(x32[zero], lo[zero])
        assert np.all(x32[5, 256:512] == np.float32(-0.75))
        mag = np.maximum(np.abs(lo), np.abs(hi)).astype(np.float64)
        assert np.all(np.abs(x32 - x64) <= 2.0 ** -22 * mag + 1e-30)


def test_quantize_groups_structure_and_error_bound():
    """Groups are one coefficient of 256 consecutive Gaussians; the group's
    min and max are exact codes 0 and 2^b - 1; nearest rounding is off by at
    most half a step (plus float32 rounding of the scale)."""
    rng = np.random.default_rng(2)
    n, K = 700, 4                           # 3 groups, the last one ragged
    sh = rng.normal(0, 1, (n, K, 3)).astype(np.float32)
    sh[256:512, 2, 1] = 0.25                # one constant group
    for bits in (8, 16):
        codes, bounds = O.sh_quantize(sh, bits)
        qmax = (1 << bits) - 1
        assert codes.shape == (12, 768) and bounds.shape == (12, 3, 2)
        j = 2 * 3 + 1
        grp = sh[256:512, 2, 1]
        assert bounds[j, 1, 0] == grp.min() and bounds[j, 1, 1] == grp.max()
        assert np.all(codes[j, 256:512] == 0)
        x = O.dequantize_groups(codes, bounds, n, bits)
        assert np.all(x[j, 256:512] == 0.25)
        vals = sh.reshape(n, -1).T
        for jj in range(12):
            for g in range(3):
                a, b = 256 * g, min(256 * (g + 1), n)
                blk = vals[jj, a:b]
                assert bounds[jj, g, 0] == blk.min() and bounds[jj, g, 1] == blk.max()
                if blk.max() > blk.min():
                    assert codes[jj, a + int(np.argmin(blk))] == 0
                    assert codes[jj, a + int(np.argmax(blk))] == qmax
                    step = (float(blk.max()) - float(blk.min())) / qmax
                    err = np.abs(x[jj, a:b] - blk)
                    # half a step, plus the float32 rounding of t = (x - min) inv
                    # (a few ulps of t <= 2^b - 1)
                    assert err.max() <= step * (0.5 + 4 * qmax * 2.0 ** -24) + 1e-6 * abs(blk).max()
        assert np.all(codes[:, n:] == 0)    # padding untouched


def test_stochastic_rounding_is_unbiased_and_adjacent():
    rng = np.random.default_rng(3)
    x = np.zeros((1, 256), np.float32)
    x[0] = rng.uniform(-1, 1, 256).astype(np.float32)
    x[0, 0], x[0, 1] = -1.0, 1.0            # pin the range to exactly [-1, 1]
    qmax = 255
    step = 2.0 / qmax
    t = (x[0].astype(np.float64) + 1.0) / step
    acc = np.zeros(256)
    S = 400
    for s in range(S):
        c, b = O.quantize_groups(x, 256, 8, rounding=1, seed=1234, step=s + 1)
        q = c[0].astype(np.float64)
        assert np.all((q == np.floor(t + 1e-6)) | (q == np.floor(t + 1e-6) + 1)
                      | (q == np.ceil(t - 1e-6)))
        acc += -1.0 + q * step
    mean = acc / S
    # each draw's error is within one step with variance <= step^2 / 4
    assert np.all(np.abs(mean - x[0]) < 5 * step / 2 / np.sqrt(S))


def test_adam_on_quantised_state_against_plain_adam():
    """16-bit codes with nearest rounding: the re-encoded parameters equal the
    plain Adam step from the decoded values within half a step of the new
    groups, and the moments are the bfloat16 of the plain moments."""
    rng = np.random.default_rng(4)
    n, K = 600, 4
    sh = rng.normal(0, 0.5, (n, K, 3)).astype(np.float32)
    codes, bounds = O.sh_quantize(sh, 16)
    n_pad = codes.shape[1]
    m16 = O.to_bf16(rng.normal(0, 1e-3, (12, n_pad)))
    v16 = O.to_bf16(rng.uniform(0, 1e-6, (12, n_pad)))
    grad = rng.normal(0, 1e-3, (n, K, 3)).astype(np.float32)
    c2, b2, m2, v2, p_new = O.adam_sh_quant(codes, bounds, grad, m16, v16, n, 16, lr=2.5e-3,
                                            step=3)
    p0 = O.dequantize_groups(codes, bounds, n, 16)
    g = grad.reshape(n, -1).T.astype(np.float64)
    m0, v0 = O.from_bf16(m16[:, :n]), O.from_bf16(v16[:, :n])
    m1 = 0.9 * m0 + 0.1 * g
    v1 = 0.999 * v0 + 0.001 * g * g
    p1 = p0 - 2.5e-3 * (m1 / (1 - 0.9 ** 3)) / (np.sqrt(v1 / (1 - 0.999 ** 3)) + 1e-15)
    np.testing.assert_allclose(p_new, p1, rtol=1e-12, atol=1e-15)
    assert np.array_equal(m2[:, :n], O.to_bf16(m1)) and np.array_equal(v2[:, :n], O.to_bf16(v1))
    x = O.dequantize_groups(c2, b2, n, 16)
    step = (b2[:, :, 1] - b2[:, :, 0]).astype(np.float64) / 65535
    tol = step[:, np.arange(n) // 256] * (0.5 + 4 * 65535 * 2.0 ** -24) + 1e-7
    assert np.all(np.abs(x - p1) <= tol)
    # the moments' padding lanes are left alone
    assert np.array_equal(m2[:, n:], m16[:, n:])


def test_pure_l1_gradient_is_the_sign_over_n():
    rng = np.random.default_rng(9)
    x, y = rng.random((2, 3, 9, 11)), rng.random((2, 3, 9, 11))
    x[0, 0, 0, 0] = y[0, 0, 0, 0]
    _, g = O.l1_dssim_loss(x, y, lam=0.0)
    np.testing.assert_array_equal(g, np.sign(x - y) / (3 * 9 * 11))


def test_sixteen_bit_stochastic_rounding_lands_next_to_nearest():
    """With 16-bit codes a stochastic code is floor(t) or floor(t) + 1, so it
    is never more than one step from the nearest-rounded code."""
    rng = np.random.default_rng(10)
    x = rng.normal(0, 1, (6, 512)).astype(np.float32)
    cn, bn = O.quantize_groups(x, 500, 16, rounding=0)
    cs, bs = O.quantize_groups(x, 500, 16, rounding=1, seed=5, step=3)
    assert np.array_equal(bn, bs)
    d = np.abs(cn[:, :500].astype(np.int64) - cs[:, :500].astype(np.int64))
    assert d.max() <= 1 and 0.2 < (d > 0).mean() < 0.8
    assert np.all(cs[:, 500:] == 0)
