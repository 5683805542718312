"""Host-side checks of the C-ABI library that need no GPU: it loads, exports
every function include/gs.h declares, and rejects bad arguments before any
CUDA call."""

import ctypes
import os
import re

import numpy as np
import pytest

from gaussian_splatting_differentiable_ewa_b200 import api
from gaussian_splatting_differentiable_ewa_b200 import scenes as S

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    text = open(os.path.join(ROOT, "include", "gs.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gs_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    L = api.lib()
    names = _declared()
    assert len(names) >= 10
    for name in names:
        assert hasattr(L, name), name
    assert {s[0] for s in api.SIGNATURES} == set(names)


def test_abi_version_and_status_strings():
    assert api.gs_abi_version() == 4
    for s in range(7):
        assert api.status_string(s) not in ("", "unknown status")


def test_workspace_size_validates_and_grows():
    sc = S.make_scene("train_1m_1080p", n=1000)
    cams = api.cameras(sc.cameras)
    a = api.gs_workspace_size(1000, cams, 1, 10_000, api.GS_SORT_FULL64)
    b = api.gs_workspace_size(1000, cams, 1, 1_000_000, api.GS_SORT_FULL64)
    c = api.gs_workspace_size(1000, cams, 1, 1_000_000, api.GS_SORT_PRESORT)
    assert 0 < a < b and c > 0
    assert b - a >= (1_000_000 - 10_000) * 20  # two 8-byte key buffers + 4-byte ids
    assert api.gs_workspace_size(-1, cams, 1, 10, 0) == 0
    assert api.gs_workspace_size(10, cams, 0, 10, 0) == 0
    assert api.gs_workspace_size(10, cams, 1, -5, 0) == 0
    assert api.gs_workspace_size(10, cams, 1, 10, 7) == 0
    # views of different sizes are rejected
    two = api.cameras([sc.cameras[0], S.make_scene("fwd_1k_128", n=1).cameras[0]])
    assert api.gs_workspace_size(10, two, 2, 10, 0) == 0


def test_bad_arguments_are_rejected_before_any_cuda_call():
    L = api.lib()
    sc = S.make_scene("fwd_1k_128", n=10)
    cams = api.cameras(sc.cameras)
    p = api.GsParams(None, None, None, None, None, 0, 0, 10)
    out = api.GsProjected(None, None)
    # an aligned address that is never dereferenced: each call returns first
    ws = ctypes.c_void_p(4096)
    assert L.gs_project(ctypes.byref(p), cams, 1, ctypes.byref(out), ws, None) == \
        api.GS_ERR_INVALID_ARG
    p.sh_degree = 4
    assert L.gs_project(ctypes.byref(p), cams, 1, ctypes.byref(out), ws, None) == \
        api.GS_ERR_INVALID_ARG
    p.n = 1 << 31
    p.sh_degree = 0
    assert L.gs_project(ctypes.byref(p), cams, 1, ctypes.byref(out), ws, None) == \
        api.GS_ERR_OVERFLOW
    assert L.gs_project(ctypes.byref(p), cams, 0, ctypes.byref(out), ws, None) == \
        api.GS_ERR_INVALID_ARG
    # the status word is required, and must be 256-byte aligned
    assert L.gs_project(ctypes.byref(p), cams, 1, ctypes.byref(out), None, None) == \
        api.GS_ERR_INVALID_ARG
    assert L.gs_project(ctypes.byref(p), cams, 1, ctypes.byref(out), ctypes.c_void_p(4100),
                        None) == api.GS_ERR_INVALID_ARG
    bn = api.GsBinned(None, None, None, 10)
    bg = (ctypes.c_float * 3)()
    assert L.gs_rasterize_fwd(ctypes.byref(out), ctypes.byref(bn), cams, 1, 10, bg, None, None,
                              None, None, None, None) == api.GS_ERR_INVALID_ARG
    assert L.gs_rasterize_bwd(ctypes.byref(p), ctypes.byref(out), ctypes.byref(bn), cams, 1, bg,
                              None, None, None, None, None, None, None, None) == \
        api.GS_ERR_INVALID_ARG
    b = api.GsBinned(None, None, None, 10)
    assert L.gs_bin_sort(ctypes.byref(out), cams, 1, 10, 0, ctypes.byref(b), None, 0, None) == \
        api.GS_ERR_INVALID_ARG
    grp = (api.GsAdamGroup * 1)()
    assert L.gs_adam_step(grp, 1, 0.9, 0.999, 1e-15, 0, None) == api.GS_ERR_INVALID_ARG
    assert L.gs_adam_step(grp, 9, 0.9, 0.999, 1e-15, 1, None) == api.GS_ERR_INVALID_ARG
    assert L.gs_adam_step(grp, 1, 1.5, 0.999, 1e-15, 1, None) == api.GS_ERR_INVALID_ARG
    assert L.gs_densify_stats(None, None, 0, 10, None, None, None, None) == api.GS_ERR_INVALID_ARG
    assert L.gs_get_status(None, None) == api.GS_ERR_INVALID_ARG


def test_debug_stall_arguments():
    assert api.lib().gs_debug_stall(api.GS_STALL_RASTER_FWD, -1, 0.0) == api.GS_ERR_INVALID_ARG
    assert api.lib().gs_debug_stall(9, 0, 0.0) == api.GS_ERR_INVALID_ARG
    assert api.lib().gs_debug_stall(api.GS_STALL_SORT_LOOKBACK + 1, 0, 0.0) == api.GS_ERR_INVALID_ARG
    api.gs_debug_stall(api.GS_STALL_SORT_LOOKBACK, 1, 0.05)
    assert api.lib().gs_debug_stall(api.GS_STALL_NONE, 0, -1.0) == api.GS_ERR_INVALID_ARG
    assert api.lib().gs_debug_stall(api.GS_STALL_NONE, 0, 61.0) == api.GS_ERR_INVALID_ARG
    api.gs_debug_stall(api.GS_STALL_RASTER_BWD, 3, 0.05)
    api.gs_debug_stall(api.GS_STALL_NONE)


def test_loss_and_quant_arguments_are_rejected_before_any_cuda_call():
    L = api.lib()
    assert api.gs_l1_dssim_workspace_size(3) == 3 * 16 + 16
    assert api.gs_l1_dssim_workspace_size(-1) == 0
    p = ctypes.c_void_p(16)  # never dereferenced: validation fails first
    bad = [(p, p, 1, 0, 8, 0.2, p, None, p, 64),        # empty image
           (p, p, 1, 8, 8, 1.5, p, None, p, 64),        # lambda outside [0, 1]
           (None, p, 1, 8, 8, 0.2, p, None, p, 64),     # no image
           (p, p, 1, 8, 8, 0.2, p, None, p, 8),         # workspace too small
           (p, p, 21846, 8, 8, 0.2, p, None, p, 1 << 20)]
    for a in bad:
        assert L.gs_l1_dssim(*a, None) == api.GS_ERR_INVALID_ARG, a
    assert L.gs_l1_dssim(None, None, 0, 0, 0, 0.2, None, None, None, 0, None) == api.GS_OK
    q = api.GsShQuant(16, 16, 100, 12, 12)              # 12-bit codes
    assert L.gs_sh_quantize(p, ctypes.byref(q), None) == api.GS_ERR_INVALID_ARG
    q = api.GsShQuant(16, 16, 100, 10, 8)               # k3 not 3 (K) for K in 1, 4, 9, 16
    assert L.gs_sh_dequantize(ctypes.byref(q), p, None) == api.GS_ERR_INVALID_ARG
    q = api.GsShQuant(16, 16, 100, 12, 8)
    assert L.gs_adam_step_sh_quant(ctypes.byref(q), p, p, p, 1e-3, 0.9, 0.999, 1e-15, 1, 2, 0,
                                   None) == api.GS_ERR_INVALID_ARG   # rounding 2
    assert L.gs_adam_step_sh_quant(ctypes.byref(q), p, p, p, 1e-3, 1.0, 0.999, 1e-15, 1, 0, 0,
                                   None) == api.GS_ERR_INVALID_ARG   # beta1 1
    q = api.GsShQuant(None, None, 0, 12, 8)
    assert L.gs_sh_quantize(None, ctypes.byref(q), None) == api.GS_OK
    # packed state: moments travel in the blocks, so separate moment arrays are refused
    qp = api.GsShQuant(16, 16, 100, 12, 16, api.GS_QUANT_PACKED, 0)
    assert L.gs_adam_step_sh_quant(ctypes.byref(qp), p, p, p, 1e-3, 0.9, 0.999, 1e-15, 1, 0, 0,
                                   None) == api.GS_ERR_INVALID_ARG
    qx = api.GsShQuant(16, 16, 100, 12, 16, 7, 0)        # no such layout
    assert L.gs_sh_quantize(p, ctypes.byref(qx), None) == api.GS_ERR_INVALID_ARG
    # densify of the codes: mismatched widths or layouts, a count above 2 n,
    # planar moments missing, a workspace too small
    a = api.GsShQuant(16, 16, 100, 12, 8, api.GS_QUANT_PLANAR, 0)
    b16 = api.GsShQuant(16, 16, 150, 12, 16, api.GS_QUANT_PLANAR, 0)
    big = api.GsShQuant(16, 16, 201, 12, 8, api.GS_QUANT_PLANAR, 0)
    ok = api.GsShQuant(16, 16, 150, 12, 8, api.GS_QUANT_PLANAR, 0)
    ws = ctypes.c_void_p(4096)
    nws = api.gs_densify_sh_quant_workspace_size(100, 150)
    assert nws > 0 and api.gs_densify_sh_quant_workspace_size(-1, 0) == 0
    f = L.gs_densify_sh_quant
    assert f(ctypes.byref(a), p, p, p, ctypes.byref(b16), p, p, ws, nws, None) == \
        api.GS_ERR_INVALID_ARG
    assert f(ctypes.byref(a), p, p, p, ctypes.byref(big), p, p, ws, nws, None) == \
        api.GS_ERR_INVALID_ARG
    assert f(ctypes.byref(a), None, p, p, ctypes.byref(ok), p, p, ws, nws, None) == \
        api.GS_ERR_INVALID_ARG
    assert f(ctypes.byref(a), p, p, p, ctypes.byref(ok), p, p, ws, 8, None) == \
        api.GS_ERR_INVALID_ARG
    # the fused step tail: quantised SH, step 0, beta1 = 1, half the statistics
    cams = api.cameras(S.make_scene("fwd_1k_128", n=10).cameras)
    pr = api.GsParams(16, 16, 16, 16, 16, 0, 0, 10, None)
    g = api.GsGrads(16, 16, 16, 16, 16)
    lr5 = (ctypes.c_float * 5)(1e-3, 1e-3, 1e-3, 1e-3, 1e-3)
    fa = L.gs_project_bwd_adam
    assert fa(ctypes.byref(pr), cams, 1, p, p, ctypes.byref(g), ctypes.byref(g), lr5, 0.9,
              0.999, 1e-15, 0, None, None, None, None) == api.GS_ERR_INVALID_ARG
    assert fa(ctypes.byref(pr), cams, 1, p, p, ctypes.byref(g), ctypes.byref(g), lr5, 1.0,
              0.999, 1e-15, 1, None, None, None, None) == api.GS_ERR_INVALID_ARG
    assert fa(ctypes.byref(pr), cams, 1, p, p, ctypes.byref(g), ctypes.byref(g), lr5, 0.9,
              0.999, 1e-15, 1, p, None, None, None) == api.GS_ERR_INVALID_ARG
    qs = api.GsShQuant(16, 16, 10, 3, 8, api.GS_QUANT_PLANAR, 0)
    prq = api.GsParams(16, 16, 16, 16, None, 0, 0, 10,
                       ctypes.cast(ctypes.pointer(qs), ctypes.c_void_p))
    assert fa(ctypes.byref(prq), cams, 1, p, p, ctypes.byref(g), ctypes.byref(g), lr5, 0.9,
              0.999, 1e-15, 1, None, None, None, None) == api.GS_ERR_INVALID_ARG


def test_densify_thresholds_convert_to_the_raw_parameter_units():
    """The cut-offs travel as a log-scale and a logit: comparing raw
    parameters against them decides as comparing activated values against the
    given thresholds (exp and the logistic function are increasing)."""
    dp = api.densify_params(0.0002, 0.05, 0.005, 1.0, 1.6)
    assert dp.grad_threshold == np.float32(0.0002)
    assert dp.log_scale_split == np.float32(np.log(0.05))
    assert dp.logit_min_opacity == np.float32(np.log(0.005 / 0.995))
    assert dp.log_max_scale == 0.0 and dp.log_split_shrink == np.float32(np.log(1.6))
    rng = np.random.default_rng(3)
    ls = rng.uniform(-8, 2, 2000).astype(np.float32)
    lg = rng.uniform(-9, 9, 2000).astype(np.float32)
    s, o = np.exp(ls.astype(np.float64)), 1 / (1 + np.exp(-lg.astype(np.float64)))
    far = (np.abs(s - 0.05) > 1e-5) & (np.abs(o - 0.005) > 1e-6)
    assert np.array_equal((ls > np.float32(dp.log_scale_split))[far], (s > 0.05)[far])
    assert np.array_equal((lg < np.float32(dp.logit_min_opacity))[far], (o < 0.005)[far])
    L = api.lib()
    out = api.GsDensifyParams()
    for bad in ((2e-4, 0.0, 0.005, 1.0, 1.6), (2e-4, 0.05, 0.0, 1.0, 1.6),
                (2e-4, 0.05, 1.0, 1.0, 1.6), (2e-4, 0.05, 0.005, -1.0, 1.6),
                (2e-4, 0.05, 0.005, 1.0, 0.0), (2e-4, 0.05, float("nan"), 1.0, 1.6)):
        assert L.gs_densify_params_from_cutoffs(*bad, ctypes.byref(out)) == api.GS_ERR_INVALID_ARG
    assert L.gs_densify_params_from_cutoffs(2e-4, 0.05, 0.005, 1.0, 1.6, None) == \
        api.GS_ERR_INVALID_ARG
    assert 0 < api.gs_densify_workspace_size(1000) < api.gs_densify_workspace_size(10 ** 6)
    assert api.gs_densify_workspace_size(-1) == 0


def test_sort_plan_follows_the_grid_and_mode():
    """gs_bin_sort_plan (host only) names the emission path the workspace is
    laid out for: tile placement up to 16384 tiles per view while the
    (tiles + 1)^2 difference array fits, emission by column up to 256
    columns, by tile id beyond; radix pass counts of 8-bit digits; placement
    blocks of about four per SM below a million Gaussians."""
    def plan(W, H, n, views, mode):
        cam = S.make_scene("fwd_1k_128").cameras[0]
        cam.width, cam.height, cam.cx, cam.cy = W, H, W / 2, H / 2
        return api.gs_bin_sort_plan(n, api.cameras([cam] * views), views, mode)
    p = plan(1920, 1080, 1_000_000, 1, api.GS_SORT_PRESORT)
    assert (p.path, p.presort_passes, p.pair_passes) == (api.GS_PATH_TILES, 4, 0)
    assert (p.gaussians_per_block, p.blocks_per_view) == (768, 1303)
    p = plan(1920, 1080, 3_000_000, 1, api.GS_SORT_PRESORT)       # larger blocks past 2M
    assert (p.gaussians_per_block, p.blocks_per_view) == (4096, 733)
    p = plan(3840, 2160, 10_000_000, 1, api.GS_SORT_PRESORT)      # 4K: 240 x 135 tiles
    assert (p.path, p.pair_passes) == (api.GS_PATH_COLUMNS, 1)
    assert p.pair_single_sweep == 0                                 # 32-bit row keys
    assert p.ranges_from_counts == 1                                # 241 x 136 ints fit
    assert p.pair_key_bytes == 1                                    # 135 rows: the row alone
    p = plan(3840, 2160, 1000, 2, api.GS_SORT_PRESORT)            # 270 rows: two bytes
    assert (p.pair_key_bytes, p.pair_passes, p.ranges_from_counts) == (2, 2, 1)
    assert ctypes.sizeof(api.GsSortPlan) == 40
    p = plan(128, 128, 1000, 1, api.GS_SORT_PRESORT)               # small scene: 32 per block
    assert (p.path, p.gaussians_per_block, p.blocks_per_view) == (api.GS_PATH_TILES, 32, 32)
    p = plan(800, 800, 100_000, 1, api.GS_SORT_PRESORT)
    assert (p.gaussians_per_block, p.blocks_per_view) == (160, 625)
    p = plan(4096, 2576, 1000, 1, api.GS_SORT_PRESORT)            # 256 x 161 tiles
    assert (p.path, p.pair_passes) == (api.GS_PATH_COLUMNS, 1)
    assert p.ranges_from_counts == 0                                # 257 x 162 ints do not
    assert p.pair_key_bytes == 4                                    # row << 8 | column
    p = plan(8192, 1296, 1000, 1, api.GS_SORT_PRESORT)            # 512 x 81 tiles
    assert (p.path, p.pair_passes) == (api.GS_PATH_TILE_ID, 2)
    assert p.pair_single_sweep == 0
    p = plan(8192, 1296, 1000, 2, api.GS_SORT_PRESORT)            # 82944 tiles: 17 bits, 6 + 6 + 5
    assert (p.pair_passes, p.pair_single_sweep) == (3, 0)       # 82944 tiles: 17 bits
    p = plan(1920, 1080, 1000, 8, api.GS_SORT_PRESORT)            # 3 view bits in the key
    assert p.presort_passes == 5
    p = plan(1920, 1080, 1000, 1, api.GS_SORT_FULL64)             # 13 tile bits + 32
    assert (p.path, p.presort_passes, p.pair_passes) == (api.GS_PATH_TILE_ID, 0, 6)
    assert p.pair_single_sweep == 1 and p.ranges_from_counts == 1
    p = plan(8192, 1296, 1000, 1, api.GS_SORT_FULL64)             # 513 x 82 counters: too many
    assert p.ranges_from_counts == 0
    with pytest.raises(api.GsError):
        plan(1920, 1080, -1, 1, api.GS_SORT_PRESORT)


def test_bench_work_model_uses_the_library_plan():
    import types
    import bench
    cams = api.cameras(S.make_scene("train_1m_1080p", n=10).cameras)
    sp = types.SimpleNamespace(n=1_000_000, V=1, W=1920, H=1080, cams=cams)
    plan = bench.sort_plan(sp, "presort")
    assert plan == dict(path="tiles", pre=4, pair=0, bpv=1303, tiles=8160, pair_sweep=False,
                        count_ranges=False, key_bytes=0)
    # project; depth keys, digit counts, 4 single-sweep passes, count, scan, base,
    # place; raster fwd, raster bwd, project bwd, densify stats, Adam
    assert bench.launches_per_step(sp, "presort") == 1 + (1 + 1 + 4 + 4) + 5
    assert bench.sort_plan(sp, "full64")["pair"] == 6
    # emit, digit counts, 6 passes, tile histogram, ranges from it
    assert bench.sort_plan(sp, "full64")["count_ranges"]
    assert bench.launches_per_step(sp, "full64") == 1 + (1 + 1 + 6 + 2) + 5
    # the fused tail: raster fwd, raster bwd, projection backward + statistics + Adam
    assert bench.launches_per_step(sp, "presort", fused=True) == 1 + (1 + 1 + 4 + 4) + 3
    # a 4K view: depth keys, digit counts, 4 passes, column count, tile histogram,
    # ranges from it, column scan, emission, one row pass (count, scan, scatter)
    sp4 = types.SimpleNamespace(n=10_000_000, V=1, W=3840, H=2160,
                                cams=api.cameras(S.make_scene("train_10m_4k", n=10).cameras))
    assert bench.sort_plan(sp4, "presort")["count_ranges"]
    assert bench.launches_per_step(sp4, "presort", fused=True) == \
        1 + (1 + 1 + 4 + 1 + 2 + 2 + 3) + 3
    # blend kernels: bytes on the examined entries, FP32 operations on the
    # evaluations and the contributing pixels
    sp.K = 16
    P = 1920 * 1080
    w = bench.algorithmic_work(sp, 26_000_000, "presort", 1.0e8, 2_000_000, 3.0e8)
    assert w["gs_rasterize_fwd"]["bytes"] == 2_000_000 * 44 + P * 20
    assert w["gs_rasterize_bwd"]["bytes"] == 2_000_000 * 84 + P * 12
    assert w["gs_rasterize_fwd"]["ops"] == 3.0e8 * bench.OPS_EVAL + 1.0e8 * bench.OPS_FWD_CONTRIB
    assert w["gs_rasterize_bwd"]["ops"] == 3.0e8 * bench.OPS_EVAL + 1.0e8 * bench.OPS_BWD_CONTRIB
    assert w["gs_project_bwd_adam"]["bytes"] == 1_000_000 * (6 * 236 + 36 + 24)
    # without the examined count every pair is charged (the scope table's ceiling)
    w0 = bench.algorithmic_work(sp, 26_000_000, "presort", 1.0e8)
    assert w0["gs_rasterize_fwd"]["bytes"] == 26_000_000 * 44 + P * 20
    # full-64 mode, ranges from the tile counts: per pair 12 B emitted, 24 B a pass,
    # 8 B of digit counts, the last pass's 8 B of keys not written; per Gaussian
    # and view 24 B read for the keys and 16 B for the tile histogram
    wf = bench.algorithmic_work(sp, 26_000_000, "full64", 0.0)
    assert wf["gs_bin_sort"]["bytes"] == 26_000_000 * (12 + 6 * 24 + 8 - 8) + 1_000_000 * 40
    # the 4K column path: one-byte row keys emitted with the ids, one rows pass
    # (read and written), the last write without keys; per Gaussian the depth
    # keys' 4 passes and the rectangles read for the histogram
    sp4.K = 16
    w4 = bench.algorithmic_work(sp4, 849_000_000, "presort", 0.0)
    assert w4["gs_bin_sort"]["bytes"] == (849_000_000 * ((1 + 4) + 2 * (1 + 4) - 1)
                                          + 10_000_000 * (16 + 8 + 4 * 24 + 12 + 16))
    assert bench.alu_peak_gops(1965.0) == pytest.approx(148 * 128 * 1.965)
