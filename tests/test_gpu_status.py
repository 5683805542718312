"""Device-side conditions reported through the status word (`-m gpu`).

Each bounded wait of the library gives up after a time limit, sets the timeout
bit and lets its kernel finish; gs_debug_stall makes one such wait run out on
purpose (a tile, an emission block or a radix partition waits for a copy or
a flag that nothing provides), with a short limit. Malformed list entries and ranges are clipped by
the rasteriser's own bounds checks and reported. Nothing here faults: every
access stays inside its buffer.
"""

import numpy as np
import pytest
import torch

from gaussian_splatting_differentiable_ewa_b200 import api
from gaussian_splatting_differentiable_ewa_b200 import scenes as S
from gaussian_splatting_differentiable_ewa_b200.pipeline import Splatter

pytestmark = pytest.mark.gpu

LIMIT_S = 0.05


@pytest.fixture(autouse=True)
def _no_stall_after():
    yield
    api.gs_debug_stall(api.GS_STALL_NONE)


def _splatter(mode=api.GS_SORT_PRESORT):
    sc = S.make_scene("fwd_100k_800", n=3000, width=200, height=152)
    sp = Splatter(sc, sort_mode=mode)
    sp.ensure_capacity()
    sp.forward()
    torch.cuda.synchronize()
    assert sp.status() == api.GS_OK
    return sc, sp


def _busy_tile(sp) -> int:
    r = sp.ranges.cpu().numpy()
    return int(np.argmax(r[:, 1] - r[:, 0]))


def _tile_mask(sp, tile):
    tx = (sp.W + 15) // 16
    ty, tx0 = divmod(tile, tx)
    m = np.zeros((sp.H, sp.W), bool)
    m[ty * 16:(ty + 1) * 16, tx0 * 16:(tx0 + 1) * 16] = True
    return m


def test_raster_fwd_wait_that_runs_out_is_reported():
    sc, sp = _splatter()
    want = sp.image.cpu().numpy()
    tile = _busy_tile(sp)
    api.gs_debug_stall(api.GS_STALL_RASTER_FWD, tile, LIMIT_S)
    sp.rasterize_fwd()
    torch.cuda.synchronize()
    api.gs_debug_stall(api.GS_STALL_NONE)
    assert sp.status() == api.GS_ERR_DEVICE_TIMEOUT
    got = sp.image.cpu().numpy()
    m = _tile_mask(sp, tile)
    # the stalled tile composited nothing (background, T = 1); the others are
    # untouched bit for bit
    assert np.array_equal(got[0][:, ~m], want[0][:, ~m])
    for ch in range(3):
        assert np.all(got[0, ch][m] == sc.background[ch])
    assert torch.all(sp.final_T[0][torch.as_tensor(m, device="cuda")] == 1.0)
    # and the next call, with the hook off, is normal again
    sp.rasterize_fwd()
    torch.cuda.synchronize()
    assert sp.status() == api.GS_OK
    assert np.array_equal(sp.image.cpu().numpy(), want)


def test_raster_bwd_wait_that_runs_out_is_reported():
    sc, sp = _splatter()
    c = sc.cameras[0]
    dL = torch.as_tensor(S.make_upstream_grad(1, c.height, c.width, seed=1)).cuda()
    sp.rasterize_bwd(dL)
    torch.cuda.synchronize()
    assert sp.status() == api.GS_OK
    full = sp.grad2d.clone()
    api.gs_debug_stall(api.GS_STALL_RASTER_BWD, _busy_tile(sp), LIMIT_S)
    sp.rasterize_bwd(dL)
    torch.cuda.synchronize()
    api.gs_debug_stall(api.GS_STALL_NONE)
    assert sp.status() == api.GS_ERR_DEVICE_TIMEOUT
    assert torch.isfinite(sp.grad2d).all()
    assert not torch.equal(sp.grad2d, full)   # the stalled tile's share is missing
    sp.rasterize_bwd(dL)
    torch.cuda.synchronize()
    assert sp.status() == api.GS_OK


def test_emission_lookback_wait_that_runs_out_is_reported():
    # full 64-bit keys: the emission scans its blocks with decoupled
    # look-back; block 1 never publishes, so block 2's wait runs out
    sc, sp = _splatter(api.GS_SORT_FULL64)
    ids = sp.ids.clone()
    ranges = sp.ranges.clone()
    api.gs_debug_stall(api.GS_STALL_EMIT_LOOKBACK, 1, LIMIT_S)
    sp.bin_sort()
    torch.cuda.synchronize()
    api.gs_debug_stall(api.GS_STALL_NONE)
    st = sp.status()
    assert st == api.GS_ERR_DEVICE_TIMEOUT, api.status_string(st)
    sp.bin_sort()
    torch.cuda.synchronize()
    assert sp.status() == api.GS_OK
    assert torch.equal(sp.ranges, ranges)
    n = int(sp.n_pairs.item())
    assert torch.equal(sp.ids[:n], ids[:n])


@pytest.mark.parametrize("mode", [api.GS_SORT_PRESORT, api.GS_SORT_FULL64])
def test_sort_lookback_wait_that_runs_out_is_reported(mode):
    # the 64-bit radix passes (depth keys in presort mode, pair keys in
    # full-64 mode) are single-sweep: partition 1 never publishes its counts,
    # so partition 2 waits for it in every pass until the limit
    sc = S.make_scene("fwd_100k_800", n=12000, width=200, height=152)
    sp = Splatter(sc, sort_mode=mode)
    sp.ensure_capacity()
    sp.project()
    sp.bin_sort()
    torch.cuda.synchronize()
    assert sp.status() == api.GS_OK
    keys = 12000 if mode == api.GS_SORT_PRESORT else int(sp.n_pairs.item())
    assert keys > 2 * 4096   # at least three partitions
    ids = sp.ids.clone()
    ranges = sp.ranges.clone()
    api.gs_debug_stall(api.GS_STALL_SORT_LOOKBACK, 1, LIMIT_S)
    sp.bin_sort()
    torch.cuda.synchronize()
    api.gs_debug_stall(api.GS_STALL_NONE)
    st = sp.status()
    assert st == api.GS_ERR_DEVICE_TIMEOUT, api.status_string(st)
    sp.bin_sort()
    torch.cuda.synchronize()
    assert sp.status() == api.GS_OK
    assert torch.equal(sp.ranges, ranges)
    n = int(sp.n_pairs.item())
    assert torch.equal(sp.ids[:n], ids[:n])


def test_clipped_ids_and_ranges_are_reported():
    sc, sp = _splatter()
    want = sp.image.cpu().numpy()
    tile = _busy_tile(sp)
    start, end = (int(x) for x in sp.ranges[tile].cpu())
    good = sp.ids[start].item()
    sp.ids[start] = sc.n + 7                      # names no Gaussian
    sp.rasterize_fwd()
    torch.cuda.synchronize()
    assert sp.status() == api.GS_ERR_OVERFLOW
    m = _tile_mask(sp, tile)
    got = sp.image.cpu().numpy()
    assert np.array_equal(got[0][:, ~m], want[0][:, ~m])
    assert np.isfinite(got).all()
    c = sc.cameras[0]
    dL = torch.as_tensor(S.make_upstream_grad(1, c.height, c.width, seed=1)).cuda()
    sp.rasterize_bwd(dL)
    torch.cuda.synchronize()
    assert sp.status() == api.GS_ERR_OVERFLOW
    assert torch.isfinite(sp.grad2d).all()
    sp.ids[start] = good
    # a range past the end of the ids buffer renders as empty
    saved = sp.ranges[tile].clone()
    sp.ranges[tile, 1] = sp.capacity + 100
    sp.rasterize_fwd()
    torch.cuda.synchronize()
    assert sp.status() == api.GS_ERR_OVERFLOW
    got = sp.image.cpu().numpy()
    assert np.array_equal(got[0][:, ~m], want[0][:, ~m])
    for ch in range(3):
        assert np.all(got[0, ch][m] == sc.background[ch])
    sp.ranges[tile] = saved
    sp.rasterize_fwd()
    torch.cuda.synchronize()
    assert sp.status() == api.GS_OK
    assert np.array_equal(sp.image.cpu().numpy(), want)
