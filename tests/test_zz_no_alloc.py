"""gs_bin_sort_noalloc: binning and depth sort for callers that cannot allocate
device memory (its scratch is a fixed array inside the library). Its tile lists
must be identical, bit for bit, to those of gs_bin_sort with a caller-allocated
workspace, call after call, since the array keeps the previous call's contents.
This file is collected last so that a failure here comes after every other
test has run."""

import numpy as np
import pytest
import torch

from gaussian_splatting_differentiable_ewa_b200 import api
from gaussian_splatting_differentiable_ewa_b200 import scenes as S
from gaussian_splatting_differentiable_ewa_b200.pipeline import Splatter

pytestmark = pytest.mark.gpu

CASES = [
    ("fwd_1k_128", dict(), api.GS_SORT_FULL64),
    ("fwd_1k_128", dict(), api.GS_SORT_PRESORT),
    ("fwd_100k_800", dict(n=20000, width=792, height=600), api.GS_SORT_FULL64),
    ("fwd_100k_800", dict(), api.GS_SORT_PRESORT),
    ("train_6m_8x1080p", dict(n=4000, n_views=2), api.GS_SORT_PRESORT),
]


def _outputs(sp):
    ids = torch.full_like(sp.ids, -1)
    ranges = torch.full_like(sp.ranges, -1)
    n_pairs = torch.full_like(sp.n_pairs, -1)
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    return ids, ranges, n_pairs, status, api.binned(ids, ranges, n_pairs, sp.capacity)


@pytest.mark.parametrize("name,kw,mode", CASES)
def test_noalloc_matches_workspace_path_twice(name, kw, mode):
    sc = S.make_scene(name, **kw)
    sp = Splatter(sc, sort_mode=mode)
    sp.ensure_capacity()
    torch.cuda.synchronize()
    assert sp.status() == api.GS_OK
    need = api.gs_workspace_size(sp.n, sp.cams, sp.V, sp.capacity, mode)
    assert need <= api.GS_NOALLOC_SCRATCH_BYTES
    n_ref = int(sp.n_pairs.item())
    ids_ref = sp.ids[:n_ref].cpu().numpy()
    ranges_ref = sp.ranges.cpu().numpy()
    for _ in range(2):
        ids, ranges, n_pairs, status, out = _outputs(sp)
        api.gs_bin_sort_noalloc(sp.c_proj, sp.cams, sp.V, sp.n, mode, out, status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert int(n_pairs.item()) == n_ref
        assert np.array_equal(ranges.cpu().numpy(), ranges_ref)
        assert np.array_equal(ids[:n_ref].cpu().numpy(), ids_ref)


def test_noalloc_rejects_requests_beyond_its_scratch():
    sc = S.make_scene("train_1m_1080p", n=1000)
    sp = Splatter(sc, sort_mode=api.GS_SORT_FULL64, pair_capacity=4_000_000)
    assert api.gs_workspace_size(sp.n, sp.cams, 1, 4_000_000, 0) > api.GS_NOALLOC_SCRATCH_BYTES
    ids, ranges, n_pairs, status, out = _outputs(sp)
    with pytest.raises(api.GsError) as e:
        api.gs_bin_sort_noalloc(sp.c_proj, sp.cams, 1, sp.n, api.GS_SORT_FULL64, out, status)
    assert e.value.status == api.GS_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert int(n_pairs.item()) == -1 and int(status.item()) == -1  # nothing was enqueued
