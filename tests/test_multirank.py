"""Host-side logic of the multi-GPU step on CPU: `gloo` ranks.

Each rank gets a distinct orbit view, step times are reduced with MAX, a flat
buffer summed across ranks is the same everywhere, and the sharded optimiser
(reduce-scatter of the flat gradient, Adam on each rank's slice, all-gather of
the parameters) ends with every rank holding the replicated Adam step. The
Adam arithmetic here is the oracle's; the slicing and the collectives are the
library's own helpers. No GPU is involved."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from gaussian_splatting_differentiable_ewa_b200 import dist as gdist
        from gaussian_splatting_differentiable_ewa_b200 import scenes as S
        from oracle import oracle as O
        sc = S.make_scene("train_1m_1080p", n=64)
        cam = gdist.orbit_view(sc, rank, world)
        # rank-dependent "gradients" and a shared starting point
        rng = np.random.default_rng(100 + rank)
        flat = torch.tensor(rng.normal(size=1000), dtype=torch.float32)
        gdist.allreduce_grads(flat)
        p0 = np.linspace(-1, 1, 1000)
        p1, _, _ = O.adam(p0, flat.numpy(), np.zeros(1000), np.zeros(1000), 1e-3, 1)
        t = gdist.max_over_ranks(float(rank + 1) * 0.5)
        out[rank] = dict(campos=np.asarray(cam.campos).tolist(), grad=flat.numpy().tolist(),
                         p1=p1.tolist(), tmax=t)
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_gloo_ranks_share_summed_gradients_and_distinct_views():
    world = 2
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    expect = sum(np.random.default_rng(100 + r).normal(size=1000) for r in range(world))
    for r in range(world):
        np.testing.assert_allclose(res[r]["grad"], expect, rtol=1e-5, atol=1e-6)
        assert res[r]["tmax"] == 1.0
    assert res[0]["p1"] == res[1]["p1"]
    assert np.linalg.norm(np.subtract(res[0]["campos"], res[1]["campos"])) > 1.0
    for r in range(world):
        assert abs(np.linalg.norm(res[r]["campos"]) - 8.0) < 1e-5


def _shard_worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from gaussian_splatting_differentiable_ewa_b200 import dist as gdist
        from oracle import oracle as O
        n = 37
        sizes = [("means", 4 * n), ("log_scales", 4 * n), ("quats", 4 * n),
                 ("opacity_logit", n), ("sh", 48 * n)]
        lr = dict(means=1.6e-4, log_scales=5e-3, quats=1e-3, opacity_logit=5e-2, sh=2.5e-3)
        offs, total = gdist.flat_layout(sizes, 1024)
        p0 = torch.tensor(np.random.default_rng(7).normal(size=total), dtype=torch.float32)
        grad = torch.tensor(np.random.default_rng(200 + rank).normal(size=total),
                            dtype=torch.float32)
        param, m, v = p0.clone(), torch.zeros(total), torch.zeros(total)
        lo, hi = gdist.shard_bounds(total, rank, world)
        shard = torch.empty(hi - lo)
        dist.reduce_scatter_tensor(shard, grad)          # the summed gradient of the slice
        for k, a, b in gdist.shard_slices(offs, dict(sizes), lo, hi):
            pn, mn, vn = O.adam(param[a:b].numpy(), shard[a - lo:b - lo].numpy(),
                                m[a:b].numpy(), v[a:b].numpy(), lr[k], 1)
            param[a:b] = torch.tensor(pn, dtype=torch.float32)
            m[a:b] = torch.tensor(mn, dtype=torch.float32)
        dist.all_gather_into_tensor(param, param[lo:hi].clone())
        out[rank] = dict(param=param.numpy().tolist(), offs=offs, total=total, lo=lo, hi=hi)
    finally:
        dist.barrier()
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_sharded_adam_equals_the_replicated_step(world):
    """Reduce-scatter of the flat gradient, Adam on each rank's slice only,
    all-gather of the parameters: every rank ends with the parameters of one
    Adam step on the summed gradient over the whole buffer (group by group,
    padding untouched), and the slices tile the buffer."""
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_shard_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    from gaussian_splatting_differentiable_ewa_b200 import dist as gdist
    from oracle import oracle as O
    total, offs = res[0]["total"], res[0]["offs"]
    assert [(res[r]["lo"], res[r]["hi"]) for r in range(world)] == \
        [(r * total // world, (r + 1) * total // world) for r in range(world)]
    assert all(res[r]["lo"] % 4 == 0 for r in range(world))
    n = 37
    sizes = dict(means=4 * n, log_scales=4 * n, quats=4 * n, opacity_logit=n, sh=48 * n)
    lr = dict(means=1.6e-4, log_scales=5e-3, quats=1e-3, opacity_logit=5e-2, sh=2.5e-3)
    p0 = np.random.default_rng(7).normal(size=total).astype(np.float32)
    g = sum(np.random.default_rng(200 + r).normal(size=total).astype(np.float32)
            for r in range(world))
    want = p0.copy()
    for k, off in offs.items():
        sl = slice(off, off + sizes[k])
        pn, _, _ = O.adam(p0[sl], g[sl], np.zeros(sizes[k]), np.zeros(sizes[k]), lr[k], 1)
        want[sl] = pn.astype(np.float32)
    for r in range(world):
        got = np.asarray(res[r]["param"], np.float32)
        np.testing.assert_allclose(got, want, rtol=0, atol=2e-7)
    assert np.array_equal(np.asarray(res[0]["param"]), np.asarray(res[world - 1]["param"]))
    # padding between groups and after the last one keeps its starting value
    ends = sorted((off + sizes[k], off + (sizes[k] + 3) // 4 * 4) for k, off in offs.items())
    for a, b in ends + [(max(o + (sizes[k] + 3) // 4 * 4 for k, o in offs.items()), total)]:
        assert np.array_equal(np.asarray(res[0]["param"], np.float32)[a:b], p0[a:b])
    assert gdist.shard_slices(offs, sizes, 0, total) == [
        (k, o, o + sizes[k]) for k, o in offs.items()]


def _densify_worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from gaussian_splatting_differentiable_ewa_b200 import dist as gdist
        total = 1024
        lo, hi = gdist.shard_bounds(total, rank, world)
        accum = torch.tensor(np.arange(10, dtype=np.float32) * (rank + 1))
        denom = torch.tensor(np.full(10, rank + 1, dtype=np.int32))
        # each rank's moments are current on its own slice only
        m = torch.full((total,), -1.0)
        m[lo:hi] = torch.arange(lo, hi, dtype=torch.float32)
        gdist.gather_for_densify((accum, denom), (m,), (lo, hi))
        out[rank] = dict(accum=accum.tolist(), denom=denom.tolist(), m=m.tolist())
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_densify_inputs_are_summed_and_gathered_across_ranks():
    world = 4
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_densify_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    tri = world * (world + 1) // 2
    for r in range(world):
        assert res[r]["accum"] == (np.arange(10) * tri).tolist()
        assert res[r]["denom"] == [tri] * 10
        assert res[r]["m"] == np.arange(1024, dtype=np.float32).tolist()


def _splatter_worker(rank, world, port, out):
    """The Splatter's own sharded optimiser and densify gathering on CPU
    tensors: only the Adam arithmetic (a GPU kernel) is replaced, by the
    oracle's, so the slicing, collectives and buffer handling are the
    product code."""
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from gaussian_splatting_differentiable_ewa_b200 import api
        from gaussian_splatting_differentiable_ewa_b200 import pipeline
        from gaussian_splatting_differentiable_ewa_b200 import scenes as S
        from oracle import oracle as O

        def cpu_adam(groups, beta1, beta2, eps, step, stream=None):
            for p, g, m, v, lr in groups:
                pn, mn, vn = O.adam(p.numpy(), g.numpy(), m.numpy(), v.numpy(), lr, step,
                                    beta1, beta2, eps)
                p.copy_(torch.from_numpy(pn.astype(np.float32)))
                m.copy_(torch.from_numpy(mn.astype(np.float32)))
                v.copy_(torch.from_numpy(vn.astype(np.float32)))

        api.gs_adam_step = cpu_adam
        sp = pipeline.Splatter(S.make_scene("fwd_1k_128", n=300), device="cpu")
        sp.shard_optimizer(rank, world)
        rng = np.random.default_rng(50 + rank)
        for _ in range(2):
            sp.grad_flat.copy_(torch.from_numpy(
                rng.normal(size=sp.flat_total).astype(np.float32)))
            sp.adam_step()
        sp.accum_abs.fill_(float(rank + 1))
        sp.denom.fill_(rank + 1)
        sp._gather_for_densify()
        out[rank] = dict(param=sp.param_flat.numpy().tolist(), m=sp.m_flat.numpy().tolist(),
                         accum=sp.accum_abs.numpy().tolist(), denom=sp.denom.numpy().tolist(),
                         offs=sp.flat_offsets, sizes=sp.flat_sizes, total=sp.flat_total,
                         lr=sp.lr)
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_splatter_sharded_optimizer_on_gloo_ranks():
    world = 2
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_splatter_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    from gaussian_splatting_differentiable_ewa_b200 import scenes as S
    from oracle import oracle as O
    r0 = res[0]
    total, offs, sizes, lr = r0["total"], r0["offs"], r0["sizes"], r0["lr"]
    sc = S.make_scene("fwd_1k_128", n=300)
    start = {"means": sc.means, "log_scales": sc.log_scales, "quats": sc.quats,
             "opacity_logit": sc.opacity_logit, "sh": sc.sh}
    p = np.zeros(total, np.float32)
    for k, off in offs.items():
        p[off:off + sizes[k]] = np.asarray(start[k], np.float32).reshape(-1)
    m = np.zeros(total, np.float32)
    v = np.zeros(total, np.float32)
    rngs = [np.random.default_rng(50 + r) for r in range(world)]
    for step in (1, 2):
        g = sum(rg.normal(size=total).astype(np.float32) for rg in rngs)
        for k, off in offs.items():
            sl = slice(off, off + sizes[k])
            pn, mn, vn = O.adam(p[sl], g[sl], m[sl], v[sl], lr[k], step, 0.9, 0.999, 1e-15)
            p[sl], m[sl], v[sl] = pn.astype(np.float32), mn.astype(np.float32), vn.astype(np.float32)
    for r in range(world):
        np.testing.assert_allclose(np.asarray(res[r]["param"], np.float32), p, rtol=0, atol=1e-6)
        # after the densify gathering every rank holds every slice of the moments
        np.testing.assert_allclose(np.asarray(res[r]["m"], np.float32), m, rtol=0, atol=1e-6)
        assert res[r]["accum"] == [3.0] * 300 and res[r]["denom"] == [3] * 300
    assert res[0]["param"] == res[1]["param"]
