"""Host-side logic of the multi-GPU step on CPU: two `gloo` ranks.

Each rank gets a distinct orbit view, the flat gradient buffer is summed across
ranks (so every rank applies the same Adam update), and step times are reduced
with MAX. No GPU is involved."""

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
