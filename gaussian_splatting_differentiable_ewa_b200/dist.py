"""Multi-GPU plumbing of the training step: one process per GPU, sharded by view.

Every rank holds the same Gaussians and renders its own view; the parameter
gradients of the step are summed across ranks (one all-reduce over the flat
gradient buffer, NCCL over NVLink on GPUs), after which every rank applies the
identical Adam step. Timings are reduced with MAX so a step costs what the
slowest rank took. Nothing here computes any part of the method.
"""

from __future__ import annotations

import math

import numpy as np


def orbit_view(scene, rank: int, world: int, radius: float = 8.0):
    """Camera of `rank` among `world` views spaced evenly on an orbit around the
    origin (same intrinsics as the scene's first camera)."""
    from . import scenes as S
    c0 = scene.cameras[0]
    a = 2.0 * math.pi * rank / world
    centre = (radius * math.sin(a), 0.0, -radius * math.cos(a))
    return S.Camera(viewmat=S.look_at(centre).astype(np.float32), fx=c0.fx, fy=c0.fy,
                    cx=c0.cx, cy=c0.cy, width=c0.width, height=c0.height,
                    campos=np.asarray(centre, np.float32))


def allreduce_grads(flat, group=None) -> None:
    """Sum the flat gradient buffer over all ranks, in place."""
    import torch.distributed as dist
    if dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(flat, op=dist.ReduceOp.SUM, group=group)


def max_over_ranks(value: float, device=None) -> float:
    """Largest `value` over all ranks (a step takes as long as its slowest rank)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_initialized() and dist.get_world_size() > 1):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
