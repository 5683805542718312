"""Multi-GPU plumbing of the training step: one process per GPU, sharded by view.

Every rank holds the same Gaussians and renders its own view. The parameter
gradients of the step are summed across ranks with one reduce-scatter over the
flat gradient buffer (NCCL over NVLink on GPUs): each rank receives the summed
gradient of its own contiguous slice of the flat parameter buffer, runs Adam
on that slice only (its optimiser work and moments are 1/world of the whole),
and one all-gather hands every rank the updated parameters. Timings are
reduced with MAX so a step costs what the slowest rank took. Nothing here
computes any part of the method.
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


def flat_layout(sizes, pad: int):
    """Offsets of parameter groups [(name, numel), ...] laid end to end in one
    flat float buffer, each at a 16-byte aligned offset, and the buffer's
    length rounded up to a multiple of `pad` floats (at least `pad`)."""
    offsets, total = {}, 0
    for k, numel in sizes:
        offsets[k] = total
        total += (int(numel) + 3) // 4 * 4
    return offsets, max(-(-total // pad), 1) * pad


def shard_bounds(total: int, rank: int, world: int):
    """This rank's [lo, hi) of a flat buffer of `total` floats: `world` equal
    contiguous chunks; `total` must be a multiple of 4 * world so that every
    chunk starts 16-byte aligned."""
    if world < 1 or not 0 <= rank < world or total % (4 * world):
        raise ValueError("flat buffer of %d floats does not split in %d aligned chunks"
                         % (total, world))
    chunk = total // world
    return rank * chunk, (rank + 1) * chunk


def shard_slices(offsets: dict, sizes: dict, lo: int, hi: int):
    """The parts of each parameter group inside [lo, hi): (name, a, b) with
    lo <= a < b <= hi, group `name` occupying [offsets[name], offsets[name] +
    sizes[name]) of the flat buffer, in group order."""
    out = []
    for k, off in offsets.items():
        a, b = max(lo, off), min(hi, off + sizes[k])
        if a < b:
            out.append((k, a, b))
    return out


def allreduce_grads(flat, group=None) -> None:
    """Sum a buffer over all ranks, in place (the densify statistics before
    densify_and_prune; a whole gradient buffer for a replicated optimiser)."""
    import torch.distributed as dist
    if dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(flat, op=dist.ReduceOp.SUM, group=group)


def gather_for_densify(stats, flats, bounds=None, group=None) -> None:
    """Before densify_and_prune on several ranks: sum each statistics tensor
    in `stats` over the ranks (every rank then decides alike) and, when the
    optimiser is sharded (`bounds` = this rank's [lo, hi)), all-gather every
    rank's slice of each flat moment buffer in `flats`, in place."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size(group) < 2:
        return
    for t in stats:
        dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
    if bounds is not None:
        lo, hi = bounds
        for buf in flats:
            dist.all_gather_into_tensor(buf, buf[lo:hi].clone(), group=group)


def max_over_ranks(value: float, device=None) -> float:
    """Largest `value` over all ranks (a step takes as long as its slowest rank)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_initialized() and dist.get_world_size() > 1):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
