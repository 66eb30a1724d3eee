"""Frames of a clip across GPUs: one process per GPU, contiguous frame ranges,
one all-gather of the results.

The shallow flow f_S acts on each latent frame on its own ("STARFlow-V ...
paper notes", key design 1: f_S works inside a frame), so the frames of a
clip are independent units of the forward pass and of the block-Jacobi
inverse alike: rank r takes a contiguous range of frames, runs the stack on
them with no communication, and the clip is assembled afterwards by one
all-gather of the frames (NCCL over NVLink / NVSwitch on GPUs, gloo on CPU)
and of their per-frame log-determinants.  Ranges differ in length by at most
one frame; the all-gather pads every rank's slab to the longest range.

This module is the partition and the exchange only; what a rank computes on
its frames is passed in by the caller (the CUDA library on GPUs).
"""
from __future__ import annotations

from typing import Callable, List, Tuple

import torch


def frame_ranges(n_frames: int, world: int) -> List[Tuple[int, int]]:
    """Contiguous [start, end) frame ranges of ranks 0..world-1, covering
    0..n_frames-1 in order; the first n_frames % world ranks take one extra."""
    if n_frames < 0 or world < 1:
        raise ValueError("need n_frames >= 0 and world >= 1")
    base, extra = divmod(n_frames, world)
    out, start = [], 0
    for r in range(world):
        n = base + (1 if r < extra else 0)
        out.append((start, start + n))
        start += n
    return out


def gather_frames(local: torch.Tensor, n_frames: int, dist, group=None) -> torch.Tensor:
    """All-gather every rank's contiguous slab of frames (dim 0) into the whole
    clip, on every rank.  `local` holds this rank's frame_ranges() slab; slabs
    are padded to the longest range for the collective and trimmed after."""
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    ranges = frame_ranges(n_frames, world)
    lo, hi = ranges[rank]
    if local.shape[0] != hi - lo:
        raise ValueError(f"rank {rank} holds {local.shape[0]} frames, its range is {hi - lo}")
    width = max(e - s for s, e in ranges)
    slab = local.new_zeros((width,) + tuple(local.shape[1:]))
    slab[: hi - lo] = local
    slabs = [torch.empty_like(slab) for _ in range(world)]
    dist.all_gather(slabs, slab, group=group)
    return torch.cat([slabs[r][: e - s] for r, (s, e) in enumerate(ranges)], dim=0)


def run_sharded(clip_frames: Callable[[int, int], torch.Tensor], per_frames: Callable[[torch.Tensor], Tuple],
                n_frames: int, dist, group=None) -> Tuple[torch.Tensor, ...]:
    """This rank's frames through `per_frames`, then every output gathered.

    clip_frames(lo, hi) returns frames lo..hi-1 of the clip (dim 0 = frame);
    per_frames(frames) returns a tuple of tensors whose dim 0 is the frame."""
    world = dist.get_world_size(group) if dist is not None and dist.is_initialized() else 1
    rank = dist.get_rank(group) if world > 1 else 0
    ranges = frame_ranges(n_frames, world)
    lo, hi = ranges[rank]
    outs = tuple(per_frames(clip_frames(lo, hi))) if hi > lo else None
    if world == 1:
        return outs
    if any(e == s for s, e in ranges):
        # a rank without frames computes nothing; rank 0 (which has frames when
        # any rank does) tells it the outputs' shapes and types for the gather
        meta = [[(tuple(o.shape[1:]), o.dtype) for o in outs] if rank == 0 else None]
        dist.broadcast_object_list(meta, src=0, group=group)
        if outs is None:
            dev = clip_frames(0, 0).device
            outs = tuple(torch.empty((0,) + shp, dtype=dt, device=dev) for shp, dt in meta[0])
    return tuple(gather_frames(o, n_frames, dist, group) for o in outs)


def max_over_ranks(t: torch.Tensor, dist=None) -> torch.Tensor:
    """Element-wise max of `t` over all ranks (in place); identity without a group."""
    if dist is not None and dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t


def job_throughput(units_total: float, seconds: float) -> float:
    """Whole-job units per second: every rank's units over the slowest rank's time."""
    return units_total / seconds
