"""Frames of one clip across ranks (video_generation_b200.shard), on CPU with
the gloo backend: contiguous frame ranges, each rank running the shallow
stack on its own frames, one all-gather assembling the clip.  The per-frame
computation here is the CPU oracle (no GPU on this machine); the
partition and the exchange are the code bench.py runs over NCCL.  The
assembled result must equal the whole clip computed in one process, bit for
bit, for even and uneven partitions and for a rank with no frames."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import synthetic as syn
from video_generation_b200 import shard

SHAPE = syn.ModelShape(C=8, d=16, heads=2, layers=1, mlp_ratio=2, frame_len=8, max_frames=1, dtype="fp32")
DIRS = (0, 1, 0)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _blocks():
    from oracle import af_oracle as O
    return [O.Block(SHAPE, syn.make_weights(SHAPE, block=t, perturb=True, head_std=0.1)) for t in range(3)]


def _clip(n_frames):
    return syn.make_latents(n_frames, SHAPE.frame_len, SHAPE.C, 77)


def _per_frames(frames):
    """The shallow stack, forward and inverse, on a slab of frames (frames = batch)."""
    from oracle import af_oracle as O
    blocks = _blocks()
    x = frames.numpy()
    z, ld = O.stack_forward(blocks, DIRS, x)
    xi, it = O.stack_inverse(blocks, DIRS, z, SHAPE.frame_len, 1e-8, SHAPE.frame_len, False)
    return (torch.from_numpy(z), torch.from_numpy(ld), torch.from_numpy(xi), torch.from_numpy(it.transpose(1, 0, 2).copy()))


def _rank(rank, world, port, n_frames, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        clip = torch.from_numpy(_clip(n_frames))
        res = shard.run_sharded(lambda lo, hi: clip[lo:hi], _per_frames, n_frames, dist)
        t = torch.tensor([0.01 * (rank + 1)], dtype=torch.float64)
        shard.max_over_ranks(t, dist)
        dist.barrier()
        out.put((rank, [r.numpy() for r in res], float(t[0])))
    finally:
        dist.destroy_process_group()


def _run(world, n_frames):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, n_frames, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=180) for _ in range(world)), key=lambda r: r[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return res


def test_frame_ranges_are_contiguous_balanced_and_cover_the_clip():
    assert shard.frame_ranges(5, 2) == [(0, 3), (3, 5)]
    assert [e - s for s, e in shard.frame_ranges(21, 8)] == [3, 3, 3, 3, 3, 2, 2, 2]
    assert shard.frame_ranges(1, 2) == [(0, 1), (1, 1)]
    for n in range(0, 30):
        for w in range(1, 9):
            r = shard.frame_ranges(n, w)
            assert r[0][0] == 0 and r[-1][1] == n
            assert all(r[i][1] == r[i + 1][0] for i in range(w - 1))
            sizes = [e - s for s, e in r]
            assert max(sizes) - min(sizes) <= 1


@pytest.mark.parametrize("n_frames", [4, 5, 1])
def test_two_ranks_assemble_the_clip_bitwise(n_frames):
    world = 2
    res = _run(world, n_frames)
    whole = [r.numpy() for r in _per_frames(torch.from_numpy(_clip(n_frames)))]
    for rank, got, tmax in res:
        assert tmax == 0.02                                  # every rank sees the slowest rank's time
        for g, w in zip(got, whole):
            assert g.shape == w.shape
            np.testing.assert_array_equal(g, w)
