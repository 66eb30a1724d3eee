"""The multi-rank (replica) path on CPU: two gloo ranks, each running its own
clip through the CPU oracle as a stand-in device, then the same bookkeeping
bench.py uses on GPUs (distinct seeds, MAX over ranks, whole-job throughput)."""
import os
import socket
import time

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import synthetic as syn
from video_generation_b200 import replicas

SHAPE = syn.ModelShape(C=8, d=16, heads=2, layers=1, mlp_ratio=2, frame_len=8, max_frames=1, dtype="fp32")


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    from oracle import af_oracle as O
    blk = O.Block(SHAPE, syn.make_weights(SHAPE))
    x = syn.make_latents(2, 8, 8, replicas.rank_seed(syn.DATA_SEED, rank))
    t0 = time.perf_counter()
    z, ld = O.af_forward(blk, x, O.L2R)
    dt = time.perf_counter() - t0 + 0.01 * rank          # ranks differ in time
    t = torch.tensor([dt], dtype=torch.float64)
    replicas.max_over_ranks(t, dist)
    zs = [torch.zeros(2 * 8 * 8, dtype=torch.float64) for _ in range(world)]
    dist.all_gather(zs, torch.from_numpy(z.ravel()))
    dist.barrier()
    dist.destroy_process_group()
    out.put((rank, dt, float(t[0]), [a.numpy() for a in zs]))


def test_two_replicas_independent_work_and_max_time():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    tmax = res[0][2]
    assert all(r[2] == tmax for r in res)                 # every rank sees the same max
    assert tmax >= max(r[1] for r in res) - 1e-12
    z0, z1 = res[0][3]
    assert not np.allclose(z0, z1)                        # distinct clips per rank
    assert replicas.job_throughput(16, world, tmax) == 32 / tmax


def test_seeds_distinct_per_rank():
    assert len({replicas.rank_seed(5678, r) for r in range(8)}) == 8
