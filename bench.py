"""Throughput of the STARFlow-V affine-autoregressive-flow hot path on B200.

Workload (default): the shallow f_S stack -- T = 3 AF blocks of alternating
direction (L->R, R->L, L->R), 4 layers each, d = 768, 12 heads, MLP 4x, bf16
tensor cores -- applied per frame to 21 latent frames x 390 tokens x 192
channels (a 5 s, 480p, 16 fps clip after a 16x/4x 48-channel VAE and 2x2
patches).  One step = flow_stack_forward(x) -> (z, logdet) followed by the
block-Jacobi flow_stack_inverse(z') of a fresh z' ~ N(0, 1) (B = 390, tau =
1e-3, max_iter = 390), both over the 8190 tokens.

Reported: value = Jacobi-inverse latent tokens/s (whole job, all ranks),
fwd_tokens_per_s, and the tensor-core roofline of the inverse graph from the
algorithmic flops of the updates actually run.  `--impl reference` times the
CPU float64 oracle on a bounded sample of the same workload instead.

Multi-GPU (torchrun): each rank inverts its own clip (independent frames, no
collective on the data path): weak scaling, max-over-ranks time.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synthetic as syn  # noqa: E402
from video_generation_b200 import flops as FL  # noqa: E402
from video_generation_b200 import replicas  # noqa: E402

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return PEAKS_FALLBACK, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms while running."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out = ""
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in getattr(self, "lines", []):
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def count_launches(w, iters_np):
    """Kernels of libaf launched by one step (forward stack + inverse stack)."""
    per_pass = 4 + 7 * w.shape.layers
    fwd = w.T * (1 + per_pass + 1)
    inv = 0
    nb = w.L // w.B
    for t in range(w.T):
        inv += 1                               # call init
        for b in range(nb):
            k = int(iters_np[t, :, b].max())
            inv += 1 + k * (per_pass + 1) + 1  # block init, updates (+ step), advance
    return fwd + inv


def run_oracle_sample(w, frames: int):
    """The CPU oracle on `frames` frames of the workload: forward stack and Jacobi inverse.

    Frames are batch entries for the per-frame shallow stack, and the first
    `frames` blocks of the sequence (a causal prefix) for the deep flow.
    Returns (tokens, fwd seconds, inverse seconds, threads used)."""
    from oracle import af_oracle as O
    blocks = [O.Block(w.shape, syn.make_weights(w.shape, block=t)) for t in range(w.T)]
    if w.L > w.B:
        x = syn.workload_latents(w, "x")[:1, :frames * w.B]
        z = syn.workload_latents(w, "z")[:1, :frames * w.B]
    else:
        x = syn.workload_latents(w, "x")[:frames]
        z = syn.workload_latents(w, "z")[:frames]
    t0 = time.perf_counter()
    O.stack_forward(blocks, w.dirs, x)
    t1 = time.perf_counter()
    O.stack_inverse(blocks, w.dirs, z, w.B, w.tau, w.max_iter, bool(w.warm_start))
    t2 = time.perf_counter()
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        threads = os.cpu_count()
    return x.shape[0] * x.shape[1], t1 - t0, t2 - t1, threads


def reference_arm(args, w, rank, world):
    """--impl reference: the float64 CPU oracle, as it stands, on host cores."""
    if rank != 0:
        return
    frames = args.ref_frames
    vals = []
    for i in range(args.warmup + args.steps):
        tok, tf, ti, threads = run_oracle_sample(w, frames)
        if i >= args.warmup:
            vals.append((tok, tf, ti))
    tok = sum(v[0] for v in vals)
    ti = sum(v[2] for v in vals)
    tf = sum(v[1] for v in vals)
    value = tok / ti
    line = {"metric": "jacobi_inverse_latent_tokens_per_s", "value": value, "unit": "tokens/s",
            "impl": "reference", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * (ti + tf) / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "fwd_tokens_per_s": tok / tf,
            "config": {"workload": w.name, "frames_per_step": frames, "tokens_per_step": tok // args.steps},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                             "sample": f"{frames} of {w.batch} frames per step, full T={w.T} stack "
                                       f"forward and Jacobi inverse"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", type=int, default=3, help="workload id (3 = f_S stack, the default)")
    ap.add_argument("--ref-frames", type=int, default=2, help="frames per oracle step (reference arm)")
    ap.add_argument("--cpu-frames", type=int, default=2, help="frames in the cpu_baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    w = syn.WORKLOADS[args.config]

    if args.impl == "reference":
        reference_arm(args, w, rank, world)
        return

    import torch
    import torch.distributed as dist
    from video_generation_b200 import flow

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    models = [flow.AFModel(w.shape, syn.make_weights(w.shape, block=t)) for t in range(w.T)]
    # each rank inverts its own clip: distinct seeds per rank
    x_np = syn.make_latents(w.batch, w.L, w.shape.C, replicas.rank_seed(syn.DATA_SEED + w.cid, rank))
    z_np = syn.make_latents(w.batch, w.L, w.shape.C, replicas.rank_seed(syn.DATA_SEED + w.cid + 100, rank))
    x = torch.from_numpy(x_np).to(dev)
    z_in = torch.from_numpy(z_np).to(dev)
    ws_f = models[0].workspace(w.batch, w.L, w.L, device=dev)
    ws_i = models[0].workspace(w.batch, w.L, w.B, device=dev)
    zf = torch.empty_like(x)
    ld = torch.empty(w.batch, dtype=torch.float32, device=dev)
    xi = torch.empty_like(x)
    iters = torch.zeros((w.T, w.batch, w.L // w.B), dtype=torch.int32, device=dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)   # > 126 MB L2
    st = torch.cuda.current_stream()

    def fwd():
        flow.flow_stack_forward(models, w.dirs, x, ws=ws_f, z=zf, logdet=ld)

    def inv():
        flow.flow_stack_inverse(models, w.dirs, z_in, w.B, w.tau, w.max_iter, w.warm_start, ws=ws_i, x=xi,
                                iters=iters)

    for _ in range(args.warmup):
        fwd()
        inv()
    torch.cuda.synchronize()
    err = models[0].device_error()
    if err:
        raise RuntimeError(f"device error {err} during warm-up")

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    iters_all = []
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        for i in range(args.steps):
            flush.zero_()                         # L2 flushed between timed steps
            ev[i][0].record(st)
            fwd()
            ev[i][1].record(st)
            inv()
            ev[i][2].record(st)
            iters_all.append(iters.clone())
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    t_fwd = sum(e[0].elapsed_time(e[1]) for e in ev) / 1e3
    t_inv = sum(e[1].elapsed_time(e[2]) for e in ev) / 1e3
    t = replicas.max_over_ranks(torch.tensor([t_fwd, t_inv], dtype=torch.float64, device=dev), dist)
    t_fwd, t_inv = float(t[0]), float(t[1])

    # algorithmic work from the iterations actually run
    it_np = [i.cpu().numpy() for i in iters_all]
    inv_flops = sum(FL.jacobi_flops(w.shape, a, w.L, w.B) for a in it_np)
    fwd_flops = args.steps * FL.forward_flops(w.shape, w.batch, w.L, w.T)
    tok = w.batch * w.L * args.steps * world
    peaks, peak_kind = load_peaks()
    inv_tf = inv_flops / t_inv / 1e12
    fwd_tf = fwd_flops / t_fwd / 1e12
    launches = sum(count_launches(w, a) for a in it_np)

    # end to end through the public API with host buffers: pinned z -> device,
    # inverse, x -> pinned host, every step inside the timed region
    z_host = torch.from_numpy(z_np).pin_memory()
    x_host = torch.empty_like(z_host).pin_memory()
    z_dev = torch.empty_like(z_in)
    e2e_ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e2e_ev[0].record(st)
    for _ in range(args.steps):
        z_dev.copy_(z_host, non_blocking=True)
        flow.flow_stack_inverse(models, w.dirs, z_dev, w.B, w.tau, w.max_iter, w.warm_start, ws=ws_i, x=xi,
                                iters=iters)
        x_host.copy_(xi, non_blocking=True)
    e2e_ev[1].record(st)
    torch.cuda.synchronize()
    t_e2e = replicas.max_over_ranks(
        torch.tensor([e2e_ev[0].elapsed_time(e2e_ev[1]) / 1e3], dtype=torch.float64, device=dev), dist)
    e2e_val = tok / float(t_e2e[0])
    bytes_step = w.batch * w.L * w.shape.C * 4

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        ctok, ctf, cti, threads = run_oracle_sample(w, args.cpu_frames)
        cpu = {"value": ctok / cti, "unit": "tokens/s", "cores": threads, "kind": "oracle",
               "sample": f"{args.cpu_frames} of {w.batch} frames, full T={w.T} stack Jacobi inverse "
                         f"(forward: {ctok / ctf:.1f} tokens/s)"}

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    peak = peaks["bf16_tflops"]
    line = {
        "metric": "jacobi_inverse_latent_tokens_per_s", "value": tok / t_inv, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * (t_fwd + t_inv) / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "frames": w.batch, "tokens_per_frame": w.L, "T": w.T,
                   "layers": w.shape.layers, "d_model": w.shape.d, "B": w.B, "tau": w.tau,
                   "max_iter": w.max_iter, "l2": "flushed between steps", "parallelism": f"replicas{world}"},
        "fwd_tokens_per_s": tok / t_fwd,
        "fwd_tflops": fwd_tf,
        "inverse_tflops": inv_tf,
        "mean_iters_per_block": float(np.mean([a.mean() for a in it_np])),
        "max_iters_per_block": int(max(a.max() for a in it_np)),
        "roofline": {"bound": "tensor", "achieved": inv_tf, "peak": peak, "unit": "TFLOP/s",
                     "frac": inv_tf / peak, "traffic": None,
                     "kernel": "flow_stack_inverse graph (tcgen05 GEMMs dominate)",
                     "peak_kind": f"bf16 dense burst, {peak_kind}",
                     "frac_of_sustained": inv_tf / peaks.get("bf16_tflops_sustained", peak)},
        "clocks": clk.summary(),
        "e2e": {"value": e2e_val, "unit": "tokens/s", "h2d_bytes_per_step": bytes_step,
                "d2h_bytes_per_step": bytes_step},
        "gpu_launches": launches,
    }
    if cpu is not None:
        line["cpu_baseline"] = cpu
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
