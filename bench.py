"""Throughput of the STARFlow-V affine-autoregressive-flow hot path on B200.

Workload (default, config 3): the shallow f_S stack -- T = 3 AF blocks of
alternating direction (L->R, R->L, L->R), 4 layers each, d = 768, 12 heads,
MLP 4x, bf16 tensor cores -- applied per frame to latent frames of 390 tokens
x 192 channels (480p, 16 fps, 16x/4x 48-channel VAE, 2x2 patches); 21 frames
(a 5 s clip) per GPU.  One step = flow_stack_forward(x) -> (z, logdet) then
the block-Jacobi flow_stack_inverse(z') of a fresh z' ~ N(0, 1) (B = 390, tau
= 1e-3, max_iter = 390) over the frames.

Several GPUs (`--gpus N`, one process per GPU; without torchrun the script
relaunches itself under torch.distributed.run): the job is a clip of N x 21
frames; rank r takes a contiguous range of frames (video_generation_b200.shard),
runs the stack on them and the clip is assembled by one NCCL all-gather of z,
logdet and x per step, inside the timed region.  Per-GPU work is fixed (weak
scaling); time is the max over ranks.  The deep-flow configs (4, 5: one video
is sequential across blocks) run one video per rank with no exchange.

Reported: value = Jacobi-inverse latent tokens/s of the whole job;
fwd_tokens_per_s; the tensor-core roofline of the inverse graph from the
algorithmic flops of the updates actually run; e2e through pinned host
buffers (upload of the next step's z and download of the previous step's x
overlap the current step on a copy stream); with one GPU also configs 2, 4
and 5 (`extra`) and the CPU oracle baselines.  `--impl reference` times the
CPU float64 oracle on a bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import json
import os
import socket
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synthetic as syn  # noqa: E402
from video_generation_b200 import flops as FL  # noqa: E402
from video_generation_b200 import shard  # noqa: E402

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# DRAM bytes (read + write) of one launch of the config-3 Jacobi inverse graph:
# twice the ncu dram__bytes of one forward graph (the inverse runs the same
# pass over the same 8190 rows 6 times, the forward 3 times), from the launch
# list in profiles/launch_list_fs_stack_T3_21frames_forward.md.
C3_INVERSE_DRAM_BYTES = 2 * 2.356e9
SMS = 148


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


# ----------------------------------------------------------------------------- bookkeeping

def attention_may_split(w) -> bool:
    """Whether libaf's attention launches its split-merge kernel for this workload
    (some pass has too few query tiles to fill the GPU and keys beyond 512)."""
    return w.shape.dtype == "bf16" and w.shape.heads * w.batch < 2 * SMS and w.L > 512


def count_launches(w, iters_np, batch):
    """Kernels of libaf launched by one step (forward stack + inverse stack)."""
    comb = w.shape.layers if attention_may_split(w) else 0
    per_pass = 4 + 7 * w.shape.layers + comb
    fwd = w.T * (1 + per_pass + 1)
    inv = 1                                    # block table
    nb = w.L // w.B
    for t in range(w.T):
        inv += 1                               # call init
        for b in range(nb):
            k = int(iters_np[t, :, b].max())
            inv += 1 + k * (per_pass + 1) + 1  # block init, updates (+ step), advance
    return fwd + inv


def frame_sharded(w) -> bool:
    """Workloads whose sequences are single frames (the shallow stack): frames shard across ranks."""
    return w.L == w.shape.frame_len


# ----------------------------------------------------------------------------- CPU oracle legs

def oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        return os.cpu_count()


def run_oracle_sample(w, frames: int, single_thread: bool = False):
    """The CPU oracle on `frames` frames of the workload: forward stack and Jacobi inverse.

    Frames are batch entries for per-frame workloads, and the first `frames`
    blocks of the sequence (a causal prefix) for the deep flow.
    Returns (tokens, fwd seconds, inverse seconds, threads used, inverse flops)."""
    from oracle import af_oracle as O
    blocks = [O.Block(w.shape, syn.make_weights(w.shape, block=t)) for t in range(w.T)]
    if frame_sharded(w):
        x = syn.clip_frames(w, "x", 0, frames)
        z = syn.clip_frames(w, "z", 0, frames)
    else:
        x = syn.workload_latents(w, "x")[:1, :frames * w.B]
        z = syn.workload_latents(w, "z")[:1, :frames * w.B]

    def go():
        t0 = time.perf_counter()
        O.stack_forward(blocks, w.dirs, x)
        t1 = time.perf_counter()
        _, it = O.stack_inverse(blocks, w.dirs, z, w.B, w.tau, w.max_iter, bool(w.warm_start))
        t2 = time.perf_counter()
        return t1 - t0, t2 - t1, it

    if single_thread:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            tf, ti, it = go()
        threads = 1
    else:
        tf, ti, it = go()
        threads = oracle_threads()
    inv_flops = FL.jacobi_flops(w.shape, it, x.shape[1], w.B)
    return x.shape[0] * x.shape[1], tf, ti, threads, inv_flops


def reference_arm(args, w, rank, world):
    """--impl reference: the float64 CPU oracle, as it stands, on host cores."""
    if rank != 0:
        return
    frames = args.ref_frames
    vals = []
    threads = 1
    for i in range(args.warmup + args.steps):
        tok, tf, ti, threads, _ = run_oracle_sample(w, frames)
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


def cpu_baselines(w, args, gpu_inv_flops_per_step, gpu_tokens_per_step):
    """The oracle on bounded samples: all-core and single-thread rates; for the
    deep flow also the time of the full inverse, extrapolated (labelled as
    such) from the oracle's measured flop rate on the first frame."""
    tok, tf, ti, threads, inv_fl = run_oracle_sample(w, args.cpu_frames)
    out = {"value": tok / ti, "unit": "tokens/s", "cores": threads, "kind": "oracle",
           "sample": f"{args.cpu_frames} frame(s) of the workload, full T={w.T} stack Jacobi inverse "
                     f"(forward: {tok / tf:.1f} tokens/s)"}
    tok1, tf1, ti1, _, _ = run_oracle_sample(w, 1, single_thread=True)
    out["single_thread_value"] = tok1 / ti1
    out["single_thread_sample"] = "1 frame, one BLAS thread"
    if not frame_sharded(w):
        rate = inv_fl / ti                                  # oracle flop/s on the causal prefix
        t_full = gpu_inv_flops_per_step / rate
        out["extrapolated_full_inverse_s"] = t_full
        out["extrapolated_tokens_per_s"] = gpu_tokens_per_step / t_full
        out["extrapolation"] = ("full-sequence inverse time = its algorithmic flops (from the GPU run's "
                                "iteration counts) / the oracle's measured flop rate on the first frame")
    return out


# ----------------------------------------------------------------------------- one workload on the GPU

def measure(w, args, rank, world, dist, dev, with_e2e=True):
    """Times `args.steps` steps (forward + inverse) of workload w on this rank,
    max over ranks.  Returns a dict of results."""
    import torch
    from video_generation_b200 import flow

    models = [flow.AFModel(w.shape, syn.make_weights(w.shape, block=t)) for t in range(w.T)]
    sharded = frame_sharded(w) and world > 1
    if frame_sharded(w):
        n_frames = w.batch * world                      # weak scaling: w.batch frames per GPU
        lo, hi = shard.frame_ranges(n_frames, world)[rank]
        x_np = syn.clip_frames(w, "x", lo, hi)
        z_np = syn.clip_frames(w, "z", lo, hi)
    else:                                               # one video per rank
        n_frames = world
        x_np = syn.make_latents(1, w.L, w.shape.C, syn.DATA_SEED + w.cid + 1000 * rank)
        z_np = syn.make_latents(1, w.L, w.shape.C, syn.DATA_SEED + w.cid + 100 + 1000 * rank)
    batch = x_np.shape[0]
    x = torch.from_numpy(x_np).to(dev)
    z_in = torch.from_numpy(z_np).to(dev)
    ws_f = models[0].workspace(batch, w.L, w.L, device=dev)
    ws_i = models[0].workspace(batch, w.L, w.B, device=dev)
    zf = torch.empty_like(x)
    ld = torch.empty(batch, dtype=torch.float32, device=dev)
    xi = torch.empty_like(x)
    iters = torch.zeros((w.T, batch, w.L // w.B), dtype=torch.int32, device=dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)   # > 126 MB L2
    st = torch.cuda.current_stream()

    def fwd():
        flow.flow_stack_forward(models, w.dirs, x, ws=ws_f, z=zf, logdet=ld)
        if sharded:
            shard.gather_frames(zf, n_frames, dist)
            shard.gather_frames(ld, n_frames, dist)

    def inv(zsrc=z_in, xdst=xi):
        flow.flow_stack_inverse(models, w.dirs, zsrc, w.B, w.tau, w.max_iter, w.warm_start, ws=ws_i, x=xdst,
                                iters=iters)
        return shard.gather_frames(xdst, n_frames, dist) if sharded else xdst

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
    with ClockSampler(dev.index) as clk:
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
    t = shard.max_over_ranks(torch.tensor([t_fwd, t_inv], dtype=torch.float64, device=dev), dist)
    t_fwd, t_inv = float(t[0]), float(t[1])
    it_np = [a.cpu().numpy() for a in iters_all]
    r = {"t_fwd": t_fwd, "t_inv": t_inv, "it_np": it_np, "batch": batch, "clk": clk.summary(),
         "tokens_per_step_rank": batch * w.L,
         "inv_flops_rank": sum(FL.jacobi_flops(w.shape, a, w.L, w.B) for a in it_np),
         "fwd_flops_rank": args.steps * FL.forward_flops(w.shape, batch, w.L, w.T),
         "launches": sum(count_launches(w, a, batch) for a in it_np) // args.steps}

    if with_e2e:
        # end to end through the public API with host buffers: every step uploads
        # its z from pinned memory and downloads its x.  The upload of step i+1
        # (its own copy stream) and the download of step i-1 (another) overlap
        # step i; device buffers are double-buffered.
        cp_up = torch.cuda.Stream(device=dev)
        cp_dn = torch.cuda.Stream(device=dev)
        z_host = torch.from_numpy(z_np).pin_memory()
        n_out = batch * world if sharded else batch
        x_host = torch.empty((n_out, w.L, w.shape.C), dtype=torch.float32).pin_memory()
        z_dev = [torch.empty_like(z_in) for _ in range(2)]
        x_dev = [torch.empty_like(z_in) for _ in range(2)]
        up = [torch.cuda.Event() for _ in range(2)]
        done = [torch.cuda.Event() for _ in range(2)]
        down = [torch.cuda.Event() for _ in range(2)]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        t0.record(st)
        cp_up.wait_stream(st)
        cp_dn.wait_stream(st)
        with torch.cuda.stream(cp_up):
            z_dev[0].copy_(z_host, non_blocking=True)
            up[0].record(cp_up)
        for i in range(args.steps):
            j = i % 2
            if i + 1 < args.steps:
                with torch.cuda.stream(cp_up):
                    if i >= 1:
                        cp_up.wait_event(done[1 - j])    # z_dev[1-j] read by step i-1's inverse
                    z_dev[1 - j].copy_(z_host, non_blocking=True)
                    up[1 - j].record(cp_up)
            st.wait_event(up[j])
            if i >= 2:
                st.wait_event(down[j])                   # x_dev[j] downloaded by step i-2
            out = inv(z_dev[j], x_dev[j])
            done[j].record(st)
            with torch.cuda.stream(cp_dn):
                cp_dn.wait_event(done[j])
                x_host.copy_(out, non_blocking=True)
                down[j].record(cp_dn)
        st.wait_stream(cp_up)
        st.wait_stream(cp_dn)
        t1.record(st)
        torch.cuda.synchronize()
        te = shard.max_over_ranks(torch.tensor([t0.elapsed_time(t1) / 1e3], dtype=torch.float64, device=dev), dist)
        r["t_e2e"] = float(te[0])
        r["h2d"] = z_host.numel() * 4
        r["d2h"] = x_host.numel() * 4
    for m in models:
        m.close()
    return r


def time_calls(fn, warmup, steps, st):
    """Mean device time (s) of `steps` calls of fn after `warmup` calls, CUDA events on `st`."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(steps):
        fn()
    e1.record(st)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / 1e3 / steps


def deep_flow_extras(args, dev, peaks):
    """The deep flow (config 4) in the shapes the pages discuss: a sweep of the
    Jacobi block size and the asymmetric schedule (small blocks for the first
    frame, large after it; the pages' key findings), pipelined deep -> shallow
    decoding of the 5 s clip against its parts (key design 3), and the
    flow-score-matching denoiser over the clip (key design 2)."""
    import torch
    from video_generation_b200 import flow
    st = torch.cuda.current_stream()
    w4, w3 = syn.WORKLOADS[4], syn.WORKLOADS[3]
    deep = flow.AFModel(w4.shape, syn.make_weights(w4.shape))
    z = torch.from_numpy(syn.workload_latents(w4, "z")).to(dev)
    out = {}
    # block-size sweep (uniform blocks) and the asymmetric schedule
    sweep = {}
    F = w4.shape.frame_len
    schedules = {f"B{b}": [b] * (w4.L // b) for b in (130, 195, 390, 819, 1170, 1638)}   # divisors of 8190
    schedules["first_frame_65_then_780"] = [65] * (F // 65) + [780] * ((w4.L - F) // 780)
    for name, sizes in schedules.items():
        assert sum(sizes) == w4.L
        ws = deep.workspace(1, w4.L, max(sizes), device=dev)
        x = torch.empty_like(z)
        it = torch.zeros((1, len(sizes)), dtype=torch.int32, device=dev)
        run = lambda: flow.af_inverse_jacobi_schedule(deep, z, 0, sizes, w4.tau, w4.max_iter, True, ws=ws, x=x, iters=it)
        t = time_calls(run, 3, 2, st)
        itn = it.cpu().numpy()
        fl = 0.0
        starts = np.concatenate([[0], np.cumsum(sizes)])
        for b, k in enumerate(itn[0]):
            f1 = FL.pass_flops(w4.shape.d, w4.shape.C, w4.shape.layers, w4.shape.mlp_ratio, sizes[b],
                               FL.causal_pairs(int(starts[b]), sizes[b]))
            fl += float(k) * f1 + (f1 if b + 1 < len(sizes) else 0.0)
        sweep[name] = {"ms": 1e3 * t, "tokens_per_s": w4.L / t, "tflops": fl / t / 1e12,
                       "mean_iters": float(itn.mean()), "blocks": len(sizes)}
        del ws
    out["fd_5s_block_size_sweep"] = sweep
    # pipelined decoding: f_D^{-1}, and f_S^{-1} of each group of frames as the
    # deep flow finishes it, on a second stream; against the two run one after
    # the other (the deep inverse, then the shallow stack of all 21 frames as
    # one batch)
    shallow = [flow.AFModel(w3.shape, syn.make_weights(w3.shape, block=t)) for t in range(w3.T)]
    nf = w4.L // F
    ws_d = deep.workspace(1, w4.L, w4.B, device=dev)
    u = torch.empty_like(z)
    deep_only = lambda: flow.af_inverse_jacobi(deep, z, 0, w4.B, w4.tau, w4.max_iter, True, ws=ws_d, x=u)
    t_deep = time_calls(deep_only, 3, 2, st)
    frames = u.view(nf, F, w4.shape.C)
    ws_b = shallow[0].workspace(nf, F, F, device=dev)
    xs = torch.empty_like(frames)
    shallow_batched = lambda: flow.flow_stack_inverse(shallow, w3.dirs, frames, F, w3.tau, w3.max_iter, False,
                                                      ws=ws_b, x=xs)
    t_sh = time_calls(shallow_batched, 3, 3, st)
    xp = torch.empty_like(z)
    by_group = {}
    # the deep flow's stream at the highest priority, so that its kernels'
    # CTAs are placed ahead of the shallow calls' when SMs free up
    # (torch maps a priority past the device's range to its end)
    s_deep = torch.cuda.Stream(device=dev, priority=-100)
    s_sh = torch.cuda.Stream(device=dev, priority=0)
    for g in (1, 3, 7, nf):
        ws_s = flow.pipeline_workspace(shallow, 1, F, g, device=dev)
        pipe = lambda: flow.flow_pipeline_inverse(deep, shallow, w3.dirs, z, w4.B, w4.tau, w4.max_iter, w3.max_iter,
                                                  True, group=g, ws_deep=ws_d, ws_shallow=ws_s, x=xp,
                                                  stream=s_deep, stream_shallow=s_sh)
        by_group[f"group{g}"] = 1e3 * time_calls(pipe, 2, 2, s_deep)
        del ws_s
    best = min(by_group, key=by_group.get)
    out["pipelined_decode_5s"] = {"ms": by_group[best], "best": best, "ms_by_frames_per_shallow_call": by_group,
                                  "deep_alone_ms": 1e3 * t_deep, "shallow_21_frames_batched_ms": 1e3 * t_sh,
                                  "sequential_sum_ms": 1e3 * (t_deep + t_sh),
                                  "tokens_per_s": w4.L / (by_group[best] / 1e3),
                                  "streams": "deep at the highest priority, shallow at the lowest"}
    for m in shallow:
        m.close()
    deep.close()
    # the denoiser over the 5 s clip
    den = flow.AFModel(syn.DENOISER, syn.make_denoiser_weights(syn.DENOISER), denoiser=True)
    L = 21 * syn.DENOISER.frame_len
    xn = torch.from_numpy(syn.make_latents(1, L, syn.DENOISER.C, 83)).to(dev)
    ws_n = den.workspace(1, L, device=dev)
    xo = torch.empty_like(xn)
    t_den = time_calls(lambda: flow.af_denoise(den, xn, 0.1, ws=ws_n, x=xo), 3, 5, st)
    fl = FL.denoiser_flops(syn.DENOISER, 1, L)
    out["denoiser_5s"] = {"ms": 1e3 * t_den, "tokens_per_s": L / t_den, "tflops": fl / t_den / 1e12,
                          "frac_of_bf16_peak": fl / t_den / 1e12 / peaks["bf16_tflops"]}
    den.close()
    return out


def extra_line(w, args, dev, peaks):
    """One more workload on this GPU (single process), as a dict for the `extra` key."""
    r = measure(w, args, 0, 1, None, dev, with_e2e=False)
    tok = r["tokens_per_step_rank"] * args.steps
    inv_tf = r["inv_flops_rank"] / r["t_inv"] / 1e12
    out = {"workload": w.name, "steps": args.steps, "warmup": args.warmup,
           "inverse_tokens_per_s": tok / r["t_inv"], "fwd_tokens_per_s": tok / r["t_fwd"],
           "inverse_tflops": inv_tf, "fwd_tflops": r["fwd_flops_rank"] / r["t_fwd"] / 1e12,
           "inverse_frac_of_bf16_peak": inv_tf / peaks["bf16_tflops"],
           "mean_iters_per_block": float(np.mean([a.mean() for a in r["it_np"]])),
           "clocks": r["clk"]}
    return out, r


# ----------------------------------------------------------------------------- main

def fd_passes(args, dev):
    """The deep flow's Jacobi passes in a graph ncu can profile: the flow-encode
    of the 5 s clip in passes of 390 query rows, each attending the cache of
    the frames before it -- the shape of one Jacobi update of each block (the
    Jacobi graph itself has conditional nodes, whose kernels ncu does not
    profile).  Prints one JSON line (not the throughput contract's)."""
    import torch
    from video_generation_b200 import flow
    w = syn.WORKLOADS[4]
    model = flow.AFModel(w.shape, syn.make_weights(w.shape))
    x = torch.from_numpy(syn.workload_latents(w, "x")).to(dev)
    B = w.B // 2                                   # passes of 2B = 390 rows
    ws = model.workspace(1, w.L, B, device=dev)
    st = torch.cuda.current_stream()
    t = time_calls(lambda: flow.af_prefix_encode(model, x, 0, B, w.L, ws), args.warmup, args.steps, st)
    n_pass = w.L // (2 * B)
    fl = sum(FL.pass_flops(w.shape.d, w.shape.C, w.shape.layers, w.shape.mlp_ratio, 2 * B,
                           FL.causal_pairs(i * 2 * B, 2 * B)) for i in range(n_pass))
    peaks, kind = load_peaks()
    print(json.dumps({"mode": "fd_passes", "workload": w.name, "passes": n_pass, "rows_per_pass": 2 * B,
                      "ms_per_pass": 1e3 * t / n_pass, "tflops": fl / t / 1e12,
                      "frac_of_bf16_peak": fl / t / 1e12 / peaks["bf16_tflops"], "peak_kind": kind}), flush=True)


def relaunch_under_torchrun(args):
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={args.gpus}",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__)] + sys.argv[1:]
    os.execv(sys.executable, cmd)


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
    ap.add_argument("--no-extras", action="store_true", help="skip configs 2, 4, 5 in a one-GPU run")
    ap.add_argument("--fd-passes", action="store_true",
                    help="time (or profile) the deep flow's 390-row Jacobi passes outside the Jacobi graph")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        relaunch_under_torchrun(args)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        sys.stderr.write(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world}\n")
        sys.exit(2)
    w = syn.WORKLOADS[args.config]

    if args.impl == "reference":
        reference_arm(args, w, rank, world)
        return

    import torch
    import torch.distributed as dist

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if args.fd_passes:
        fd_passes(args, dev)
        return
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    r = measure(w, args, rank, world, dist if world > 1 else None, dev)
    peaks, peak_kind = load_peaks()
    tok = r["tokens_per_step_rank"] * args.steps * world
    inv_tf_rank = r["inv_flops_rank"] / r["t_inv"] / 1e12
    fwd_tf_rank = r["fwd_flops_rank"] / r["t_fwd"] / 1e12

    extras, cpu = {}, None
    if world == 1 and rank == 0:
        if not args.no_extras and args.config == 3:
            ex_args = argparse.Namespace(**vars(args))
            fd_inv_flops = None
            for cid, steps in ((2, max(3, min(args.steps, 20))), (4, 2), (5, 1)):
                ex_args.steps = steps
                try:
                    extras[syn.WORKLOADS[cid].name], rr = extra_line(syn.WORKLOADS[cid], ex_args, dev, peaks)
                    if cid == 5:
                        fd_inv_flops = rr["inv_flops_rank"] / steps
                except Exception as e:          # an extra must not lose the headline line
                    extras[syn.WORKLOADS[cid].name] = {"error": repr(e)[:200]}
            try:
                extras.update(deep_flow_extras(ex_args, dev, peaks))
            except Exception as e:
                extras["deep_flow_extras"] = {"error": repr(e)[:200]}
            if fd_inv_flops and not args.no_cpu_baseline:
                # the oracle's flop rate on the deep flow's first frame, and the
                # 30 s inverse's time extrapolated from it (labelled as such)
                w5 = syn.WORKLOADS[5]
                tok1, _, ti1, thr1, fl1 = run_oracle_sample(w5, 1)
                t_full = fd_inv_flops / (fl1 / ti1)
                extras[w5.name]["cpu_baseline"] = {
                    "kind": "oracle", "cores": thr1, "first_frame_inverse_s": ti1,
                    "extrapolated_full_inverse_s": t_full, "extrapolated_tokens_per_s": w5.L / t_full,
                    "sample": "the first frame (390 tokens, 24 layers) of the deep flow, Jacobi inverse",
                    "extrapolation": "the 30 s inverse's algorithmic flops (from the GPU run's iteration counts) "
                                     "over the oracle's measured flop rate on that frame"}
        if not args.no_cpu_baseline:
            cpu = cpu_baselines(w, args, r["inv_flops_rank"] / args.steps, r["tokens_per_step_rank"])

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    peak = peaks["bf16_tflops"]
    line = {
        "metric": "jacobi_inverse_latent_tokens_per_s", "value": tok / r["t_inv"], "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * (r["t_fwd"] + r["t_inv"]) / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "frames_per_gpu": r["batch"] if frame_sharded(w) else None,
                   "tokens_per_frame": w.shape.frame_len, "L": w.L, "T": w.T, "layers": w.shape.layers,
                   "d_model": w.shape.d, "B": w.B, "tau": w.tau, "max_iter": w.max_iter,
                   "l2": "flushed between steps",
                   "parallelism": (f"frames{world}" if frame_sharded(w) else f"replicas{world}")},
        "fwd_tokens_per_s": tok / r["t_fwd"],
        "fwd_tflops": fwd_tf_rank * world,
        "inverse_tflops": inv_tf_rank * world,
        "mean_iters_per_block": float(np.mean([a.mean() for a in r["it_np"]])),
        "max_iters_per_block": int(max(a.max() for a in r["it_np"])),
        "roofline": {"bound": "tensor", "achieved": inv_tf_rank, "peak": peak, "unit": "TFLOP/s",
                     "frac": inv_tf_rank / peak,
                     "traffic": C3_INVERSE_DRAM_BYTES if args.config == 3 else None,
                     "traffic_note": "DRAM bytes per inverse-graph launch, from an ncu capture of the forward "
                                     "graph scaled by passes (6 / 3); the graph moves them at "
                                     f"{C3_INVERSE_DRAM_BYTES / (r['t_inv'] / args.steps) / 1e9:.0f} GB/s"
                                     if args.config == 3 else None,
                     "kernel": "flow_stack_inverse graph, per GPU (tcgen05 GEMMs dominate)",
                     "peak_kind": f"bf16 dense burst, {peak_kind}",
                     "frac_of_sustained": inv_tf_rank / peaks.get("bf16_tflops_sustained", peak)},
        "clocks": r["clk"],
        "e2e": {"value": tok / r["t_e2e"], "unit": "tokens/s", "h2d_bytes_per_step": r["h2d"],
                "d2h_bytes_per_step": r["d2h"]},
        "gpu_launches": r["launches"] * args.steps,
    }
    if extras:
        line["extra"] = extras
    if cpu is not None:
        line["cpu_baseline"] = cpu
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
