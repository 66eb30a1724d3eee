"""Seeded synthetic workloads shared by the oracle tests, the GPU tests and the bench.

This module only *draws numbers*: model shapes, seeded random weights and
seeded latents.  It holds none of the flow's arithmetic (no normalisation, no
attention, no affine map, no rounding), so both the CUDA path and the CPU
oracle can take their inputs from here without sharing any of the method.

Workloads follow the five configurations of the affine-autoregressive-flow
hot path of STARFlow-V ("STARFlow-V: End-to-End Video Generative Modeling with
Autoregressive Normalizing Flows", paper notes, section "Method / overall
framework"): latents of a WAN2.2-style 3D causal VAE (48 channels, 16x spatial,
4x temporal compression) at 480p, 16 fps, patchified 2x2 into tokens of
C = 192 channels; 30x52 latent pixels per frame give 390 tokens per frame.
A 5 s clip is 81 frames -> 21 latent frames; a 30 s clip is taken as 120
latent frames.

Weight init (the pages give none; the plain reading used throughout):
  * every projection matrix ~ N(0, 0.02^2) (std 0.02),
  * the (mu, log-sigma) head ~ N(0, 1e-3^2) (std 1e-3), so the flow starts
    near the identity,
  * learned absolute position tables ~ N(0, 0.02^2),
  * biases 0, LayerNorm gain 1 and shift 0.
``perturb=True`` draws non-trivial biases / LayerNorm parameters and a larger
head scale, so that tests exercise every term.
"""
from __future__ import annotations

import dataclasses
from typing import List

import numpy as np

L2R, R2L = 0, 1


@dataclasses.dataclass(frozen=True)
class ModelShape:
    C: int            # channels per token
    d: int            # transformer width
    heads: int
    layers: int
    mlp_ratio: int
    frame_len: int    # tokens per latent frame (spatial position table rows)
    max_frames: int   # temporal position table rows
    dtype: str        # "fp32" or "bf16": the arithmetic the GPU path uses

    @property
    def max_len(self) -> int:
        return self.frame_len * self.max_frames

    @property
    def hd(self) -> int:
        return self.d // self.heads


@dataclasses.dataclass(frozen=True)
class Workload:
    cid: int
    name: str
    shape: ModelShape
    batch: int
    L: int
    dirs: tuple       # one direction per AF block of the stack
    B: int
    tau: float
    max_iter: int
    warm_start: int

    @property
    def T(self) -> int:
        return len(self.dirs)

    @property
    def tokens(self) -> int:
        return self.batch * self.L


_FS = dict(C=192, d=768, heads=12, mlp_ratio=4, frame_len=390, max_frames=1, dtype="bf16")
_FD = ModelShape(C=192, d=2048, heads=16, layers=24, mlp_ratio=4, frame_len=390,
                 max_frames=120, dtype="bf16")

WORKLOADS = {
    1: Workload(1, "tiny_af_fp32",
                ModelShape(C=16, d=64, heads=2, layers=2, mlp_ratio=4, frame_len=64,
                           max_frames=1, dtype="fp32"),
                batch=2, L=64, dirs=(L2R,), B=64, tau=1e-3, max_iter=64, warm_start=0),
    2: Workload(2, "fs_single_frame_8L_d768_bf16", ModelShape(layers=8, **_FS),
                batch=4, L=390, dirs=(L2R,), B=390, tau=1e-3, max_iter=390, warm_start=0),
    3: Workload(3, "fs_stack_T3_4L_d768_21frames_bf16", ModelShape(layers=4, **_FS),
                batch=21, L=390, dirs=(L2R, R2L, L2R), B=390, tau=1e-3, max_iter=390,
                warm_start=0),
    4: Workload(4, "fd_24L_d2048_5s_8190tok_bf16", _FD,
                batch=1, L=8190, dirs=(L2R,), B=390, tau=1e-3, max_iter=32, warm_start=1),
    5: Workload(5, "fd_24L_d2048_30s_46800tok_bf16", _FD,
                batch=1, L=46800, dirs=(L2R,), B=390, tau=1e-3, max_iter=32, warm_start=1),
}

WEIGHT_SEED = 1234
DATA_SEED = 5678


def tensor_specs(s: ModelShape):
    """Canonical (name, shape, kind) order of one AF block's tensors.

    ``kind`` selects the init: 'w' projection, 'head', 'pos', 'bias', 'gain',
    'shift'.  Matrices are [out_features, in_features] (row-major).
    """
    d, C, f = s.d, s.C, s.mlp_ratio * s.d
    spec = [("w_in", (d, C), "w"), ("b_in", (d,), "bias"),
            ("pos_space", (s.frame_len, d), "pos"), ("pos_time", (s.max_frames, d), "pos")]
    for l in range(s.layers):
        spec += [(f"l{l}.ln1_g", (d,), "gain"), (f"l{l}.ln1_b", (d,), "shift"),
                 (f"l{l}.w_qkv", (3 * d, d), "w"), (f"l{l}.b_qkv", (3 * d,), "bias"),
                 (f"l{l}.w_o", (d, d), "w"), (f"l{l}.b_o", (d,), "bias"),
                 (f"l{l}.ln2_g", (d,), "gain"), (f"l{l}.ln2_b", (d,), "shift"),
                 (f"l{l}.w_1", (f, d), "w"), (f"l{l}.b_1", (f,), "bias"),
                 (f"l{l}.w_2", (d, f), "w"), (f"l{l}.b_2", (d,), "bias")]
    spec += [("lnf_g", (d,), "gain"), ("lnf_b", (d,), "shift"),
             ("w_head", (2 * C, d), "head"), ("b_head", (2 * C,), "headbias")]
    return spec


def make_weights(s: ModelShape, seed: int = WEIGHT_SEED, block: int = 0,
                 perturb: bool = False, head_std: float | None = None,
                 zero: tuple = ()) -> List[np.ndarray]:
    """Seeded fp32 weights of one AF block, in ``tensor_specs`` order.

    ``zero`` lists tensor kinds to set to 0 (special-case tests).
    """
    rng = np.random.default_rng([seed, block])
    hs = head_std if head_std is not None else (2e-2 if perturb else 1e-3)
    out = []
    for name, shape, kind in tensor_specs(s):
        if kind in zero:
            out.append(np.zeros(shape, np.float32))
            continue
        if kind in ("w", "pos"):
            a = rng.standard_normal(shape, dtype=np.float32) * np.float32(0.02)
        elif kind == "head":
            a = rng.standard_normal(shape, dtype=np.float32) * np.float32(hs)
        elif kind in ("bias", "shift", "headbias"):
            a = (rng.standard_normal(shape, dtype=np.float32) * np.float32(0.02)
                 if perturb else np.zeros(shape, np.float32))
        elif kind == "gain":
            a = (np.float32(1.0) + rng.standard_normal(shape, dtype=np.float32) * np.float32(0.1)
                 if perturb else np.ones(shape, np.float32))
        else:  # pragma: no cover
            raise ValueError(kind)
        out.append(np.ascontiguousarray(a, dtype=np.float32))
    return out


def denoiser_specs(s: ModelShape):
    """Tensor order of the flow-score-matching denoiser: the AF block's, with a
    head of C rows (s_phi has one output per channel)."""
    spec = tensor_specs(s)
    return spec[:-2] + [("w_head", (s.C, s.d), "w"), ("b_head", (s.C,), "bias")]


def make_denoiser_weights(s: ModelShape, seed: int = WEIGHT_SEED, block: int = 100,
                          perturb: bool = False) -> List[np.ndarray]:
    """Seeded fp32 denoiser weights in ``denoiser_specs`` order (head ~ N(0, 0.02^2)
    like the other projections)."""
    rng = np.random.default_rng([seed, block])
    out = []
    for name, shape, kind in denoiser_specs(s):
        if kind in ("w", "pos"):
            a = rng.standard_normal(shape, dtype=np.float32) * np.float32(0.02)
        elif kind in ("bias", "shift"):
            a = (rng.standard_normal(shape, dtype=np.float32) * np.float32(0.02)
                 if perturb else np.zeros(shape, np.float32))
        else:  # gain
            a = (np.float32(1.0) + rng.standard_normal(shape, dtype=np.float32) * np.float32(0.1)
                 if perturb else np.ones(shape, np.float32))
        out.append(np.ascontiguousarray(a, dtype=np.float32))
    return out


# the denoiser of the pipeline: 8 layers at the shallow blocks' width, frames of 390 tokens
DENOISER = ModelShape(C=192, d=768, heads=12, layers=8, mlp_ratio=4, frame_len=390, max_frames=21, dtype="bf16")


def make_stack_weights(w: Workload, **kw) -> List[List[np.ndarray]]:
    return [make_weights(w.shape, block=t, **kw) for t in range(w.T)]


def make_latents(batch: int, L: int, C: int, seed: int, scale: float = 1.0) -> np.ndarray:
    """x or z ~ N(0, scale^2), fp32, [batch, L, C] row-major."""
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((batch, L, C), dtype=np.float32) * np.float32(scale))


def workload_latents(w: Workload, which: str = "x") -> np.ndarray:
    off = {"x": 0, "z": 100}[which]
    return make_latents(w.batch, w.L, w.shape.C, DATA_SEED + w.cid + off)


def clip_frames(w: Workload, which: str, lo: int, hi: int) -> np.ndarray:
    """Frames lo..hi-1 of a clip of per-frame sequences (the shallow stack's
    workload: frames are its batch), [hi - lo, L, C].  Frame f is drawn from
    its own seed, so a process can draw any range of a clip of any length
    without drawing the rest."""
    off = {"x": 0, "z": 100}[which]
    out = np.empty((hi - lo, w.L, w.shape.C), np.float32)
    for i, f in enumerate(range(lo, hi)):
        rng = np.random.default_rng([DATA_SEED + w.cid + off, f])
        out[i] = rng.standard_normal((w.L, w.shape.C), dtype=np.float32)
    return out
