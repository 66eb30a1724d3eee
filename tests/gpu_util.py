"""Helpers shared by the GPU parity tests: run the CUDA path and the CPU oracle on
the same seeded synthetic inputs and measure their agreement."""
import numpy as np
import torch

import synthetic as syn
from oracle import af_oracle as O


def rel(a, b) -> float:
    a = np.asarray(a, np.float64).ravel()
    b = np.asarray(b, np.float64).ravel()
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def max_abs_rel(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.abs(a - b).max() / max(np.abs(b).max(), 1e-300))


def sum_abs_s(blk, x, direction):
    """sum_{i,c} |s_{i,c}| per sample (scale for logdet errors, avoids cancellation)."""
    out = []
    for xb in x:
        xw = np.asarray(xb[::-1] if direction == O.R2L else xb, np.float64)
        _, s, _ = O.transformer_rows(blk, O.masked_inputs(xw, 0, xw.shape[0]), 0)
        out.append(np.abs(s).sum())
    return np.array(out)


def to_dev(a):
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda()


def to_np(t):
    return t.detach().cpu().numpy().astype(np.float64)


class Pair:
    """One AF block on both sides."""

    def __init__(self, flow, shape, seed_block=0, **kw):
        self.shape = shape
        self.W = syn.make_weights(shape, block=seed_block, **kw)
        self.blk = O.Block(shape, self.W)
        self.model = flow.AFModel(shape, self.W)
