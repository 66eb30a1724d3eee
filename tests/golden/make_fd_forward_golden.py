"""Writes tests/golden/fd_5s_forward_rows.txt: the CPU oracle's forward pass of
the deep frame-causal flow f_D at full size (24 layers, d 2048, 16 heads, MLP
4x, bf16-rounded weights; a 5 s 480p 16 fps clip = 21 latent frames x 390
tokens x 192 channels, seeded synthetic weights and latents), sampled at the
first, middle and last token of every frame, plus the logdet and the sum of
|s| (the scale a bf16 logdet is judged against).

The forward is the affine AF block of "STARFlow-V: End-to-End Video Generative
Modeling with Autoregressive Normalizing Flows" (CVPR 2026 paper notes, key
design 1: z = (x - mu(x*m)) / sigma(x*m); loss section: logdet = -sum log
sigma).  Only oracle/ computes; synthetic/ draws the inputs.  The file also
records a digest of the inputs, which the GPU test recomputes so that a change
of the generator cannot go unnoticed.  Takes about ten minutes on 8 cores.

    python tests/golden/make_fd_forward_golden.py
"""
import hashlib
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import synthetic as syn  # noqa: E402
from oracle import af_oracle as O  # noqa: E402

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "fd_5s_forward_rows.txt")


def sample_rows(w):
    """Row indices (into the 8190 tokens) sampled in every frame: its first, middle and last token."""
    F = w.shape.frame_len
    return [f * F + t for f in range(w.L // F) for t in (0, F // 2, F - 1)]


def input_digest(w):
    h = hashlib.sha256()
    for a in syn.make_weights(w.shape):
        h.update(np.ascontiguousarray(a, np.float32).tobytes())
    h.update(np.ascontiguousarray(syn.workload_latents(w, "x"), np.float32).tobytes())
    return h.hexdigest()


def main():
    w = syn.WORKLOADS[4]
    blk = O.Block(w.shape, syn.make_weights(w.shape))
    x = syn.workload_latents(w, "x")
    z, ld, sabs = O.af_forward_one(blk, x[0], O.L2R, with_abs=True)
    rows = sample_rows(w)
    with open(OUT, "w") as f:
        f.write("# oracle forward of f_D (24 layers, d 2048) on the 21-frame 5 s clip; see make_fd_forward_golden.py\n")
        f.write(f"# inputs sha256 {input_digest(w)}\n")
        f.write(f"# logdet {ld!r}\n")
        f.write(f"# sum_abs_s {sabs!r}\n")
        f.write("# rows " + " ".join(str(r) for r in rows) + "\n")
        for r in rows:
            f.write(" ".join(f"{v:.9e}" for v in z[r]) + "\n")


if __name__ == "__main__":
    main()
