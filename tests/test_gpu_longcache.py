"""The long-cache attention path against the CPU oracle.

Jacobi passes of a long video have few query rows (one or two blocks) and a
long KV cache, so the tensor-core attention splits the live key range into
several splits and merges their partial (o, max, sum) triples ("STARFlow-V ...
paper notes", key design 3: finished blocks feed a KV cache that every later
block attends to).  These tests compare that path with the oracle element by
element, at sizes where the split path really runs with two or more non-empty
splits:

  * a small model (d 128, two heads of 64) on 6144 tokens: forward and the
    whole block-Jacobi inverse with warm start, every block;
  * a head-dim-128 model (d 256, two heads of 128) on the 30 s clip's 46 800
    tokens (120 frames): forward (the last two frames, from the oracle's
    forward computed frame by frame through its cache) and the inverse's last
    two blocks, teacher-forced: the oracle observes the GPU's first 118
    frames and runs the Jacobi of frames 118-119 itself;
  * the 5 s clip's geometry (d 2048, 16 heads of 128, 8190 tokens) with 2
    layers: the inverse's last frame teacher-forced the same way;
  * the full 24-layer 5 s forward against stored oracle rows of every frame
    (tests/golden/make_fd_forward_golden.py wrote them with the oracle).

Tolerances are those of the other bf16 tests: z (x) relative L2 <= 2e-2
against the oracle, the transform part z - x (x - z) <= 3e-2, GPU round trip
inverse(forward(x)) vs x <= 1e-2, Jacobi iteration counts within +-1.
"""
import hashlib
import os

import numpy as np
import pytest
import torch

import synthetic as syn
from oracle import af_oracle as O
from tests.gpu_util import rel, to_dev, to_np

pytestmark = pytest.mark.gpu

BF_X_TOL, BF_PART_TOL, BF_RT_TOL = 2e-2, 3e-2, 1e-2
GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "fd_5s_forward_rows.txt")


@pytest.fixture(scope="module")
def flow():
    from video_generation_b200 import build
    build.build()
    from video_generation_b200 import flow as F
    assert torch.cuda.is_available()
    return F


def split_region_bytes(model, batch, L, B, L_short):
    """Workspace bytes beyond what the sequence length alone explains.

    Between a call on L and one on L_short (same batch and B) only the KV
    cache, the stack buffer and the attention's split partials change size;
    the first two are known exactly, so what remains (minus alignment) is the
    split partials' region, which exists only when the call may split."""
    sh = model.shape
    es = 2 if sh.dtype == "bf16" else 4
    grow = model.workspace_bytes(batch, L, B) - model.workspace_bytes(batch, L_short, B)
    kv = es * sh.layers * 2 * batch * (L - L_short) * sh.d
    tmp = 4 * batch * (L - L_short) * sh.C
    return grow - kv - tmp


# ------------------------------------------------------------------ small split model, every block

SMALL = syn.ModelShape(C=64, d=128, heads=2, layers=2, mlp_ratio=4, frame_len=256, max_frames=24, dtype="bf16")


@pytest.fixture(scope="module")
def small(flow):
    W = syn.make_weights(SMALL, perturb=True, head_std=5e-3)
    return O.Block(SMALL, W), flow.AFModel(SMALL, W)


def test_small_split_kv_forward_matches_oracle(flow, small):
    blk, model = small
    L = SMALL.max_len
    x = syn.make_latents(1, L, SMALL.C, 31)
    z, ld = flow.af_forward(model, to_dev(x), O.L2R)
    z_ref, ld_ref = O.af_forward(blk, x, O.L2R)
    zn = to_np(z)
    assert rel(zn, z_ref) <= BF_X_TOL
    assert rel(zn - x, z_ref - x) <= BF_PART_TOL
    # the late frames, whose rows attend thousands of keys, on their own
    assert rel(zn[:, -256:] - x[:, -256:], z_ref[:, -256:] - x[:, -256:]) <= BF_PART_TOL
    assert model.device_error() == 0


def test_small_split_kv_inverse_every_block_matches_oracle(flow, small):
    blk, model = small
    L, B = SMALL.max_len, 256
    # the Jacobi passes (at most 2B query rows) split the key range
    assert split_region_bytes(model, 1, L, B, 2 * B) > 4096
    z = syn.make_latents(1, L, SMALL.C, 32)
    ws = model.workspace(1, L, B)
    x, it = flow.af_inverse_jacobi(model, to_dev(z), O.L2R, B, 1e-3, 16, True, ws=ws)
    flow.last_convergence(ws)
    x_ref, it_ref, _ = O.af_inverse_jacobi(blk, z, O.L2R, B, 1e-3, 16, True)
    xn = to_np(x)
    assert rel(xn, x_ref) <= BF_X_TOL
    assert rel(xn - z, x_ref - z) <= BF_PART_TOL
    for b in (L // B - 2, L // B - 1):         # blocks whose keys span every split
        sl = slice(b * B, (b + 1) * B)
        assert rel(xn[:, sl] - z[:, sl], x_ref[:, sl] - z[:, sl]) <= BF_PART_TOL
    assert np.abs(it.cpu().numpy() - it_ref).max() <= 1
    # round trip on the GPU: inverse(forward(x)) = x
    x0 = syn.make_latents(1, L, SMALL.C, 33)
    zz, _ = flow.af_forward(model, to_dev(x0), O.L2R)
    xb, _ = flow.af_inverse_jacobi(model, zz, O.L2R, B, 1e-3, 16, True, ws=ws)
    assert rel(to_np(xb), x0) <= BF_RT_TOL
    assert model.device_error() == 0


# ------------------------------------------------------------------ head dim 128, 46 800 tokens

HD128 = syn.ModelShape(C=64, d=256, heads=2, layers=2, mlp_ratio=4, frame_len=390, max_frames=120, dtype="bf16")


@pytest.fixture(scope="module")
def hd128(flow):
    W = syn.make_weights(HD128, perturb=True, head_std=5e-3)
    return O.Block(HD128, W), flow.AFModel(HD128, W)


def test_hd128_46800_forward_last_frames_match_oracle(flow, hd128):
    blk, model = hd128
    L, F = HD128.max_len, HD128.frame_len
    x = syn.make_latents(1, L, HD128.C, 41)
    z, ld = flow.af_forward(model, to_dev(x), O.L2R)
    z_tail, ld_ref, sabs = O.af_forward_chunked_one(blk, x[0], O.L2R, F, keep_from=L - 2 * F)
    zn = to_np(z)[0, -2 * F:]
    xt = x[0, -2 * F:]
    assert rel(zn, z_tail) <= BF_X_TOL
    assert rel(zn - xt, z_tail - xt) <= BF_PART_TOL
    assert abs(float(to_np(ld)[0]) - ld_ref) <= BF_PART_TOL * sabs
    assert model.device_error() == 0


def test_hd128_46800_inverse_last_blocks_teacher_forced(flow, hd128):
    blk, model = hd128
    L, B = HD128.max_len, HD128.frame_len
    assert split_region_bytes(model, 1, L, B, 2 * B) > 4096
    z = syn.make_latents(1, L, HD128.C, 42)
    ws = model.workspace(1, L, B)
    x, it = flow.af_inverse_jacobi(model, to_dev(z), O.L2R, B, 1e-3, 32, True, ws=ws)
    flow.last_convergence(ws)
    assert model.device_error() == 0
    xn, itn = to_np(x), it.cpu().numpy()
    nk = L // B - 2
    x_ref, it_ref, _ = O.af_inverse_jacobi(blk, z, O.L2R, B, 1e-3, 32, True, x_known=xn, n_known=nk)
    tail = slice(nk * B, L)
    assert rel(xn[:, tail], x_ref[:, tail]) <= BF_X_TOL
    assert rel(xn[:, tail] - z[:, tail], x_ref[:, tail] - z[:, tail]) <= BF_PART_TOL
    assert np.abs(itn[:, nk:] - it_ref[:, nk:]).max() <= 1


# ------------------------------------------------------------------ 5 s clip geometry, teacher-forced last frame

FD2 = syn.ModelShape(C=192, d=2048, heads=16, layers=2, mlp_ratio=4, frame_len=390, max_frames=120, dtype="bf16")


def test_fd_geometry_5s_last_frame_teacher_forced(flow):
    w = syn.WORKLOADS[4]
    W = syn.make_weights(FD2)
    blk, model = O.Block(FD2, W), flow.AFModel(FD2, W)
    del W
    assert split_region_bytes(model, 1, w.L, w.B, 2 * w.B) > 4096
    z = syn.workload_latents(w, "z")
    ws = model.workspace(1, w.L, w.B)
    x, it = flow.af_inverse_jacobi(model, to_dev(z), O.L2R, w.B, w.tau, w.max_iter, True, ws=ws)
    flow.last_convergence(ws)
    assert model.device_error() == 0
    xn, itn = to_np(x), it.cpu().numpy()
    nk = w.L // w.B - 1
    x_ref, it_ref, _ = O.af_inverse_jacobi(blk, z, O.L2R, w.B, w.tau, w.max_iter, True, x_known=xn, n_known=nk)
    tail = slice(nk * w.B, w.L)
    assert rel(xn[:, tail], x_ref[:, tail]) <= BF_X_TOL
    assert rel(xn[:, tail] - z[:, tail], x_ref[:, tail] - z[:, tail]) <= BF_PART_TOL
    assert abs(int(itn[0, nk]) - int(it_ref[0, nk])) <= 1
    # and the whole inverse passes the round trip through the GPU forward
    zz, _ = flow.af_forward(model, x, O.L2R)
    assert rel(to_np(zz), z) <= BF_RT_TOL
    model.close()


# ------------------------------------------------------------------ full 24-layer 5 s forward vs stored oracle rows

def _read_golden():
    meta, rows = {}, []
    with open(GOLDEN) as f:
        for line in f:
            if line.startswith("# inputs sha256"):
                meta["digest"] = line.split()[-1]
            elif line.startswith("# logdet"):
                meta["logdet"] = float(line.split()[-1])
            elif line.startswith("# sum_abs_s"):
                meta["sum_abs_s"] = float(line.split()[-1])
            elif line.startswith("# rows"):
                meta["rows"] = [int(v) for v in line.split()[2:]]
            elif not line.startswith("#"):
                rows.append([float(v) for v in line.split()])
    return meta, np.array(rows)


def test_fd_5s_full_forward_every_frame_matches_oracle_rows(flow):
    w = syn.WORKLOADS[4]
    meta, z_ref = _read_golden()
    W = syn.make_weights(w.shape)
    x = syn.workload_latents(w, "x")
    h = hashlib.sha256()
    for a in W:
        h.update(np.ascontiguousarray(a, np.float32).tobytes())
    h.update(np.ascontiguousarray(x, np.float32).tobytes())
    assert h.hexdigest() == meta["digest"], "synthetic inputs differ from those the golden rows were made from"
    model = flow.AFModel(w.shape, W)
    del W
    z, ld = flow.af_forward(model, to_dev(x), O.L2R)
    rows = meta["rows"]
    assert len(rows) == 3 * (w.L // w.B) and len(set(r // w.B for r in rows)) == w.L // w.B
    zn = to_np(z)[0, rows]
    xr = x[0, rows]
    assert rel(zn, z_ref) <= BF_X_TOL
    assert rel(zn - xr, z_ref - xr) <= BF_PART_TOL
    for f in range(w.L // w.B):                  # every frame on its own
        sl = slice(3 * f, 3 * f + 3)
        assert rel(zn[sl] - xr[sl], z_ref[sl] - xr[sl]) <= BF_PART_TOL, f
    assert abs(float(to_np(ld)[0]) - meta["logdet"]) <= BF_PART_TOL * meta["sum_abs_s"]
    assert model.device_error() == 0
    model.close()
