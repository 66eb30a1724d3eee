"""The flow-score-matching denoiser forward (af_denoise) against the CPU oracle
("STARFlow-V ... paper notes", key design 2: s_phi(x_{<=n+1}) regresses the
scaled score of frame n; the sample is refined as x_noisy + sigma * s_phi).

fp32 path: x relative L2 and max-abs <= 1e-5.  bf16 path: the refinement
sigma * s_phi = x - x_noisy within 3e-2 relative L2 of the oracle's (x itself
is within 2e-2).  On the GPU the look-ahead must hold bit for bit: frame n's
output never changes with frames > n + 1, and does change with frame n + 1.
"""
import numpy as np
import pytest
import torch

import synthetic as syn
from oracle import af_oracle as O
from tests.gpu_util import max_abs_rel, rel, to_dev, to_np

pytestmark = pytest.mark.gpu

TOL32, BF_X_TOL, BF_PART_TOL = 1e-5, 2e-2, 3e-2
FP32 = syn.ModelShape(C=16, d=64, heads=2, layers=3, mlp_ratio=4, frame_len=16, max_frames=4, dtype="fp32")
BF16 = syn.ModelShape(C=128, d=128, heads=2, layers=2, mlp_ratio=4, frame_len=130, max_frames=4, dtype="bf16")


@pytest.fixture(scope="module")
def flow():
    from video_generation_b200 import build
    build.build()
    from video_generation_b200 import flow as F
    assert torch.cuda.is_available()
    return F


def _pair(flow, shape, block=100):
    W = syn.make_denoiser_weights(shape, block=block, perturb=True)
    return O.DenoiserBlock(shape, W), flow.AFModel(shape, W, denoiser=True)


def test_fp32_denoise_matches_oracle(flow):
    blk, model = _pair(flow, FP32)
    xn = syn.make_latents(2, 64, FP32.C, 81)
    x = to_np(flow.af_denoise(model, to_dev(xn), 0.3))
    x_ref = O.denoise(blk, xn, 0.3)
    assert rel(x, x_ref) <= TOL32 and max_abs_rel(x, x_ref) <= TOL32
    assert rel(x - xn, x_ref - xn) <= 10 * TOL32
    assert model.device_error() == 0


def test_bf16_denoise_matches_oracle(flow):
    blk, model = _pair(flow, BF16)
    xn = syn.make_latents(2, 520, BF16.C, 82)
    x = to_np(flow.af_denoise(model, to_dev(xn), 0.25))
    x_ref = O.denoise(blk, xn, 0.25)
    assert rel(x, x_ref) <= BF_X_TOL
    assert rel(x - xn, x_ref - xn) <= BF_PART_TOL
    assert model.device_error() == 0


def test_denoiser_workload_first_frames_match_oracle(flow):
    """The pipeline's denoiser (8 layers, d 768) on the 21-frame clip: the first
    two frames depend only on frames 0-2, which the oracle computes alone."""
    sh = syn.DENOISER
    blk, model = _pair(flow, sh)
    F = sh.frame_len
    xn = syn.make_latents(1, 21 * F, sh.C, 83)
    x = to_np(flow.af_denoise(model, to_dev(xn), 0.1))
    x_ref = O.denoise(blk, xn[:, :3 * F], 0.1)
    assert rel(x[:, :2 * F] - xn[:, :2 * F], x_ref[:, :2 * F] - xn[:, :2 * F]) <= BF_PART_TOL
    assert np.isfinite(x).all()
    assert model.device_error() == 0


@pytest.mark.parametrize("shape", [FP32, BF16], ids=["fp32", "bf16"])
def test_lookahead_is_exactly_one_frame_on_gpu(flow, shape):
    blk, model = _pair(flow, shape)
    F = shape.frame_len
    L = shape.max_len
    xn = syn.make_latents(1, L, shape.C, 84)
    y = flow.af_denoise(model, to_dev(xn), 0.5)
    x2 = xn.copy()
    x2[0, 2 * F:] += 1.0                                  # frames >= 2
    y2 = flow.af_denoise(model, to_dev(x2), 0.5)
    assert torch.equal(y[0, :F], y2[0, :F])               # frame 0 does not see frame 2 or later
    assert (y[0, F:2 * F] - y2[0, F:2 * F]).abs().max().item() > 1e-4   # frame 1 does see frame 2


def test_denoiser_and_flow_calls_reject_each_others_models(flow):
    _, den = _pair(flow, FP32)
    fl = flow.AFModel(FP32, syn.make_weights(FP32))
    x = torch.zeros((1, 64, FP32.C), device="cuda")
    with pytest.raises(flow.AFError):
        flow.af_denoise(fl, x, 0.1, ws=fl.workspace(1, 64))
    with pytest.raises(flow.AFError):
        flow.af_forward(den, x, 0, ws=den.workspace(1, 64))


def test_bf16_denoiser_needs_a_head_tile_width(flow):
    bad = syn.ModelShape(C=64, d=128, heads=2, layers=1, mlp_ratio=4, frame_len=130, max_frames=1, dtype="bf16")
    with pytest.raises(flow.AFError):
        flow.AFModel(bad, syn.make_denoiser_weights(bad), denoiser=True)
