"""CUDA path vs the CPU oracle on seeded synthetic inputs, through the C ABI.

Tolerances (stated per precision):
  fp32 path (SIMT, no tensor cores): z and x relative L2 <= 1e-5 and max-abs
    <= 1e-5 * max|ref|; logdet |diff| <= 1e-5 * max(|ref|, sum|s|); Jacobi
    iteration counts identical.
  bf16 path (tensor cores, bf16 operands, fp32 accumulation and fp32 x/z/
    logdet): z relative L2 <= 2e-2 and GPU round trip inverse(forward(x)) vs x
    relative L2 <= 1e-2; in addition the transform part z - x (which carries
    all of mu and s) within 3e-2 relative L2, x within 2e-2 of the oracle's
    inverse and iteration counts within +-1 of the oracle's.
"""
import numpy as np
import pytest
import torch

import synthetic as syn
from oracle import af_oracle as O
from tests.gpu_util import Pair, max_abs_rel, rel, sum_abs_s, to_dev, to_np

pytestmark = pytest.mark.gpu

TOL32 = 1e-5


@pytest.fixture(scope="module")
def flow():
    from video_generation_b200 import build
    build.build()
    from video_generation_b200 import flow as F
    assert torch.cuda.is_available()
    return F


C1 = syn.WORKLOADS[1]
# c1 shapes with a temporal position table, for multi-block Jacobi with a KV cache
C1_FRAMES = syn.ModelShape(C=16, d=64, heads=2, layers=2, mlp_ratio=4, frame_len=16, max_frames=4, dtype="fp32")

FP32_VARIANTS = {
    "config": dict(shape=C1.shape, kw={}),
    "perturbed": dict(shape=C1.shape, kw=dict(perturb=True, head_std=0.05)),
    "frames": dict(shape=C1_FRAMES, kw=dict(perturb=True, head_std=0.05)),
}


def check_fp32_forward(pair, flow, x, direction):
    z_ref, ld_ref = O.af_forward(pair.blk, x, direction)
    z, ld = flow.af_forward(pair.model, to_dev(x), direction)
    torch.cuda.synchronize()
    z, ld = to_np(z), to_np(ld)
    assert rel(z, z_ref) <= TOL32 and max_abs_rel(z, z_ref) <= TOL32
    scale = np.maximum(np.abs(ld_ref), sum_abs_s(pair.blk, x, direction))
    assert (np.abs(ld - ld_ref) <= TOL32 * scale).all(), (ld, ld_ref)


@pytest.mark.parametrize("variant", sorted(FP32_VARIANTS))
@pytest.mark.parametrize("direction", [O.L2R, O.R2L])
def test_fp32_forward_matches_oracle(flow, variant, direction):
    v = FP32_VARIANTS[variant]
    pair = Pair(flow, v["shape"], **v["kw"])
    x = syn.make_latents(C1.batch, C1.L, C1.shape.C, syn.DATA_SEED + 1)
    check_fp32_forward(pair, flow, x, direction)


JACOBI_CASES = {
    # the configuration as specified: B = L = 64, tau 1e-3, max_iter 64
    "config": dict(shape=C1.shape, kw={}, B=64, tau=1e-3, max_iter=64, warm=0, dir=O.L2R),
    # a less trivial flow and a tight tau: several updates per block
    "tight_tau": dict(shape=C1.shape, kw=dict(perturb=True, head_std=0.05), B=64, tau=1e-7, max_iter=64,
                      warm=0, dir=O.L2R),
    # 4 blocks of 16: KV-cache commit, warm start, R->L flip
    "blocks_warm": dict(shape=C1_FRAMES, kw=dict(perturb=True, head_std=0.05), B=16, tau=1e-6, max_iter=16,
                        warm=1, dir=O.L2R),
    "blocks_cold_r2l": dict(shape=C1_FRAMES, kw=dict(perturb=True, head_std=0.05), B=16, tau=1e-6, max_iter=16,
                            warm=0, dir=O.R2L),
    # ragged: B = 8 (8 blocks), warm start
    "blocks8_warm_r2l": dict(shape=C1_FRAMES, kw=dict(perturb=True, head_std=0.05), B=8, tau=1e-5, max_iter=8,
                             warm=1, dir=O.R2L),
}


@pytest.mark.parametrize("case", sorted(JACOBI_CASES))
def test_fp32_jacobi_matches_oracle(flow, case):
    c = JACOBI_CASES[case]
    pair = Pair(flow, c["shape"], **c["kw"])
    z = syn.make_latents(C1.batch, C1.L, C1.shape.C, syn.DATA_SEED + 101)
    x_ref, it_ref, conv_ref = O.af_inverse_jacobi(pair.blk, z, c["dir"], c["B"], c["tau"], c["max_iter"],
                                                  bool(c["warm"]))
    ws = pair.model.workspace(C1.batch, C1.L, c["B"])
    x, it = flow.af_inverse_jacobi(pair.model, to_dev(z), c["dir"], c["B"], c["tau"], c["max_iter"], c["warm"],
                                   ws=ws)
    nonconv = flow.last_convergence(ws)
    x, it = to_np(x), it.cpu().numpy()
    np.testing.assert_array_equal(it, it_ref)
    assert nonconv == int((~conv_ref).sum())
    assert rel(x, x_ref) <= TOL32 and max_abs_rel(x, x_ref) <= TOL32
    assert pair.model.device_error() == 0


def test_fp32_jacobi_max_iter_cap_reports_not_converged(flow):
    pair = Pair(flow, C1_FRAMES, perturb=True, head_std=0.3)
    z = syn.make_latents(2, 64, 16, 7)
    x_ref, it_ref, conv_ref = O.af_inverse_jacobi(pair.blk, z, O.L2R, 16, 0.0, 2, True)
    ws = pair.model.workspace(2, 64, 16)
    x, it = flow.af_inverse_jacobi(pair.model, to_dev(z), O.L2R, 16, 0.0, 2, True, ws=ws)
    assert flow.last_convergence(ws) == 2 * 4
    assert (it.cpu().numpy() == 2).all() and not conv_ref.any()
    assert rel(to_np(x), x_ref) <= TOL32


def test_fp32_stack_matches_oracle(flow):
    dirs = (O.L2R, O.R2L, O.L2R)
    pairs = [Pair(flow, C1_FRAMES, seed_block=t, perturb=True, head_std=0.05) for t in range(3)]
    blocks = [p.blk for p in pairs]
    models = [p.model for p in pairs]
    x = syn.make_latents(2, 64, 16, 11)
    z_ref, ld_ref = O.stack_forward(blocks, dirs, x)
    z, ld = flow.flow_stack_forward(models, dirs, to_dev(x))
    torch.cuda.synchronize()
    assert rel(to_np(z), z_ref) <= TOL32
    assert np.abs(to_np(ld) - ld_ref).max() <= TOL32 * np.abs(ld_ref).max() * 10
    zr = syn.make_latents(2, 64, 16, 12)
    x_ref, it_ref = O.stack_inverse(blocks, dirs, zr, 16, 1e-6, 16, True)
    xg, itg = flow.flow_stack_inverse(models, dirs, to_dev(zr), 16, 1e-6, 16, True)
    np.testing.assert_array_equal(itg.cpu().numpy(), it_ref)
    assert rel(to_np(xg), x_ref) <= TOL32


def test_fp32_head_zero_identity_and_one_update(flow):
    pair = Pair(flow, C1.shape, perturb=True, zero=("head", "headbias"))
    x = syn.make_latents(2, 64, 16, 3)
    z, ld = flow.af_forward(pair.model, to_dev(x), O.L2R)
    xi, it = flow.af_inverse_jacobi(pair.model, z, O.L2R, 64, 1e-3, 64, False)
    np.testing.assert_array_equal(to_np(z), x.astype(np.float64))
    assert (to_np(ld) == 0).all()
    np.testing.assert_array_equal(to_np(xi), x.astype(np.float64))
    assert (it.cpu().numpy() == 1).all()


def test_gpu_results_are_deterministic(flow):
    pair = Pair(flow, C1_FRAMES, perturb=True, head_std=0.05)
    z = to_dev(syn.make_latents(2, 64, 16, 5))
    a, ia = flow.af_inverse_jacobi(pair.model, z, O.L2R, 16, 1e-6, 16, True)
    b, ib = flow.af_inverse_jacobi(pair.model, z, O.L2R, 16, 1e-6, 16, True)
    assert torch.equal(a, b) and torch.equal(ia, ib)


def test_later_frames_never_change_earlier_frames_on_gpu(flow):
    pair = Pair(flow, C1_FRAMES, perturb=True, head_std=0.05)
    z = syn.make_latents(1, 64, 16, 6)
    z2 = z.copy()
    z2[0, 48:] += 1.0
    a, _ = flow.af_inverse_jacobi(pair.model, to_dev(z), O.L2R, 16, 1e-6, 16, True)
    b, _ = flow.af_inverse_jacobi(pair.model, to_dev(z2), O.L2R, 16, 1e-6, 16, True)
    assert torch.equal(a[0, :48], b[0, :48])
    assert (a[0, 48:] - b[0, 48:]).abs().max().item() > 1e-3


# ------------------------------------------------------------------ bf16 (tensor cores)

BF_X_TOL = 2e-2       # z vs oracle (relative L2)
BF_RT_TOL = 1e-2      # GPU round trip
BF_PART_TOL = 3e-2    # transform part z - x vs the oracle's


def bf16_forward_check(pair, flow, x, direction, x_np_ref=None):
    z_ref, ld_ref = O.af_forward(pair.blk, x, direction)
    z, ld = flow.af_forward(pair.model, to_dev(x), direction)
    torch.cuda.synchronize()
    z, ld = to_np(z), to_np(ld)
    assert rel(z, z_ref) <= BF_X_TOL
    assert rel(z - x, z_ref - x) <= BF_PART_TOL, rel(z - x, z_ref - x)
    scale = sum_abs_s(pair.blk, x, direction)
    assert (np.abs(ld - ld_ref) <= BF_PART_TOL * scale).all(), (ld, ld_ref)
    return z


@pytest.fixture(scope="module")
def c2(flow):
    w = syn.WORKLOADS[2]
    return w, Pair(flow, w.shape)


def test_bf16_c2_forward_matches_oracle(flow, c2):
    w, pair = c2
    x = syn.workload_latents(w, "x")
    bf16_forward_check(pair, flow, x, O.L2R)


def test_bf16_c2_perturbed_forward_matches_oracle(flow):
    w = syn.WORKLOADS[2]
    pair = Pair(flow, w.shape, perturb=True, head_std=5e-3)
    x = syn.workload_latents(w, "x")[:2]
    bf16_forward_check(pair, flow, x, O.R2L)


def test_bf16_c2_jacobi_matches_oracle_and_round_trips(flow, c2):
    w, pair = c2
    z = syn.workload_latents(w, "z")
    x_ref, it_ref, _ = O.af_inverse_jacobi(pair.blk, z, O.L2R, w.B, w.tau, w.max_iter, bool(w.warm_start))
    x, it = flow.af_inverse_jacobi(pair.model, to_dev(z), O.L2R, w.B, w.tau, w.max_iter, w.warm_start)
    xn = to_np(x)
    assert rel(xn, x_ref) <= BF_X_TOL
    assert rel(xn - z, x_ref - z) <= BF_PART_TOL
    assert np.abs(it.cpu().numpy() - it_ref).max() <= 1
    # round trip on the GPU: forward(x) then inverse
    x0 = syn.workload_latents(w, "x")
    zz, _ = flow.af_forward(pair.model, to_dev(x0), O.L2R)
    xb, _ = flow.af_inverse_jacobi(pair.model, zz, O.L2R, w.B, w.tau, w.max_iter, w.warm_start)
    assert rel(to_np(xb), x0) <= BF_RT_TOL
    assert pair.model.device_error() == 0


def test_bf16_c3_stack_sampled_frames_match_oracle(flow):
    w = syn.WORKLOADS[3]
    pairs = [Pair(flow, w.shape, seed_block=t) for t in range(w.T)]
    models = [p.model for p in pairs]
    blocks = [p.blk for p in pairs]
    frames = [0, 10, 20]
    x = syn.workload_latents(w, "x")
    z, ld = flow.flow_stack_forward(models, w.dirs, to_dev(x))
    z_ref, ld_ref = O.stack_forward(blocks, w.dirs, x[frames])
    zn = to_np(z)[frames]
    assert rel(zn, z_ref) <= BF_X_TOL
    assert rel(zn - x[frames], z_ref - x[frames]) <= BF_PART_TOL
    zr = syn.workload_latents(w, "z")
    xg, itg = flow.flow_stack_inverse(models, w.dirs, to_dev(zr), w.B, w.tau, w.max_iter, w.warm_start)
    x_ref, it_ref = O.stack_inverse(blocks, w.dirs, zr[frames], w.B, w.tau, w.max_iter, bool(w.warm_start))
    xn = to_np(xg)[frames]
    assert rel(xn, x_ref) <= BF_X_TOL
    assert rel(xn - zr[frames], x_ref - zr[frames]) <= BF_PART_TOL
    assert np.abs(itg.cpu().numpy()[:, frames] - it_ref).max() <= 1
    # full-size round trip through all 21 frames
    xb, _ = flow.flow_stack_inverse(models, w.dirs, z, w.B, w.tau, w.max_iter, w.warm_start)
    assert rel(to_np(xb), x) <= BF_RT_TOL
