"""bf16 tensor-core paths that the configuration-sized tests do not reach,
against the CPU oracle on small seeded inputs:

  * passes of fewer than 256 rows, which run the single-SM GEMM tiles
    (cta_group::1) instead of SM pairs;
  * odd sizes: 130-token sequences (a ragged 128-row query tile and 64-key
    tile), batch 3, Jacobi blocks of 65;
  * the max_iter cap: every block stops unconverged and is counted;
  * an identity head (all head weights 0): z = x and logdet = 0 exactly, one
    Jacobi update per block;
  * determinism: bitwise-equal reruns of the forward and the inverse.

bf16 tolerances as in test_gpu_parity: z (x) relative L2 <= 2e-2 against the
oracle, the transform part z - x (x - z) <= 3e-2, iteration counts within +-1.
"""
import numpy as np
import pytest
import torch

import synthetic as syn
from oracle import af_oracle as O
from tests.gpu_util import Pair, rel, sum_abs_s, to_dev, to_np

pytestmark = pytest.mark.gpu

BF_X_TOL, BF_PART_TOL = 2e-2, 3e-2
SHAPE = syn.ModelShape(C=64, d=128, heads=2, layers=2, mlp_ratio=4, frame_len=130, max_frames=2, dtype="bf16")


@pytest.fixture(scope="module")
def flow():
    from video_generation_b200 import build
    build.build()
    from video_generation_b200 import flow as F
    assert torch.cuda.is_available()
    return F


@pytest.fixture(scope="module")
def pair(flow):
    return Pair(flow, SHAPE, perturb=True, head_std=1e-2)


def _forward_check(flow, pair, x, direction):
    z, ld = flow.af_forward(pair.model, to_dev(x), direction)
    z_ref, ld_ref = O.af_forward(pair.blk, x, direction)
    zn, ldn = to_np(z), to_np(ld)
    assert rel(zn, z_ref) <= BF_X_TOL
    assert rel(zn - x, z_ref - x) <= BF_PART_TOL
    scale = sum_abs_s(pair.blk, x, direction)
    assert (np.abs(ldn - ld_ref) <= BF_PART_TOL * scale).all()


@pytest.mark.parametrize("direction", [O.L2R, O.R2L])
def test_fewer_than_256_rows_single_sm_tiles(flow, pair, direction):
    # one sample of 200 tokens: every GEMM of the pass has 200 rows
    x = syn.make_latents(1, 200, SHAPE.C, 51)
    _forward_check(flow, pair, x, direction)
    # Jacobi blocks of 100: the passes carry 100 or 200 rows
    z = syn.make_latents(1, 200, SHAPE.C, 52)
    x_ref, it_ref, _ = O.af_inverse_jacobi(pair.blk, z, direction, 100, 1e-3, 8, True)
    xg, it = flow.af_inverse_jacobi(pair.model, to_dev(z), direction, 100, 1e-3, 8, True)
    xn = to_np(xg)
    assert rel(xn, x_ref) <= BF_X_TOL and rel(xn - z, x_ref - z) <= BF_PART_TOL
    assert np.abs(it.cpu().numpy() - it_ref).max() <= 1
    assert pair.model.device_error() == 0


def test_odd_sizes_batch3_L130_B65(flow, pair):
    x = syn.make_latents(3, 130, SHAPE.C, 53)
    _forward_check(flow, pair, x, O.R2L)
    z = syn.make_latents(3, 130, SHAPE.C, 54)
    for warm in (False, True):
        x_ref, it_ref, conv_ref = O.af_inverse_jacobi(pair.blk, z, O.L2R, 65, 1e-3, 12, warm)
        ws = pair.model.workspace(3, 130, 65)
        xg, it = flow.af_inverse_jacobi(pair.model, to_dev(z), O.L2R, 65, 1e-3, 12, warm, ws=ws)
        flow.last_convergence(ws)
        xn = to_np(xg)
        assert rel(xn, x_ref) <= BF_X_TOL and rel(xn - z, x_ref - z) <= BF_PART_TOL
        assert np.abs(it.cpu().numpy() - it_ref).max() <= 1
    assert pair.model.device_error() == 0


def test_max_iter_cap_reports_every_block_unconverged(flow, pair):
    z = syn.make_latents(2, 260, SHAPE.C, 55)
    ws = pair.model.workspace(2, 260, 65)
    # tau = 0 can never be passed by a non-zero update: every block runs 2 updates
    xg, it = flow.af_inverse_jacobi(pair.model, to_dev(z), O.L2R, 65, 0.0, 2, True, ws=ws)
    assert flow.last_convergence(ws) == 2 * 4
    assert (it.cpu().numpy() == 2).all()
    x_ref, it_ref, conv_ref = O.af_inverse_jacobi(pair.blk, z, O.L2R, 65, 0.0, 2, True)
    assert not conv_ref.any() and (it_ref == 2).all()
    assert rel(to_np(xg) - z, x_ref - z) <= BF_PART_TOL
    assert pair.model.device_error() == 0


def test_identity_head_is_exact(flow):
    p = Pair(flow, SHAPE, perturb=True, zero=("head", "headbias"))
    x = syn.make_latents(2, 260, SHAPE.C, 56)
    z, ld = flow.af_forward(p.model, to_dev(x), O.R2L)
    np.testing.assert_array_equal(to_np(z), x.astype(np.float64))
    assert (to_np(ld) == 0).all()
    xi, it = flow.af_inverse_jacobi(p.model, z, O.R2L, 130, 1e-3, 8, False)
    np.testing.assert_array_equal(to_np(xi), x.astype(np.float64))
    assert (it.cpu().numpy() == 1).all()
    assert p.model.device_error() == 0


def test_bf16_results_are_bitwise_deterministic(flow, pair):
    x = to_dev(syn.make_latents(3, 260, SHAPE.C, 57))
    z1, l1 = flow.af_forward(pair.model, x, O.L2R)
    z2, l2 = flow.af_forward(pair.model, x, O.L2R)
    assert torch.equal(z1, z2) and torch.equal(l1, l2)
    a, ia = flow.af_inverse_jacobi(pair.model, z1, O.L2R, 65, 1e-3, 12, True)
    b, ib = flow.af_inverse_jacobi(pair.model, z1, O.L2R, 65, 1e-3, 12, True)
    assert torch.equal(a, b) and torch.equal(ia, ib)
