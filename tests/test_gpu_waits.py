"""Failure detection on the device: the bounded waits of the tensor-core kernels.

Every pipeline wait in the GEMM and attention kernels gives up after the
model's wait limit (af_set_wait_limit, 2 s by default): the CTA aborts, waits
(with its own bound) for the loads and MMAs it has in flight, frees its tensor
memory and sets the model's error word.  Here the limit is set to one
nanosecond, so that waits run out during a normal forward pass; the call must
return, af_device_error must report a pipeline wait (GEMM or attention, not a
failed drain), and the next call at the default limit must match the oracle.

One sample (200 rows) runs the GEMMs on single SMs; two samples (400 rows)
run them on SM pairs, whose second CTA's loads complete on the leader's
barriers: the second CTA reports how many loads it issued and the leader's
drain waits for them (completing by hand the bytes of loads it counted but the
second CTA never issued), so a pair that aborts at different k-blocks in its
two CTAs still drains every load before it exits.
"""
import numpy as np
import pytest
import torch

import synthetic as syn
from oracle import af_oracle as O
from tests.gpu_util import Pair, rel, to_dev, to_np

pytestmark = pytest.mark.gpu

SHAPE = syn.ModelShape(C=64, d=128, heads=2, layers=2, mlp_ratio=4, frame_len=200, max_frames=1, dtype="bf16")
ERR_GEMM_WAIT, ERR_DRAIN, ERR_ATTN_WAIT = 1, 2, 4   # bits of the device error word


@pytest.fixture(scope="module")
def flow():
    from video_generation_b200 import build
    build.build()
    from video_generation_b200 import flow as F
    assert torch.cuda.is_available()
    return F


@pytest.mark.parametrize("batch", [1, 2], ids=["single_sm", "sm_pair"])
def test_expired_waits_abort_cleanly_and_report(flow, batch):
    pair = Pair(flow, SHAPE, perturb=True, head_std=1e-2)
    x = syn.make_latents(batch, 200, SHAPE.C, 71)
    xd = to_dev(x)
    assert pair.model.device_error() == 0
    pair.model.set_wait_limit(1e-9)
    codes = []
    for _ in range(3):
        flow.af_forward(pair.model, xd, O.L2R)
        codes.append(pair.model.device_error())         # synchronises: the call returned
        if codes[-1]:
            break
    assert codes[-1] & (ERR_GEMM_WAIT | ERR_ATTN_WAIT), codes      # a pipeline wait ran out
    assert not codes[-1] & ERR_DRAIN, codes                          # every drain completed
    # the flag was cleared by the read; at the default limit the model works again
    pair.model.set_wait_limit(2.0)
    z, ld = flow.af_forward(pair.model, xd, O.L2R)
    z_ref, _ = O.af_forward(pair.blk, x, O.L2R)
    zn = to_np(z)
    assert rel(zn, z_ref) <= 2e-2 and rel(zn - x, z_ref - x) <= 3e-2
    assert pair.model.device_error() == 0


def test_wait_limit_rejects_bad_values(flow):
    pair = Pair(flow, SHAPE)
    lib = flow.lib()
    for bad in (0.0, -1.0, float("nan"), 61.0):
        assert lib.af_set_wait_limit(pair.model.handle, bad) == flow.AF_ERR_ARG
    assert lib.af_set_wait_limit(None, 1.0) == flow.AF_ERR_ARG
    assert lib.af_set_wait_limit(pair.model.handle, 0.5) == flow.AF_OK
