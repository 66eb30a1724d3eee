"""Argument checks of the C ABI against a real model on the device.

A tiny fp32 AF block (C 16, d 64, longest sequence 64 tokens) is created on
cuda:0; every call below with a bad argument must return the status that
include/af.h documents, with a message in af_last_error_string(), before it
enqueues any work: empty or over-long inputs, L not a multiple of B, a
non-positive iteration cap, a tau that is negative, NaN or infinite, aliased
x and z, a bad direction, stacks of blocks with different shapes, and a
workspace that is missing, short or misaligned.
"""
import ctypes
import math

import pytest
import torch

import synthetic as syn

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def env():
    from video_generation_b200 import build
    build.build()
    from video_generation_b200 import flow
    assert torch.cuda.is_available()
    shape = syn.WORKLOADS[1].shape                    # C 16, d 64, frame_len 64 x 1 frame
    model = flow.AFModel(shape, syn.make_weights(shape))
    shallower = syn.ModelShape(C=shape.C, d=shape.d, heads=shape.heads, layers=1, mlp_ratio=shape.mlp_ratio,
                               frame_len=shape.frame_len, max_frames=shape.max_frames, dtype=shape.dtype)
    other = flow.AFModel(shallower, syn.make_weights(shallower))
    return flow, model, other, shape


def _p(t):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _rejected(flow, status, expect):
    assert status == expect, flow.lib().af_status_string(status)
    assert flow.lib().af_last_error_string()


def test_forward_rejects_bad_arguments(env):
    flow, m, _, sh = env
    lib = flow.lib()
    batch, L = 2, sh.frame_len * sh.max_frames
    x = torch.randn(batch, L, sh.C, device="cuda")
    z = torch.empty_like(x)
    ld = torch.empty(batch, device="cuda")
    ws = m.workspace(batch, L)
    n = ws.numel()

    def fwd(b=batch, length=L, d=flow.L2R, xx=x, zz=z, w=_p(ws), nb=n):
        return lib.af_forward(m.handle, _p(xx), b, length, d, _p(zz), _p(ld), w, nb, None)

    assert fwd() == flow.AF_OK                         # the well-formed call, as a control
    torch.cuda.synchronize()
    _rejected(flow, fwd(b=0), flow.AF_ERR_ARG)         # empty batch
    _rejected(flow, fwd(length=0), flow.AF_ERR_ARG)    # empty sequence
    _rejected(flow, fwd(length=L + 1), flow.AF_ERR_ARG)  # longer than the model's positions
    _rejected(flow, fwd(d=2), flow.AF_ERR_ARG)         # no such direction
    _rejected(flow, fwd(zz=x), flow.AF_ERR_ARG)        # z aliases x
    _rejected(flow, fwd(w=ctypes.c_void_p(0)), flow.AF_ERR_WORKSPACE)
    _rejected(flow, fwd(nb=n - 1), flow.AF_ERR_WORKSPACE)
    _rejected(flow, fwd(w=ctypes.c_void_p(ws.data_ptr() + 16), nb=n - 16), flow.AF_ERR_WORKSPACE)
    assert lib.af_forward(None, _p(x), batch, L, 0, _p(z), _p(ld), _p(ws), n, None) == flow.AF_ERR_ARG
    assert m.device_error() == 0


def test_inverse_rejects_bad_arguments(env):
    flow, m, _, sh = env
    lib = flow.lib()
    batch, L, B = 2, sh.frame_len * sh.max_frames, 32
    z = torch.randn(batch, L, sh.C, device="cuda")
    x = torch.empty_like(z)
    it = torch.zeros(batch, L // B, dtype=torch.int32, device="cuda")
    ws = m.workspace(batch, L, B)
    n = ws.numel()

    def inv(b=batch, length=L, blk=B, tau=1e-3, mi=8, xx=x, zz=z, its=it, w=_p(ws), nb=n):
        return lib.af_inverse_jacobi(m.handle, _p(zz), b, length, 0, blk, tau, mi, 0, _p(xx), _p(its), w, nb, None)

    assert inv() == flow.AF_OK
    torch.cuda.synchronize()
    _rejected(flow, inv(blk=0), flow.AF_ERR_ARG)        # no block size
    _rejected(flow, inv(blk=24), flow.AF_ERR_ARG)       # 64 % 24 != 0
    _rejected(flow, inv(mi=0), flow.AF_ERR_ARG)         # no update allowed
    for tau in (-1e-3, math.nan, math.inf):
        _rejected(flow, inv(tau=tau), flow.AF_ERR_ARG)
    _rejected(flow, inv(xx=z), flow.AF_ERR_ARG)         # x aliases z
    _rejected(flow, inv(its=None), flow.AF_ERR_ARG)     # nowhere to count iterations
    _rejected(flow, inv(b=0), flow.AF_ERR_ARG)
    _rejected(flow, inv(length=L + B), flow.AF_ERR_ARG)
    _rejected(flow, inv(nb=n - 1), flow.AF_ERR_WORKSPACE)
    assert m.device_error() == 0


def test_stacks_need_one_shape_and_at_least_one_block(env):
    flow, m, other, sh = env
    lib = flow.lib()
    batch, L = 1, sh.frame_len * sh.max_frames
    x = torch.randn(batch, L, sh.C, device="cuda")
    z = torch.empty_like(x)
    ld = torch.empty(batch, device="cuda")
    ws = m.workspace(batch, L)
    blocks = (ctypes.c_void_p * 2)(m.handle, other.handle)
    dirs = (ctypes.c_int * 2)(flow.L2R, flow.R2L)
    _rejected(flow, lib.flow_stack_forward(blocks, dirs, 2, _p(x), batch, L, _p(z), _p(ld), _p(ws), ws.numel(),
                                           None), flow.AF_ERR_ARG)
    _rejected(flow, lib.flow_stack_forward(blocks, dirs, 0, _p(x), batch, L, _p(z), _p(ld), _p(ws), ws.numel(),
                                           None), flow.AF_ERR_ARG)
    it = torch.zeros(2, batch, 1, dtype=torch.int32, device="cuda")
    _rejected(flow, lib.flow_stack_inverse(blocks, dirs, 2, _p(z), batch, L, L, 1e-3, 8, 0, _p(x), _p(it), _p(ws),
                                           ws.numel(), None), flow.AF_ERR_ARG)
    n = ctypes.c_int(-1)
    assert lib.af_last_convergence(None, ctypes.byref(n), None) == flow.AF_ERR_ARG
