"""af_forward_noalloc: the forward pass for callers that cannot allocate device
memory (a host that owns all GPU memory itself and hands the library only
input and output buffers).  It must give af_forward's results, within the
tolerances of the other parity tests, on consecutive calls that share its
fixed scratch array, and refuse work larger than that array.

This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

import synthetic as syn

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 32 << 20


def _rel(a, b):
    a = a.double().cpu().numpy().ravel()
    b = b.double().cpu().numpy().ravel()
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


@pytest.fixture(scope="module")
def flow():
    from video_generation_b200 import build
    build.build()
    from video_generation_b200 import flow as F
    assert torch.cuda.is_available()
    return F


CASES = [
    # (shape, batch, L, direction, tolerance of the matching parity tests)
    (syn.ModelShape(C=16, d=64, heads=2, layers=2, mlp_ratio=4, frame_len=16, max_frames=4, dtype="fp32"),
     2, 64, 1, 1e-5),
    (syn.ModelShape(C=192, d=768, heads=12, layers=2, mlp_ratio=4, frame_len=390, max_frames=1, dtype="bf16"),
     1, 390, 0, 2e-2),
]


@pytest.mark.parametrize("case", range(len(CASES)))
def test_noalloc_forward_matches_af_forward_on_two_calls(flow, case):
    shape, batch, L, direction, tol = CASES[case]
    model = flow.AFModel(shape, syn.make_weights(shape, perturb=True, head_std=0.02))
    lib = flow.lib()
    assert model.workspace_bytes(batch, L) <= SCRATCH_BYTES
    stream = torch.cuda.current_stream()
    for call in range(2):
        x = torch.from_numpy(syn.make_latents(batch, L, shape.C, 900 + call)).cuda()
        z_ref, ld_ref = flow.af_forward(model, x, direction)
        z = torch.full_like(x, float("nan"))
        ld = torch.full((batch,), float("nan"), device="cuda")
        st = lib.af_forward_noalloc(model.handle, ctypes.c_void_p(x.data_ptr()), batch, L, direction,
                                    ctypes.c_void_p(z.data_ptr()), ctypes.c_void_p(ld.data_ptr()),
                                    ctypes.c_void_p(stream.cuda_stream))
        assert st == flow.AF_OK, lib.af_last_error_string()
        torch.cuda.synchronize()
        assert _rel(z, z_ref) <= tol
        assert (ld - ld_ref).abs().max().item() <= tol * max(1.0, ld_ref.abs().max().item())
    assert model.device_error() == 0


def test_noalloc_refuses_work_beyond_its_scratch(flow):
    shape = CASES[1][0]
    model = flow.AFModel(shape, syn.make_weights(shape))
    lib = flow.lib()
    batch = 8                                   # 8 frames of 390 tokens need > 32 MiB
    assert model.workspace_bytes(batch, 390) > SCRATCH_BYTES
    x = torch.zeros((batch, 390, shape.C), device="cuda")
    z = torch.empty_like(x)
    ld = torch.empty(batch, device="cuda")
    st = lib.af_forward_noalloc(model.handle, ctypes.c_void_p(x.data_ptr()), batch, 390, 0,
                                ctypes.c_void_p(z.data_ptr()), ctypes.c_void_p(ld.data_ptr()),
                                ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == flow.AF_ERR_WORKSPACE
    assert b"scratch" in lib.af_last_error_string()
