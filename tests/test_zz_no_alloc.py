"""af_forward_noalloc: the forward pass for callers that cannot allocate device
memory (a host that owns all GPU memory itself and hands the library only
input and output buffers).  It must give af_forward's results, within the
tolerances of the other parity tests, on consecutive calls that share its
fixed scratch array -- including calls of other models, precisions, batch
sizes and lengths in between, which leave their data in the scratch --
allocate nothing while doing so, and refuse work larger than that array.

This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

import synthetic as syn

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 32 << 20

FP32 = syn.ModelShape(C=16, d=64, heads=2, layers=2, mlp_ratio=4, frame_len=16, max_frames=4, dtype="fp32")
BF16 = syn.ModelShape(C=192, d=768, heads=12, layers=2, mlp_ratio=4, frame_len=390, max_frames=1, dtype="bf16")

# (model, batch, L, direction, tolerance of the matching parity tests), called in this order:
# bf16 after fp32 and back, batch and length changing from call to call
CALLS = [("bf16", 1, 390, 0, 2e-2), ("bf16", 1, 390, 0, 2e-2), ("fp32", 2, 64, 1, 1e-5), ("bf16", 2, 200, 1, 2e-2),
         ("fp32", 1, 48, 0, 1e-5), ("bf16", 1, 390, 0, 2e-2), ("fp32", 2, 64, 1, 1e-5)]


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


def _noalloc(flow, model, x, z, ld, direction, stream):
    batch, L, _ = x.shape
    return flow.lib().af_forward_noalloc(model.handle, ctypes.c_void_p(x.data_ptr()), batch, L, direction,
                                         ctypes.c_void_p(z.data_ptr()), ctypes.c_void_p(ld.data_ptr()),
                                         ctypes.c_void_p(stream.cuda_stream))


def test_noalloc_forward_matches_af_forward_on_consecutive_calls(flow):
    models = {"fp32": flow.AFModel(FP32, syn.make_weights(FP32, perturb=True, head_std=0.02)),
              "bf16": flow.AFModel(BF16, syn.make_weights(BF16, perturb=True, head_std=0.02))}
    stream = torch.cuda.current_stream()
    # every input, reference and output buffer exists before the first no-alloc call
    cases = []
    for i, (kind, batch, L, direction, tol) in enumerate(CALLS):
        m = models[kind]
        assert m.workspace_bytes(batch, L) <= SCRATCH_BYTES
        C = m.shape.C
        x = torch.from_numpy(syn.make_latents(batch, L, C, 900 + i)).cuda()
        z_ref, ld_ref = flow.af_forward(m, x, direction)
        z = torch.full_like(x, float("nan"))
        ld = torch.full((batch,), float("nan"), device="cuda")
        cases.append((m, x, z, ld, direction, tol, z_ref, ld_ref))
    # the first call on the device looks up the scratch array's address
    m, x, z, ld, direction, *_ = cases[0]
    assert _noalloc(flow, m, x, z, ld, direction, stream) == flow.AF_OK
    torch.cuda.synchronize()
    free_before, _ = torch.cuda.mem_get_info()
    for (m, x, z, ld, direction, tol, z_ref, ld_ref) in cases:
        z.fill_(float("nan"))
        st = _noalloc(flow, m, x, z, ld, direction, stream)
        assert st == flow.AF_OK, flow.lib().af_last_error_string()
    torch.cuda.synchronize()
    free_after, _ = torch.cuda.mem_get_info()
    assert free_after == free_before                  # the calls allocated no device memory
    for (m, x, z, ld, direction, tol, z_ref, ld_ref) in cases:
        assert _rel(z, z_ref) <= tol
        assert (ld - ld_ref).abs().max().item() <= tol * max(1.0, ld_ref.abs().max().item())
    for m in models.values():
        assert m.device_error() == 0


def test_noalloc_refuses_work_beyond_its_scratch(flow):
    model = flow.AFModel(BF16, syn.make_weights(BF16))
    lib = flow.lib()
    batch = 8                                   # 8 frames of 390 tokens need > 32 MiB
    assert model.workspace_bytes(batch, 390) > SCRATCH_BYTES
    x = torch.zeros((batch, 390, BF16.C), device="cuda")
    z = torch.empty_like(x)
    ld = torch.empty(batch, device="cuda")
    st = lib.af_forward_noalloc(model.handle, ctypes.c_void_p(x.data_ptr()), batch, 390, 0,
                                ctypes.c_void_p(z.data_ptr()), ctypes.c_void_p(ld.data_ptr()),
                                ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == flow.AF_ERR_WORKSPACE
    assert b"scratch" in lib.af_last_error_string()
