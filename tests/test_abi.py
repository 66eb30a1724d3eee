"""The C-ABI library: it builds, loads and exports every symbol include/af.h
declares; argument checks that need no device work.  No GPU needed."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "af.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(af_\w+|flow_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from video_generation_b200 import build
    build.build()
    from video_generation_b200 import flow
    return flow.lib()


def test_header_declares_the_boundary_calls():
    names = _declared()
    for must in ("af_forward", "af_inverse_jacobi", "flow_stack_forward", "flow_stack_inverse",
                 "af_model_create", "af_workspace_bytes"):
        assert must in names


def test_library_exports_every_declared_symbol(lib):
    missing = [n for n in _declared() if not hasattr(lib, n)]
    assert not missing, missing


def test_binding_export_list_matches_header():
    from video_generation_b200 import flow
    assert sorted(flow.EXPORTS) == _declared()


def test_argument_checks_need_no_device(lib):
    from video_generation_b200 import flow
    c = flow.AFConfigC(16, 64, 2, 2, 4, 64, 1, flow.FP32)
    assert lib.af_num_tensors(ctypes.byref(c)) == 4 + 12 * 2 + 4
    # null model / tensors / output
    assert lib.af_model_create(None, None, 0, None) == flow.AF_ERR_ARG
    h = ctypes.c_void_p()
    assert lib.af_model_create(ctypes.byref(c), None, 32, ctypes.byref(h)) == flow.AF_ERR_ARG
    # invalid configs are rejected before any CUDA call
    dummy = (ctypes.c_void_p * 32)(*([1] * 32))
    for bad in [flow.AFConfigC(16, 64, 3, 2, 4, 64, 1, flow.FP32),     # d % heads
                flow.AFConfigC(12, 64, 2, 2, 4, 64, 1, flow.FP32),     # C % 8
                flow.AFConfigC(16, 64, 2, 2, 4, 64, 1, 7),             # dtype
                flow.AFConfigC(96, 768, 12, 2, 4, 390, 1, flow.BF16),  # bf16: C % 64
                flow.AFConfigC(192, 768, 24, 2, 4, 390, 1, flow.BF16)]:  # bf16: head dim 32
        assert lib.af_model_create(ctypes.byref(bad), dummy, lib.af_num_tensors(ctypes.byref(bad)),
                                   ctypes.byref(h)) == flow.AF_ERR_ARG
    # wrong tensor count
    assert lib.af_model_create(ctypes.byref(c), dummy, 31, ctypes.byref(h)) == flow.AF_ERR_ARG
    assert lib.af_workspace_bytes(None, 1, 64, 64) == 0
    assert lib.af_forward(None, None, 1, 64, 0, None, None, None, 0, None) == flow.AF_ERR_ARG
    assert lib.af_inverse_jacobi(None, None, 1, 64, 0, 64, 1e-3, 8, 0, None, None, None, 0, None) == flow.AF_ERR_ARG
    assert lib.flow_stack_forward(None, None, 0, None, 1, 64, None, None, None, 0, None) == flow.AF_ERR_ARG
    assert lib.flow_stack_inverse(None, None, 0, None, 1, 64, 64, 1e-3, 8, 0, None, None, None, 0, None) == flow.AF_ERR_ARG
    assert lib.af_status_string(flow.AF_NOT_CONVERGED).startswith(b"AF_NOT_CONVERGED")


def test_product_path_has_no_oracle_or_cpu_fallback():
    pkg = os.path.join(ROOT, "video_generation_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                txt = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in txt and "from oracle" not in txt, f
                assert "af_oracle" not in txt, f
