"""Thin Python binding of libaf (include/af.h): argument marshalling only.

Every step of the affine-autoregressive-flow path runs in libaf's CUDA
kernels; PyTorch only provides device memory and the current stream.  If
libaf.so is missing or cannot load, importing this module raises: there is no
fallback path.

Names follow the C ABI: ``af_forward``, ``af_inverse_jacobi``,
``flow_stack_forward``, ``flow_stack_inverse``.
"""
from __future__ import annotations

import ctypes
import os
from typing import List, Sequence

import numpy as np
import torch

L2R, R2L = 0, 1
FP32, BF16 = 0, 1

AF_OK, AF_ERR_ARG, AF_ERR_CUDA, AF_ERR_WORKSPACE, AF_NOT_CONVERGED, AF_ERR_DEVICE = range(6)

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libaf.so")

EXPORTS = ("af_num_tensors", "af_model_create", "af_model_destroy", "af_workspace_bytes", "af_forward",
           "af_inverse_jacobi", "flow_stack_forward", "flow_stack_inverse", "af_last_convergence",
           "af_device_error", "af_status_string", "af_last_error_string", "af_forward_noalloc",
           "af_inverse_jacobi_schedule", "af_prefix_encode", "flow_pipeline_workspace_bytes",
           "flow_pipeline_inverse", "af_set_wait_limit", "af_denoiser_num_tensors", "af_denoiser_create",
           "af_denoise", "af_stream_workspace_bytes", "af_inverse_jacobi_stream")


class AFConfigC(ctypes.Structure):
    _fields_ = [("C", ctypes.c_int), ("d", ctypes.c_int), ("heads", ctypes.c_int), ("layers", ctypes.c_int),
                ("mlp_ratio", ctypes.c_int), ("frame_len", ctypes.c_int), ("max_frames", ctypes.c_int),
                ("dtype", ctypes.c_int)]


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise RuntimeError(f"libaf.so not built at {path}: run `python -m video_generation_b200.build`")
    lib = ctypes.CDLL(path)
    vp, i, sz, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
    P = ctypes.POINTER
    lib.af_num_tensors.argtypes = [P(AFConfigC)]
    lib.af_num_tensors.restype = i
    lib.af_model_create.argtypes = [P(AFConfigC), P(vp), i, P(vp)]
    lib.af_model_destroy.argtypes = [vp]
    lib.af_workspace_bytes.argtypes = [vp, i, i, i]
    lib.af_workspace_bytes.restype = sz
    lib.af_forward.argtypes = [vp, vp, i, i, i, vp, vp, vp, sz, vp]
    lib.af_inverse_jacobi.argtypes = [vp, vp, i, i, i, i, f, i, i, vp, vp, vp, sz, vp]
    lib.flow_stack_forward.argtypes = [P(vp), P(i), i, vp, i, i, vp, vp, vp, sz, vp]
    lib.flow_stack_inverse.argtypes = [P(vp), P(i), i, vp, i, i, i, f, i, i, vp, vp, vp, sz, vp]
    lib.af_forward_noalloc.argtypes = [vp, vp, i, i, i, vp, vp, vp]
    lib.af_inverse_jacobi_schedule.argtypes = [vp, vp, i, i, i, P(i), i, i, i, f, i, i, vp, vp, vp, sz, vp]
    lib.af_prefix_encode.argtypes = [vp, vp, i, i, i, i, i, vp, sz, vp]
    lib.af_set_wait_limit.argtypes = [vp, ctypes.c_double]
    lib.af_denoiser_num_tensors.argtypes = [P(AFConfigC)]
    lib.af_denoiser_num_tensors.restype = i
    lib.af_denoiser_create.argtypes = [P(AFConfigC), P(vp), i, P(vp)]
    lib.af_denoise.argtypes = [vp, vp, i, i, f, vp, vp, sz, vp]
    lib.af_stream_workspace_bytes.argtypes = [vp, i, i]
    lib.af_stream_workspace_bytes.restype = sz
    lib.af_inverse_jacobi_stream.argtypes = [vp, vp, i, i, i, i, f, i, i, vp, vp, vp, sz, vp]
    lib.flow_pipeline_workspace_bytes.argtypes = [vp, i, i, i, i]
    lib.flow_pipeline_workspace_bytes.restype = sz
    lib.flow_pipeline_inverse.argtypes = [vp, P(vp), P(i), i, vp, i, i, i, f, i, i, i, i, vp, vp, vp, vp, sz, vp, sz,
                                          vp, vp]
    lib.af_last_convergence.argtypes = [vp, P(i), vp]
    lib.af_device_error.argtypes = [vp, P(i)]
    lib.af_status_string.argtypes = [i]
    lib.af_status_string.restype = ctypes.c_char_p
    lib.af_last_error_string.argtypes = []
    lib.af_last_error_string.restype = ctypes.c_char_p
    for name in EXPORTS:
        if name not in ("af_status_string", "af_last_error_string", "af_num_tensors", "af_workspace_bytes",
                        "flow_pipeline_workspace_bytes", "af_denoiser_num_tensors", "af_stream_workspace_bytes"):
            getattr(lib, name).restype = i
    return lib


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _lib = load_library()
    return _lib


class AFError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        L = lib()
        msg = f"{L.af_status_string(status).decode()}: {L.af_last_error_string().decode()}"
        super().__init__(f"{what}: {msg}" if what else msg)
        self.status = status


def _check(status: int, what: str):
    if status != AF_OK:
        raise AFError(status, what)


def _ptr(t):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


class AFModel:
    """One AF block's weights (or, with denoiser=True, the denoiser's) on the
    current CUDA device (owned by libaf)."""

    def __init__(self, shape, tensors: Sequence[np.ndarray], denoiser: bool = False):
        self.shape = shape
        self.cfg = AFConfigC(shape.C, shape.d, shape.heads, shape.layers, shape.mlp_ratio, shape.frame_len,
                             shape.max_frames, BF16 if shape.dtype == "bf16" else FP32)
        arrs = [np.ascontiguousarray(t, dtype=np.float32) for t in tensors]
        ptrs = (ctypes.c_void_p * len(arrs))(*[a.ctypes.data for a in arrs])
        h = ctypes.c_void_p()
        create = lib().af_denoiser_create if denoiser else lib().af_model_create
        _check(create(ctypes.byref(self.cfg), ptrs, len(arrs), ctypes.byref(h)), "model create")
        self.handle = h

    def close(self):
        if getattr(self, "handle", None):
            lib().af_model_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def workspace_bytes(self, batch: int, L: int, B: int | None = None) -> int:
        return int(lib().af_workspace_bytes(self.handle, batch, L, L if B is None else B))

    def workspace(self, batch: int, L: int, B: int | None = None, device=None) -> torch.Tensor:
        n = self.workspace_bytes(batch, L, B)
        if n == 0:
            raise AFError(AF_ERR_ARG, "af_workspace_bytes")
        return torch.empty(n, dtype=torch.uint8, device=device or "cuda")

    def set_wait_limit(self, seconds: float):
        """Limit of one pipeline wait in the tensor-core kernels (default 2 s)."""
        _check(lib().af_set_wait_limit(self.handle, float(seconds)), "af_set_wait_limit")

    def device_error(self) -> int:
        code = ctypes.c_int(0)
        lib().af_device_error(self.handle, ctypes.byref(code))
        return code.value


def af_forward(model: AFModel, x: torch.Tensor, direction: int, ws: torch.Tensor | None = None,
               z: torch.Tensor | None = None, logdet: torch.Tensor | None = None, stream=None):
    """z = (x - mu) * exp(-s), logdet = -sum s per sample; x [batch, L, C] fp32 on the device."""
    return flow_stack_forward([model], [direction], x, ws=ws, z=z, logdet=logdet, stream=stream)


def af_inverse_jacobi(model: AFModel, z: torch.Tensor, direction: int, B: int, tau: float, max_iter: int,
                      warm_start: bool, ws: torch.Tensor | None = None, x: torch.Tensor | None = None,
                      iters: torch.Tensor | None = None, stream=None):
    """Block-Jacobi inverse; returns (x, iters [batch, L/B])."""
    x, it = flow_stack_inverse([model], [direction], z, B, tau, max_iter, warm_start, ws=ws, x=x,
                               iters=None if iters is None else iters.view(1, *iters.shape), stream=stream)
    return x, it[0]


def flow_stack_forward(models: List[AFModel], dirs: Sequence[int], x: torch.Tensor, ws: torch.Tensor | None = None,
                       z: torch.Tensor | None = None, logdet: torch.Tensor | None = None, stream=None):
    batch, L, _ = x.shape
    if ws is None:
        ws = models[0].workspace(batch, L, device=x.device)
    z = torch.empty_like(x) if z is None else z
    logdet = torch.empty(batch, dtype=torch.float32, device=x.device) if logdet is None else logdet
    T = len(models)
    hs = (ctypes.c_void_p * T)(*[m.handle for m in models])
    ds = (ctypes.c_int * T)(*dirs)
    _check(lib().flow_stack_forward(hs, ds, T, _ptr(x), batch, L, _ptr(z), _ptr(logdet), _ptr(ws), ws.numel(),
                                    _stream(stream)), "flow_stack_forward")
    return z, logdet


def flow_stack_inverse(models: List[AFModel], dirs: Sequence[int], z: torch.Tensor, B: int, tau: float,
                       max_iter: int, warm_start: bool, ws: torch.Tensor | None = None,
                       x: torch.Tensor | None = None, iters: torch.Tensor | None = None, stream=None):
    batch, L, _ = z.shape
    T = len(models)
    if ws is None:
        ws = models[0].workspace(batch, L, B, device=z.device)
    x = torch.empty_like(z) if x is None else x
    if iters is None:
        iters = torch.zeros((T, batch, L // max(B, 1)), dtype=torch.int32, device=z.device)
    hs = (ctypes.c_void_p * T)(*[m.handle for m in models])
    ds = (ctypes.c_int * T)(*dirs)
    _check(lib().flow_stack_inverse(hs, ds, T, _ptr(z), batch, L, B, float(tau), int(max_iter), int(bool(warm_start)),
                                    _ptr(x), _ptr(iters), _ptr(ws), ws.numel(), _stream(stream)),
           "flow_stack_inverse")
    return x, iters


def last_convergence(ws: torch.Tensor, stream=None) -> int:
    """Synchronises and returns how many (sample, block) pairs stopped at max_iter unconverged."""
    n = ctypes.c_int(0)
    s = lib().af_last_convergence(_ptr(ws), ctypes.byref(n), _stream(stream))
    if s not in (AF_OK, AF_NOT_CONVERGED):
        _check(s, "af_last_convergence")
    return n.value


def af_inverse_jacobi_schedule(model: AFModel, z: torch.Tensor, direction: int, block_sizes: Sequence[int],
                               tau: float, max_iter: int, warm_start: bool, b_begin: int = 0, b_end: int | None = None,
                               ws: torch.Tensor | None = None, x: torch.Tensor | None = None,
                               iters: torch.Tensor | None = None, stream=None):
    """Block-Jacobi inverse over a schedule of block sizes, blocks b_begin..b_end-1.

    Returns (x, iters [batch, n_blocks]); only the range's entries are written."""
    batch, L, _ = z.shape
    n = len(block_sizes)
    b_end = n if b_end is None else b_end
    if ws is None:
        ws = model.workspace(batch, L, max(block_sizes), device=z.device)
    x = torch.empty_like(z) if x is None else x
    iters = torch.zeros((batch, n), dtype=torch.int32, device=z.device) if iters is None else iters
    sizes = (ctypes.c_int * n)(*[int(b) for b in block_sizes])
    _check(lib().af_inverse_jacobi_schedule(model.handle, _ptr(z), batch, L, direction, sizes, n, b_begin, b_end,
                                            float(tau), int(max_iter), int(bool(warm_start)), _ptr(x), _ptr(iters),
                                            _ptr(ws), ws.numel(), _stream(stream)), "af_inverse_jacobi_schedule")
    return x, iters


def af_prefix_encode(model: AFModel, x: torch.Tensor, direction: int, B: int, n_tokens: int, ws: torch.Tensor,
                     stream=None):
    """Writes the K/V of positions 0..n_tokens-1 of x into ws (laid out for blocks of at most B)."""
    batch, L, _ = x.shape
    _check(lib().af_prefix_encode(model.handle, _ptr(x), batch, L, direction, B, n_tokens, _ptr(ws), ws.numel(),
                                  _stream(stream)), "af_prefix_encode")


def pipeline_workspace(shallow: List[AFModel], batch: int, frame_len: int, group: int = 1,
                       device=None) -> torch.Tensor:
    n = int(lib().flow_pipeline_workspace_bytes(shallow[0].handle, len(shallow), batch, frame_len, group))
    if n == 0:
        raise AFError(AF_ERR_ARG, "flow_pipeline_workspace_bytes")
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def flow_pipeline_inverse(deep: AFModel, shallow: List[AFModel], shallow_dirs: Sequence[int], z: torch.Tensor,
                          B: int, tau: float, max_iter_deep: int, max_iter_shallow: int, warm_start: bool,
                          group: int = 1, ws_deep: torch.Tensor | None = None, ws_shallow: torch.Tensor | None = None,
                          x: torch.Tensor | None = None, iters_deep: torch.Tensor | None = None,
                          iters_shallow: torch.Tensor | None = None, stream=None, stream_shallow=None):
    """x = f_S^{-1}(f_D^{-1}(z)), the shallow stack of each group of `group` frames on a second stream as
    the deep flow finishes it.  Returns (x, iters_deep [batch, L/B], iters_shallow [T, batch, L/frame_len])."""
    batch, L, _ = z.shape
    F = deep.shape.frame_len
    T = len(shallow)
    ws_deep = deep.workspace(batch, L, B, device=z.device) if ws_deep is None else ws_deep
    ws_shallow = pipeline_workspace(shallow, batch, F, group, device=z.device) if ws_shallow is None else ws_shallow
    x = torch.empty_like(z) if x is None else x
    if iters_deep is None:
        iters_deep = torch.zeros((batch, L // B), dtype=torch.int32, device=z.device)
    if iters_shallow is None:
        iters_shallow = torch.zeros((T, batch, L // F), dtype=torch.int32, device=z.device)
    hs = (ctypes.c_void_p * T)(*[m.handle for m in shallow])
    ds = (ctypes.c_int * T)(*shallow_dirs)
    s2 = stream_shallow if stream_shallow is not None else (stream if stream is not None else torch.cuda.current_stream())
    _check(lib().flow_pipeline_inverse(deep.handle, hs, ds, T, _ptr(z), batch, L, B, float(tau), int(max_iter_deep),
                                       int(max_iter_shallow), int(bool(warm_start)), int(group), _ptr(x),
                                       _ptr(iters_deep), _ptr(iters_shallow), _ptr(ws_deep), ws_deep.numel(),
                                       _ptr(ws_shallow), ws_shallow.numel(), _stream(stream), _stream(s2)),
           "flow_pipeline_inverse")
    return x, iters_deep, iters_shallow


def af_denoise(model: AFModel, x_noisy: torch.Tensor, sigma: float, ws: torch.Tensor | None = None,
               x: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """x = x_noisy + sigma * s_phi(x_noisy) with the denoiser `model` (created with denoiser=True)."""
    batch, L, _ = x_noisy.shape
    ws = model.workspace(batch, L, device=x_noisy.device) if ws is None else ws
    x = torch.empty_like(x_noisy) if x is None else x
    _check(lib().af_denoise(model.handle, _ptr(x_noisy), batch, L, float(sigma), _ptr(x), _ptr(ws), ws.numel(),
                            _stream(stream)), "af_denoise")
    return x


def af_inverse_jacobi_stream(model: AFModel, z: torch.Tensor, window: int, overlap: int, tau: float, max_iter: int,
                             warm_start: bool, ws: torch.Tensor | None = None, x: torch.Tensor | None = None,
                             iters: torch.Tensor | None = None, stream=None):
    """Streaming block-Jacobi inverse in windows of `window` frames overlapping by `overlap`;
    returns (x, iters [batch, n_frames])."""
    batch, L, _ = z.shape
    F = model.shape.frame_len
    n_frames = L // F
    if ws is None:
        n = int(lib().af_stream_workspace_bytes(model.handle, batch, window))
        if n == 0:
            raise AFError(AF_ERR_ARG, "af_stream_workspace_bytes")
        ws = torch.empty(n, dtype=torch.uint8, device=z.device)
    x = torch.empty_like(z) if x is None else x
    iters = torch.zeros((batch, n_frames), dtype=torch.int32, device=z.device) if iters is None else iters
    _check(lib().af_inverse_jacobi_stream(model.handle, _ptr(z), batch, n_frames, window, overlap, float(tau),
                                          int(max_iter), int(bool(warm_start)), _ptr(x), _ptr(iters), _ptr(ws),
                                          ws.numel(), _stream(stream)), "af_inverse_jacobi_stream")
    return x, iters
