"""Exact IO-aware attention for B200 (sm_100a).

The compute lives in ``libfa.so`` (C ABI, ``include/fa.h``); this package is
its Python binding.  Functions named like the C entry points take torch CUDA
tensors and pass their pointers through unchanged; PyTorch only provides the
device memory and the stream.  ``attention_forward`` / ``attention_backward``
additionally allocate the outputs (and the backward workspace) with torch.
"""
from __future__ import annotations

import ctypes

import torch

from ._lib import FA_OK, FAError, LIB_PATH, STATUS_CODES, STATUS_NAMES, check, lib, strerror

__all__ = [
    "FAError", "LIB_PATH", "fa_fwd", "fa_fwd_fp8", "fa_bwd", "fa_bwd_deterministic", "fa_bwd_workspace_size",
    "fa_bwd_events", "fa_fwd_plan", "fa_bwd_fp8", "fa_bwd_fp8_workspace_size", "attention_backward_fp8", "fa_get_device_status", "fa_device_status", "fa_fwd_decode", "fa_fwd_decode_workspace_size", "attention_decode",
    "fa_fwd_standard", "fa_fwd_standard_workspace_size", "attention_forward_standard",
    "fa_watchdog_selftest", "attention_forward", "attention_backward", "attention_forward_fp8", "lib",
    "STATUS_NAMES", "STATUS_CODES", "strerror",
]


def _stream_ptr(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


def _ptr(t) -> int:
    return 0 if t is None else int(t.data_ptr())


def _shape(q):
    if q.dim() != 4:
        raise ValueError("tensors must be [B, H, N, d]")
    return tuple(int(x) for x in q.shape)


def _check_tensors(ref_shape, dtype, *ts):
    for t in ts:
        if t.device.type != "cuda":
            raise ValueError("tensors must be CUDA tensors")
        if tuple(t.shape) != ref_shape or t.dtype != dtype or not t.is_contiguous():
            raise ValueError(f"expected contiguous {dtype} {ref_shape}, got {t.dtype} {tuple(t.shape)}")


def fa_fwd(q, k, v, o, lse, scale: float, causal: bool, stream=None) -> None:
    """O, LSE <- attention(q, k, v) (bf16 in/out, LSE fp32 [B,H,N])."""
    B, H, N, d = _shape(q)
    _check_tensors((B, H, N, d), torch.bfloat16, q, k, v, o)
    _check_tensors((B, H, N), torch.float32, lse)
    check(lib.fa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d, float(scale), int(bool(causal)),
                     _stream_ptr(stream)))


def fa_fwd_fp8(q8, k8, v8, q_descale, k_descale, v_descale, o, lse, scale: float, causal: bool,
               stream=None) -> None:
    """Forward with e4m3 inputs (uint8 or float8_e4m3fn tensors) and per-tensor descales."""
    B, H, N, d = _shape(q8)
    for t in (q8, k8, v8):
        if t.dtype not in (torch.uint8, torch.float8_e4m3fn) or tuple(t.shape) != (B, H, N, d) \
                or not t.is_contiguous() or t.device.type != "cuda":
            raise ValueError("e4m3 inputs must be contiguous CUDA uint8/float8_e4m3fn [B,H,N,d]")
    _check_tensors((B, H, N, d), torch.bfloat16, o)
    _check_tensors((B, H, N), torch.float32, lse)
    check(lib.fa_fwd_fp8(_ptr(q8), _ptr(k8), _ptr(v8), float(q_descale), float(k_descale), float(v_descale),
                         _ptr(o), _ptr(lse), B, H, N, d, float(scale), int(bool(causal)), _stream_ptr(stream)))


def fa_bwd_workspace_size(B: int, H: int, N: int, d: int) -> int:
    n = int(lib.fa_bwd_workspace_size(B, H, N, d))
    if n == ctypes.c_size_t(-1).value:
        raise FAError(1, "invalid shape for fa_bwd_workspace_size")
    return n


def fa_bwd(q, k, v, o, do, lse, dq, dk, dv, scale: float, causal: bool, workspace, stream=None) -> None:
    """dQ, dK, dV <- backward of attention; workspace is a CUDA uint8 tensor."""
    B, H, N, d = _shape(q)
    _check_tensors((B, H, N, d), torch.bfloat16, q, k, v, o, do, dq, dk, dv)
    _check_tensors((B, H, N), torch.float32, lse)
    wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    check(lib.fa_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv),
                     B, H, N, d, float(scale), int(bool(causal)), _ptr(workspace), wbytes, _stream_ptr(stream)))


def fa_bwd_events(q, k, v, o, do, lse, dq, dk, dv, scale: float, causal: bool, workspace, events,
                  stream=None) -> None:
    """fa_bwd that also records four torch.cuda.Event objects on the stream:
    before the preprocess, before and after the main kernel, after the last launch."""
    B, H, N, d = _shape(q)
    _check_tensors((B, H, N, d), torch.bfloat16, q, k, v, o, do, dq, dk, dv)
    _check_tensors((B, H, N), torch.float32, lse)
    if len(events) != 4:
        raise ValueError("fa_bwd_events takes four events")
    for e in events:
        if int(e.cuda_event) == 0:         # torch creates the CUDA event at its first record
            e.record(torch.cuda.current_stream() if stream is None else stream)
    arr = (ctypes.c_void_p * 4)(*(int(e.cuda_event) for e in events))
    wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    check(lib.fa_bwd_events(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv),
                            B, H, N, d, float(scale), int(bool(causal)), _ptr(workspace), wbytes, arr,
                            _stream_ptr(stream)))


def fa_bwd_fp8_workspace_size(B: int, H: int, N: int, d: int) -> int:
    n = int(lib.fa_bwd_fp8_workspace_size(B, H, N, d))
    if n == ctypes.c_size_t(-1).value:
        raise FAError(1, "invalid shape for fa_bwd_fp8_workspace_size (d must be 128)")
    return n


def _check_e4m3(shape, *ts):
    for t in ts:
        if t.dtype not in (torch.uint8, torch.float8_e4m3fn) or tuple(t.shape) != shape \
                or not t.is_contiguous() or t.device.type != "cuda":
            raise ValueError("e4m3 inputs must be contiguous CUDA uint8/float8_e4m3fn [B,H,N,d]")


def fa_bwd_fp8(q8, k8, v8, q_descale, k_descale, v_descale, o, do, lse, dq, dk, dv, scale: float, causal: bool,
               workspace, stream=None) -> None:
    """dQ, dK, dV (real units) <- backward of the e4m3 forward; workspace is a CUDA uint8 tensor."""
    B, H, N, d = _shape(q8)
    _check_e4m3((B, H, N, d), q8, k8, v8)
    _check_tensors((B, H, N, d), torch.bfloat16, o, do, dq, dk, dv)
    _check_tensors((B, H, N), torch.float32, lse)
    wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    check(lib.fa_bwd_fp8(_ptr(q8), _ptr(k8), _ptr(v8), float(q_descale), float(k_descale), float(v_descale),
                         _ptr(o), _ptr(do), _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv), B, H, N, d, float(scale),
                         int(bool(causal)), _ptr(workspace), wbytes, _stream_ptr(stream)))


def fa_fwd_plan(B: int, H: int, N: int, d: int, causal: bool):
    """(ctas, items, pair_items) of the forward's launch for this shape."""
    c, it, pi = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    check(lib.fa_fwd_plan(B, H, N, d, int(bool(causal)), ctypes.byref(c), ctypes.byref(it), ctypes.byref(pi)))
    return c.value, it.value, pi.value


def fa_bwd_deterministic(q, k, v, o, do, lse, dq, dk, dv, scale: float, causal: bool, workspace,
                         stream=None) -> None:
    """As fa_bwd, with dQ from a separate atomic-free pass: bit-reproducible results."""
    B, H, N, d = _shape(q)
    _check_tensors((B, H, N, d), torch.bfloat16, q, k, v, o, do, dq, dk, dv)
    _check_tensors((B, H, N), torch.float32, lse)
    wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    check(lib.fa_bwd_deterministic(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse), _ptr(dq), _ptr(dk),
                                   _ptr(dv), B, H, N, d, float(scale), int(bool(causal)), _ptr(workspace), wbytes,
                                   _stream_ptr(stream)))


def fa_fwd_decode_workspace_size(B: int, H: int, Nq: int, Nk: int, d: int) -> int:
    n = int(lib.fa_fwd_decode_workspace_size(B, H, Nq, Nk, d))
    if n == ctypes.c_size_t(-1).value:
        raise FAError(1, "invalid shape for fa_fwd_decode_workspace_size")
    return n


def fa_fwd_decode(q, k, v, o, lse, scale: float, causal: bool, workspace, stream=None) -> None:
    """O, LSE <- attention of q [B,H,Nq,d] (Nq <= 16) over a KV cache k, v [B,H,Nk,d]."""
    B, H, Nq, d = _shape(q)
    Nk = int(k.shape[2])
    _check_tensors((B, H, Nk, d), torch.bfloat16, k, v)
    _check_tensors((B, H, Nq, d), torch.bfloat16, q, o)
    _check_tensors((B, H, Nq), torch.float32, lse)
    wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    check(lib.fa_fwd_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, Nq, Nk, d, float(scale),
                            int(bool(causal)), _ptr(workspace), wbytes, _stream_ptr(stream)))


def attention_decode(q, k, v, scale: float | None = None, causal: bool = False, workspace=None, stream=None):
    """Allocates O, LSE (and the split workspace unless given) with torch and runs fa_fwd_decode."""
    B, H, Nq, d = _shape(q)
    Nk = int(k.shape[2])
    o = torch.empty_like(q)
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = torch.empty(max(16, fa_fwd_decode_workspace_size(B, H, Nq, Nk, d)), dtype=torch.uint8,
                                device=q.device)
    fa_fwd_decode(q, k, v, o, lse, _default_scale(d) if scale is None else scale, causal, workspace, stream)
    return o, lse


def fa_fwd_standard_workspace_size(B: int, H: int, N: int, d: int) -> int:
    n = int(lib.fa_fwd_standard_workspace_size(B, H, N, d))
    if n == ctypes.c_size_t(-1).value:
        raise FAError(1, "invalid shape for fa_fwd_standard_workspace_size")
    return n


def fa_fwd_standard(q, k, v, o, lse, scale: float, causal: bool, workspace, stream=None) -> None:
    """Standard attention with S and P materialised in the workspace (the IO baseline)."""
    B, H, N, d = _shape(q)
    _check_tensors((B, H, N, d), torch.bfloat16, q, k, v, o)
    _check_tensors((B, H, N), torch.float32, lse)
    wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    check(lib.fa_fwd_standard(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d, float(scale),
                              int(bool(causal)), _ptr(workspace), wbytes, _stream_ptr(stream)))


def attention_forward_standard(q, k, v, scale: float | None = None, causal: bool = False, workspace=None,
                               stream=None):
    B, H, N, d = _shape(q)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = torch.empty(max(256, fa_fwd_standard_workspace_size(B, H, N, d)), dtype=torch.uint8,
                                device=q.device)
    fa_fwd_standard(q, k, v, o, lse, _default_scale(d) if scale is None else scale, causal, workspace, stream)
    return o, lse


def fa_device_status(stream=None):
    """(status, where) of the device status word; synchronises the stream and clears it."""
    where = ctypes.c_uint32(0)
    st = lib.fa_device_status(_stream_ptr(stream), ctypes.byref(where))
    return st, int(where.value)


def fa_watchdog_selftest(limit_us: int, stream=None) -> None:
    check(lib.fa_watchdog_selftest(int(limit_us), _stream_ptr(stream)))


def _default_scale(d: int) -> float:
    return d ** -0.5


def attention_forward(q, k, v, scale: float | None = None, causal: bool = False, stream=None):
    """Allocates O (bf16) and LSE (fp32) with torch and runs fa_fwd."""
    B, H, N, d = _shape(q)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    fa_fwd(q, k, v, o, lse, _default_scale(d) if scale is None else scale, causal, stream)
    return o, lse


def attention_forward_fp8(q8, k8, v8, q_descale, k_descale, v_descale, scale: float | None = None,
                          causal: bool = False, stream=None):
    B, H, N, d = _shape(q8)
    o = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=q8.device)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q8.device)
    fa_fwd_fp8(q8, k8, v8, q_descale, k_descale, v_descale, o, lse,
               _default_scale(d) if scale is None else scale, causal, stream)
    return o, lse


def attention_backward(q, k, v, o, do, lse, scale: float | None = None, causal: bool = False, workspace=None,
                       stream=None, deterministic: bool = False):
    """Allocates dQ, dK, dV (and the workspace unless given) with torch and runs
    fa_bwd (or fa_bwd_deterministic)."""
    B, H, N, d = _shape(q)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    if workspace is None:
        workspace = torch.empty(max(1, fa_bwd_workspace_size(B, H, N, d)), dtype=torch.uint8, device=q.device)
    fn = fa_bwd_deterministic if deterministic else fa_bwd
    fn(q, k, v, o, do, lse, dq, dk, dv, _default_scale(d) if scale is None else scale, causal, workspace, stream)
    return dq, dk, dv


def attention_backward_fp8(q8, k8, v8, q_descale, k_descale, v_descale, o, do, lse, scale: float | None = None,
                           causal: bool = False, workspace=None, stream=None):
    """(dQ, dK, dV) bf16 of the e4m3 forward, allocating outputs and workspace with torch."""
    B, H, N, d = _shape(q8)
    dq, dk, dv = (torch.empty((B, H, N, d), dtype=torch.bfloat16, device=q8.device) for _ in range(3))
    if workspace is None:
        workspace = torch.empty(max(256, fa_bwd_fp8_workspace_size(B, H, N, d)), dtype=torch.uint8, device=q8.device)
    fa_bwd_fp8(q8, k8, v8, q_descale, k_descale, v_descale, o, do, lse, dq, dk, dv,
               _default_scale(d) if scale is None else scale, causal, workspace, stream)
    return dq, dk, dv
