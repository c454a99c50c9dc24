"""Thin ctypes binding over ``libattn.so`` (C ABI in ``include/attn.h``).

Argument marshalling only: torch tensors provide device memory and streams;
every step of the computation runs in the library's CUDA kernels.  There is
no CPU path: if the library is missing or a GPU is absent, calls raise.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

__all__ = ["ATTN_BF16", "ATTN_MXFP8", "ATTN_NVFP4", "AttnError", "lib", "workspace_size", "attn_fwd",
           "attn_fwd_noalloc", "attn_quantize_mxfp8", "attn_get_device_error", "status_string",
           "make_workspace", "attn_timing_enable", "attn_timing_read", "bwd_workspace_size",
           "make_bwd_workspace", "attn_bwd", "attn_quantize_mxfp8_rotated",
           "attn_fwd_incoherent", "attn_quantize_nvfp4", "LIB_PATH", "EXPORTED_SYMBOLS"]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libattn.so")

ATTN_BF16 = 0
ATTN_MXFP8 = 1
ATTN_NVFP4 = 2

STATUS = {
    0: "ATTN_OK", 1: "ATTN_ERR_INVALID_ARG", 2: "ATTN_ERR_UNSUPPORTED", 3: "ATTN_ERR_ALIGNMENT",
    4: "ATTN_ERR_WORKSPACE", 5: "ATTN_ERR_BAD_SEQLENS", 6: "ATTN_ERR_TIMEOUT", 7: "ATTN_ERR_CUDA",
}

EXPORTED_SYMBOLS = ("attn_workspace_size", "attn_fwd", "attn_quantize_mxfp8",
                    "attn_get_device_error", "attn_status_string", "attn_abi_version",
                    "attn_fwd_noalloc", "attn_timing_enable", "attn_timing_read",
                    "attn_bwd_workspace_size", "attn_bwd", "attn_quantize_mxfp8_rotated",
                    "attn_fwd_incoherent", "attn_quantize_nvfp4")


class AttnError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {STATUS.get(code, code)}")
        self.code = code


class _Shape(ctypes.Structure):
    _fields_ = [("total_tokens", ctypes.c_int32), ("num_seqs", ctypes.c_int32),
                ("num_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("max_seqlen", ctypes.c_int32)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load the library (once).  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m exact_tiled_attention_39_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
        L.attn_workspace_size.argtypes = [ctypes.POINTER(_Shape), ctypes.c_int]
        L.attn_workspace_size.restype = sz
        L.attn_fwd.argtypes = [vp, vp, vp, vp, vp, vp, ctypes.c_int, ctypes.c_float, ctypes.c_int,
                               vp, ctypes.POINTER(_Shape), vp, sz]
        L.attn_fwd.restype = ctypes.c_int
        L.attn_quantize_mxfp8.argtypes = [vp, vp, vp, i64, i32, vp]
        L.attn_quantize_mxfp8.restype = ctypes.c_int
        L.attn_get_device_error.argtypes = [vp, vp, ctypes.POINTER(i32)]
        L.attn_get_device_error.restype = ctypes.c_int
        L.attn_status_string.argtypes = [ctypes.c_int]
        L.attn_status_string.restype = ctypes.c_char_p
        L.attn_abi_version.argtypes = []
        L.attn_abi_version.restype = i32
        L.attn_timing_enable.argtypes = [i32]
        L.attn_timing_enable.restype = ctypes.c_int
        L.attn_timing_read.argtypes = [ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_float)]
        L.attn_timing_read.restype = ctypes.c_int
        L.attn_bwd_workspace_size.argtypes = [ctypes.POINTER(_Shape), ctypes.c_int]
        L.attn_bwd_workspace_size.restype = sz
        L.attn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_int,
                               ctypes.c_float, ctypes.c_int, vp, ctypes.POINTER(_Shape), vp, sz]
        L.attn_bwd.restype = ctypes.c_int
        L.attn_quantize_mxfp8_rotated.argtypes = [vp, vp, vp, vp, i64, i32, vp]
        L.attn_quantize_mxfp8_rotated.restype = ctypes.c_int
        L.attn_fwd_incoherent.argtypes = [vp, vp, vp, vp, vp, vp, ctypes.c_int, ctypes.c_float,
                                          vp, vp, ctypes.POINTER(_Shape), vp, sz]
        L.attn_fwd_incoherent.restype = ctypes.c_int
        L.attn_quantize_nvfp4.argtypes = [vp, vp, vp, i64, i32, vp]
        L.attn_quantize_nvfp4.restype = ctypes.c_int
        _lib = L
    return _lib


def status_string(code: int) -> str:
    return lib().attn_status_string(code).decode()


@dataclass(frozen=True)
class Shape:
    total_tokens: int
    num_seqs: int
    num_heads: int
    head_dim: int
    max_seqlen: int

    def c(self) -> _Shape:
        return _Shape(self.total_tokens, self.num_seqs, self.num_heads, self.head_dim,
                      self.max_seqlen)


def workspace_size(shape: Shape, dtype: int = ATTN_BF16) -> int:
    s = shape.c()
    return int(lib().attn_workspace_size(ctypes.byref(s), dtype))


def make_workspace(shape: Shape, dtype: int = ATTN_BF16, device=None) -> torch.Tensor:
    n = workspace_size(shape, dtype)
    if n == 0:
        raise AttnError(1, "attn_workspace_size")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream, device) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def attn_fwd(q, k, v, cu_seqlens, out, lse, causal: bool, scale: float, dtype: int = ATTN_BF16,
             stream=None, workspace=None, max_seqlen: int | None = None,
             num_seqs: int | None = None):
    """Run the forward through the C ABI.  q, k, v, out: bf16 [T, H, d]
    (contiguous, CUDA); lse: fp32 [H, T]; cu_seqlens: int32 CUDA tensor or
    None (dense: ``num_seqs`` documents of ``max_seqlen`` tokens).  With
    cu_seqlens, ``max_seqlen`` must bound every document length (a longer
    one is reported by the device as ATTN_ERR_BAD_SEQLENS).  Returns the
    workspace used (allocated if not given)."""
    shape = _check_fwd_args(q, k, v, out, lse, cu_seqlens, max_seqlen, num_seqs)
    with torch.cuda.device(q.device):
        if workspace is None:
            workspace = make_workspace(shape, dtype, q.device)
        elif not workspace.is_cuda or workspace.device != q.device:
            raise ValueError("workspace must be on the same CUDA device as q")
        s = shape.c()
        rc = lib().attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens), _ptr(out), _ptr(lse),
                            int(bool(causal)), float(scale), int(dtype),
                            _stream_handle(stream, q.device), ctypes.byref(s), _ptr(workspace),
                            workspace.numel())
    if rc != 0:
        raise AttnError(rc, "attn_fwd")
    return workspace


def attn_fwd_incoherent(q, k, v, cu_seqlens, out, lse, causal: bool, scale: float, signs,
                        stream=None, workspace=None, max_seqlen: int | None = None,
                        num_seqs: int | None = None):
    """The MXFP8 forward with incoherent processing (``attn_fwd_incoherent``):
    Q and K rotated by diag(signs) H_d before quantisation, the softmax scale
    divided by d inside the call.  signs: fp32 [d] of +-1 on q's device.
    Other arguments as ``attn_fwd``; the workspace is the MXFP8 one."""
    shape = _check_fwd_args(q, k, v, out, lse, cu_seqlens, max_seqlen, num_seqs)
    if (signs.dtype != torch.float32 or not signs.is_cuda or not signs.is_contiguous()
            or tuple(signs.shape) != (q.shape[2],) or signs.device != q.device):
        raise ValueError(f"signs must be a contiguous fp32 tensor of shape [d] on {q.device}")
    with torch.cuda.device(q.device):
        if workspace is None:
            workspace = make_workspace(shape, ATTN_MXFP8, q.device)
        elif not workspace.is_cuda or workspace.device != q.device:
            raise ValueError("workspace must be on the same CUDA device as q")
        s = shape.c()
        rc = lib().attn_fwd_incoherent(_ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens), _ptr(out),
                                       _ptr(lse), int(bool(causal)), float(scale), _ptr(signs),
                                       _stream_handle(stream, q.device), ctypes.byref(s),
                                       _ptr(workspace), workspace.numel())
    if rc != 0:
        raise AttnError(rc, "attn_fwd_incoherent")
    return workspace


def _check_fwd_args(q, k, v, out, lse, cu_seqlens, max_seqlen, num_seqs) -> Shape:
    """Checks shared by the forward entry points; returns the problem shape.
    Every tensor must be on q's CUDA device: the library launches on the
    device that is current during the call, which the callers set to q's."""
    if q.dim() != 3:
        raise ValueError("q must have shape [T, H, d]")
    T, H, d = q.shape
    for name, t in (("q", q), ("k", k), ("v", v), ("out", out)):
        if (t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous()
                or t.shape != q.shape or t.device != q.device):
            raise ValueError(f"{name} must be a contiguous bf16 tensor of shape "
                             f"{tuple(q.shape)} on {q.device}")
    if (lse.dtype != torch.float32 or not lse.is_cuda or not lse.is_contiguous()
            or tuple(lse.shape) != (H, T) or lse.device != q.device):
        raise ValueError(f"lse must be a contiguous fp32 tensor of shape [H, T] on {q.device}")
    return _doc_shape(q, cu_seqlens, max_seqlen, num_seqs)


def _doc_shape(q, cu_seqlens, max_seqlen, num_seqs) -> Shape:
    T, H, d = q.shape
    if cu_seqlens is not None:
        if (cu_seqlens.dtype != torch.int32 or not cu_seqlens.is_cuda
                or not cu_seqlens.is_contiguous() or cu_seqlens.dim() != 1
                or cu_seqlens.device != q.device):
            raise ValueError(f"cu_seqlens must be a contiguous 1-D int32 tensor on {q.device}")
        ns = cu_seqlens.numel() - 1
        if max_seqlen is None:
            raise ValueError("max_seqlen is required with cu_seqlens (no host sync is done)")
    else:
        ns = num_seqs if num_seqs is not None else 1
        if max_seqlen is None:
            max_seqlen = T // max(ns, 1)
    return Shape(T, ns, H, d, int(max_seqlen))


def bwd_workspace_size(shape: Shape, dtype: int = ATTN_BF16) -> int:
    s = shape.c()
    return int(lib().attn_bwd_workspace_size(ctypes.byref(s), dtype))


def make_bwd_workspace(shape: Shape, device=None, dtype: int = ATTN_BF16) -> torch.Tensor:
    n = bwd_workspace_size(shape, dtype)
    if n == 0:
        raise AttnError(1, "attn_bwd_workspace_size")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def attn_bwd(q, k, v, out, dout, lse, cu_seqlens, dq, dk, dv, causal: bool, scale: float,
             stream=None, workspace=None, max_seqlen: int | None = None,
             num_seqs: int | None = None, dtype: int = ATTN_BF16):
    """Gradients of the forward through the C ABI (``attn_bwd``): q, k, v,
    out (the forward's output), dout: bf16 [T, H, d]; lse: fp32 [H, T] from
    the forward; dq, dk, dv: bf16 [T, H, d], written.  Same document rules
    as ``attn_fwd``; dtype ATTN_MXFP8 differentiates the MXFP8 forward (out
    and lse from it).  Returns the workspace used (allocated if not given)."""
    T, H, d = q.shape
    for name, t in (("q", q), ("k", k), ("v", v), ("out", out), ("dout", dout), ("dq", dq),
                    ("dk", dk), ("dv", dv)):
        if (t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous()
                or t.shape != q.shape or t.device != q.device):
            raise ValueError(f"{name} must be a contiguous bf16 tensor of shape "
                             f"{tuple(q.shape)} on {q.device}")
    if (lse.dtype != torch.float32 or not lse.is_cuda or not lse.is_contiguous()
            or tuple(lse.shape) != (H, T) or lse.device != q.device):
        raise ValueError(f"lse must be a contiguous fp32 tensor of shape [H, T] on {q.device}")
    shape = _doc_shape(q, cu_seqlens, max_seqlen, num_seqs)
    with torch.cuda.device(q.device):
        if workspace is None:
            workspace = make_bwd_workspace(shape, q.device, dtype)
        elif not workspace.is_cuda or workspace.device != q.device:
            raise ValueError("workspace must be on the same CUDA device as q")
        s = shape.c()
        rc = lib().attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(dout), _ptr(lse),
                            _ptr(cu_seqlens), _ptr(dq), _ptr(dk), _ptr(dv), int(bool(causal)),
                            float(scale), int(dtype), _stream_handle(stream, q.device),
                            ctypes.byref(s), _ptr(workspace), workspace.numel())
    if rc != 0:
        raise AttnError(rc, "attn_bwd")
    return workspace


def _check_quant_args(x, codes, scales, code_bytes: int, scale_bytes: int, signs=None):
    """Checks shared by the quantiser entry points; returns (rows, cols).
    x: contiguous bf16 CUDA tensor whose last dimension is cols; codes and
    scales: contiguous uint8 tensors on x's device holding exactly
    code_bytes and scale_bytes per row (the library writes that many and
    cannot see the buffers' sizes); signs, if given: fp32 [cols]."""
    if x.dtype != torch.bfloat16 or not x.is_cuda or not x.is_contiguous() or x.dim() < 1:
        raise ValueError("x must be a contiguous bf16 CUDA tensor")
    cols = x.shape[-1]
    rows = x.numel() // cols if cols > 0 else 0
    for name, t, per_row in (("codes", codes, code_bytes), ("scales", scales, scale_bytes)):
        if (t.dtype != torch.uint8 or not t.is_cuda or not t.is_contiguous()
                or t.device != x.device or t.numel() != rows * per_row):
            raise ValueError(f"{name} must be a contiguous uint8 tensor of {rows} x {per_row} "
                             f"bytes on {x.device}")
    if signs is not None and (signs.dtype != torch.float32 or not signs.is_cuda
                              or not signs.is_contiguous() or tuple(signs.shape) != (cols,)
                              or signs.device != x.device):
        raise ValueError(f"signs must be a contiguous fp32 tensor of shape [{cols}] on {x.device}")
    return rows, cols


def attn_quantize_mxfp8(x, codes, scales, stream=None):
    """E4M3 + E8M0 quantisation of a bf16 [rows, cols] CUDA tensor (any
    leading shape; the last dimension is ``cols``, a multiple of 32): codes
    uint8 [rows, cols], scales uint8 [rows, cols / 32] (E8M0)."""
    cols = x.shape[-1] if x.dim() > 0 else 0
    rows, cols = _check_quant_args(x, codes, scales, cols, cols // 32)
    with torch.cuda.device(x.device):
        rc = lib().attn_quantize_mxfp8(_ptr(x), _ptr(codes), _ptr(scales), rows, cols,
                                       _stream_handle(stream, x.device))
    if rc != 0:
        raise AttnError(rc, "attn_quantize_mxfp8")


def attn_quantize_nvfp4(x, codes, scales, stream=None):
    """NVFP4 quantisation of a bf16 [rows, cols] CUDA tensor (any leading
    shape; cols a multiple of 16): codes uint8 [rows, cols / 2] (two E2M1
    codes per byte, low nibble first), scales uint8 [rows, cols / 16]
    (unsigned E4M3)."""
    cols = x.shape[-1] if x.dim() > 0 else 0
    rows, cols = _check_quant_args(x, codes, scales, cols // 2, cols // 16)
    with torch.cuda.device(x.device):
        rc = lib().attn_quantize_nvfp4(_ptr(x), _ptr(codes), _ptr(scales), rows, cols,
                                       _stream_handle(stream, x.device))
    if rc != 0:
        raise AttnError(rc, "attn_quantize_nvfp4")


def attn_quantize_mxfp8_rotated(x, signs, codes, scales, stream=None):
    """Incoherent processing then MXFP8 quantisation of a bf16 [rows, cols]
    CUDA tensor (cols 64 or 128; any leading shape): signs fp32 [cols] (+-1)
    on the device; codes uint8 [rows, cols], scales uint8 [rows, cols / 32]
    (``attn_quantize_mxfp8_rotated``)."""
    cols = x.shape[-1] if x.dim() > 0 else 0
    rows, cols = _check_quant_args(x, codes, scales, cols, cols // 32, signs=signs)
    with torch.cuda.device(x.device):
        rc = lib().attn_quantize_mxfp8_rotated(_ptr(x), _ptr(signs), _ptr(codes), _ptr(scales),
                                               rows, cols, _stream_handle(stream, x.device))
    if rc != 0:
        raise AttnError(rc, "attn_quantize_mxfp8_rotated")


def attn_timing_enable(enable: bool) -> None:
    """Turn per-call kernel timing on or off (``attn_timing_enable``)."""
    rc = lib().attn_timing_enable(int(bool(enable)))
    if rc != 0:
        raise AttnError(rc, "attn_timing_enable")


def attn_timing_read() -> tuple[float, float]:
    """(attention kernel ms, pre-pass ms) of the most recent timed call;
    waits for that call's events (``attn_timing_read``)."""
    a, b = ctypes.c_float(0.0), ctypes.c_float(0.0)
    rc = lib().attn_timing_read(ctypes.byref(a), ctypes.byref(b))
    if rc != 0:
        raise AttnError(rc, "attn_timing_read")
    return float(a.value), float(b.value)


def attn_get_device_error(workspace, stream=None) -> int:
    if not workspace.is_cuda:
        raise ValueError("workspace must be a CUDA tensor")
    v = ctypes.c_int32(0)
    with torch.cuda.device(workspace.device):
        rc = lib().attn_get_device_error(_ptr(workspace),
                                         _stream_handle(stream, workspace.device), ctypes.byref(v))
    if rc != 0:
        raise AttnError(rc, "attn_get_device_error")
    return int(v.value)


def attn_fwd_noalloc(q, k, v, cu_seqlens, out, lse, causal: bool, scale: float, stream=None,
                     max_seqlen: int | None = None, num_seqs: int | None = None) -> None:
    """The bf16 forward through ``attn_fwd_noalloc``: no workspace is passed
    and nothing is allocated (the library's fixed 1 MiB device scratch is
    used).  For callers that cannot allocate device memory; calls that
    overlap on the GPU race on the shared scratch."""
    L = lib()
    fn = L.attn_fwd_noalloc
    vp = ctypes.c_void_p
    fn.argtypes = [vp, vp, vp, vp, vp, vp, ctypes.c_int, ctypes.c_float, vp,
                   ctypes.POINTER(_Shape)]
    fn.restype = ctypes.c_int
    s = _check_fwd_args(q, k, v, out, lse, cu_seqlens, max_seqlen, num_seqs).c()
    # The library looks up its scratch on the current device: make that q's.
    with torch.cuda.device(q.device):
        rc = fn(_ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens), _ptr(out), _ptr(lse),
                int(bool(causal)), float(scale), _stream_handle(stream, q.device),
                ctypes.byref(s))
    if rc != 0:
        raise AttnError(rc, "attn_fwd_noalloc")
