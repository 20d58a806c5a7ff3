"""Thin Python binding of libgdn.so (the C ABI in include/gdn.h).

Argument marshalling only: tensors are checked for device, dtype, shape and
contiguity, turned into raw pointers and handed to the C entry points of the
same names, on the current torch CUDA stream.  Every step of the computation
runs in the library's CUDA kernels; there is no other implementation to fall
back to, so a missing or unloadable libgdn.so raises immediately.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgdn.so")
HEADER = os.path.join(os.path.dirname(_PKG), "include", "gdn.h")

GDN_OK, GDN_ERR_INVALID_ARG, GDN_ERR_UNSUPPORTED, GDN_ERR_CUDA, GDN_ERR_WORKSPACE = 0, 1, 2, 3, 5
GDN_F32, GDN_BF16 = 0, 1
CHUNK = 64

_lib = None


class GdnError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        msg = "%s failed: %s" % (what, status_string(status))
        if status == GDN_ERR_CUDA:
            msg += " (" + _load().gdn_last_cuda_error().decode() + ")"
        super().__init__(msg)


def _load():
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError("libgdn.so is not built (%s); run python -m "
                          "linear_attention_vlm_b200.build" % LIB_PATH)
    lib = ctypes.CDLL(LIB_PATH)
    vp, fp, sz = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t
    i32, i64 = ctypes.c_int, ctypes.c_int64
    lib.gdn_prefill_workspace_size.argtypes = [i32, i64, i32, i32, i32, i32, i32]
    lib.gdn_prefill_workspace_size.restype = sz
    lib.gdn_prefill_kernel_count.argtypes = [i32, i64, i32, i32, i32, i32, i32, i32]
    lib.gdn_prefill_kernel_count.restype = i32
    lib.gdn_prefill.argtypes = [vp, vp, vp, fp, fp, fp, vp, fp, vp, i32, i64, i32, i32, i32,
                                i32, i32, vp, sz, vp]
    lib.gdn_prefill.restype = i32
    lib.gdn_prefill_noalloc.argtypes = [vp, vp, vp, fp, fp, fp, vp, fp, vp, i32, i64, i32, i32,
                                        i32, i32, i32, vp]
    lib.gdn_prefill_noalloc.restype = i32
    lib.gdn_decode_step.argtypes = [vp, vp, vp, fp, fp, fp, fp, vp, i32, i32, i32, i32, i32, vp]
    lib.gdn_decode_step.restype = i32
    lib.gdn_status_string.argtypes = [i32]
    lib.gdn_status_string.restype = ctypes.c_char_p
    lib.gdn_last_cuda_error.argtypes = []
    lib.gdn_last_cuda_error.restype = ctypes.c_char_p
    _lib = lib
    return lib


def library() -> ctypes.CDLL:
    """The loaded libgdn.so (raises if it is missing)."""
    return _load()


def declared_symbols():
    """Names of the functions include/gdn.h declares."""
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(gdn_[a-z0-9_]+)\s*\(", src)))


def status_string(status: int) -> str:
    return _load().gdn_status_string(int(status)).decode()


def _dtype_code(t: torch.dtype) -> int:
    if t == torch.float32:
        return GDN_F32
    if t == torch.bfloat16:
        return GDN_BF16
    raise TypeError("q/k/v must be float32 or bfloat16, got %s" % t)


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return t.data_ptr() or None


def _stream(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def gdn_prefill_workspace_size(num_seqs: int, total_tokens: int, H: int, dk: int, dv: int,
                               chunk: int = CHUNK, dtype: torch.dtype = torch.bfloat16) -> int:
    return int(_load().gdn_prefill_workspace_size(num_seqs, total_tokens, H, dk, dv, chunk,
                                                  _dtype_code(dtype)))


def gdn_prefill_kernel_count(num_seqs: int, total_tokens: int, H: int, dk: int, dv: int,
                             chunk: int = CHUNK, dtype: torch.dtype = torch.bfloat16,
                             packed: bool = False) -> int:
    return int(_load().gdn_prefill_kernel_count(num_seqs, total_tokens, H, dk, dv, chunk,
                                                _dtype_code(dtype), int(packed)))


def gdn_prefill(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor,
                beta: torch.Tensor, state_in: Optional[torch.Tensor] = None,
                cu_seqlens: Optional[torch.Tensor] = None, *, num_seqs: Optional[int] = None,
                out: Optional[torch.Tensor] = None, state_out: Optional[torch.Tensor] = None,
                workspace: Optional[torch.Tensor] = None, chunk: int = CHUNK,
                want_state: bool = True) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Chunkwise prefill.  q, k [T, H, dk]; v [T, H, dv]; g, beta [T, H] fp32;
    state_in [N, H, dv, dk] fp32 or None; cu_seqlens int32 [N+1] (device) or
    None (``num_seqs`` equal sequences, default 1).  Returns (out, state_out);
    pass ``state_out=state_in`` to update the state in place."""
    T, H, dk = q.shape
    dv = v.shape[2]
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("gdn_prefill needs CUDA tensors")
    if cu_seqlens is not None:
        if cu_seqlens.dtype != torch.int32 or cu_seqlens.device != dev:
            raise ValueError("cu_seqlens must be int32 on the same device")
        N = cu_seqlens.numel() - 1
    else:
        N = 1 if num_seqs is None else int(num_seqs)
    if k.shape != (T, H, dk) or v.shape[:2] != (T, H):
        raise ValueError("q/k/v shapes disagree")
    if g.shape != (T, H) or beta.shape != (T, H) or g.dtype != torch.float32 or beta.dtype != torch.float32:
        raise ValueError("g and beta must be fp32 [T, H]")
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k, v must share a dtype")
    for t in (k, v, g, beta, state_in, out, state_out, cu_seqlens, workspace):
        if t is not None and t.device != dev:
            raise ValueError("all tensors must be on %s" % dev)
    if state_in is not None and (state_in.shape != (N, H, dv, dk) or state_in.dtype != torch.float32):
        raise ValueError("state_in must be fp32 [N, H, dv, dk]")
    if out is None:
        out = torch.empty((T, H, dv), dtype=q.dtype, device=dev)
    if state_out is None and want_state:
        state_out = torch.empty((N, H, dv, dk), dtype=torch.float32, device=dev)
    dt = _dtype_code(q.dtype)
    need = gdn_prefill_workspace_size(N, T, H, dk, dv, chunk, q.dtype)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = _load().gdn_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state_in),
                             _ptr(out), _ptr(state_out), _ptr(cu_seqlens), N, T, H, dk, dv,
                             chunk, dt, _ptr(workspace), ws_bytes, _stream(dev))
    if st != GDN_OK:
        raise GdnError(st, "gdn_prefill")
    return out, state_out


NOALLOC_SCRATCH_BYTES = 16 << 20


def gdn_prefill_noalloc(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor,
                        beta: torch.Tensor, state_in: Optional[torch.Tensor] = None,
                        cu_seqlens: Optional[torch.Tensor] = None, *,
                        num_seqs: Optional[int] = None, out: Optional[torch.Tensor] = None,
                        state_out: Optional[torch.Tensor] = None, chunk: int = CHUNK,
                        want_state: bool = True) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """gdn_prefill without a workspace: the library's fixed scratch array
    (NOALLOC_SCRATCH_BYTES per device) is used instead.  For callers that
    cannot allocate device memory; concurrent calls on one device race."""
    T, H, dk = q.shape
    dv = v.shape[2]
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("gdn_prefill_noalloc needs CUDA tensors")
    if cu_seqlens is not None:
        if cu_seqlens.dtype != torch.int32 or cu_seqlens.device != dev:
            raise ValueError("cu_seqlens must be int32 on the same device")
        N = cu_seqlens.numel() - 1
    else:
        N = 1 if num_seqs is None else int(num_seqs)
    if out is None:
        out = torch.empty((T, H, dv), dtype=q.dtype, device=dev)
    if state_out is None and want_state:
        state_out = torch.empty((N, H, dv, dk), dtype=torch.float32, device=dev)
    st = _load().gdn_prefill_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                     _ptr(state_in), _ptr(out), _ptr(state_out),
                                     _ptr(cu_seqlens), N, T, H, dk, dv, chunk,
                                     _dtype_code(q.dtype), _stream(dev))
    if st != GDN_OK:
        raise GdnError(st, "gdn_prefill_noalloc")
    return out, state_out


def gdn_decode_step(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor,
                    beta: torch.Tensor, state_in: torch.Tensor,
                    state_out: Optional[torch.Tensor] = None,
                    out: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """One decode token per sequence.  q, k [B, H, dk]; v [B, H, dv];
    g, beta [B, H] fp32; state_in [B, H, dv, dk] fp32.  ``state_out`` defaults
    to ``state_in`` (in-place update).  Returns (out [B, H, dv], state_out)."""
    B, H, dk = q.shape
    dv = v.shape[2]
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("gdn_decode_step needs CUDA tensors")
    if k.shape != (B, H, dk) or v.shape[:2] != (B, H) or g.shape != (B, H) or beta.shape != (B, H):
        raise ValueError("decode input shapes disagree")
    if state_in.shape != (B, H, dv, dk) or state_in.dtype != torch.float32:
        raise ValueError("state must be fp32 [B, H, dv, dk]")
    if g.dtype != torch.float32 or beta.dtype != torch.float32:
        raise ValueError("g and beta must be fp32")
    if state_out is None:
        state_out = state_in
    if out is None:
        out = torch.empty((B, H, dv), dtype=q.dtype, device=dev)
    st = _load().gdn_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                 _ptr(state_in), _ptr(state_out), _ptr(out), B, H, dk, dv,
                                 _dtype_code(q.dtype), _stream(dev))
    if st != GDN_OK:
        raise GdnError(st, "gdn_decode_step")
    return out, state_out
