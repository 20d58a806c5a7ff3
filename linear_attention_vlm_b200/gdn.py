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

GDN_OK, GDN_ERR_INVALID_ARG, GDN_ERR_UNSUPPORTED, GDN_ERR_CUDA, GDN_ERR_TIMEOUT, GDN_ERR_WORKSPACE = 0, 1, 2, 3, 4, 5
GDN_F32, GDN_BF16 = 0, 1
ACT_NONE, ACT_SILU = 0, 1
GATE_SIGMOID, GATE_SILU = 0, 1
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
    f32 = ctypes.c_float
    lib.gdn_preprocess.argtypes = [vp, vp, vp, fp, fp, fp, vp, vp, vp, vp, fp, fp, vp, vp, i32, i64,
                                   i32, i32, i32, f32, i32, vp]
    lib.gdn_preprocess.restype = i32
    lib.gdn_output_gate.argtypes = [vp, vp, fp, vp, i64, i32, i32, f32, i32, vp]
    lib.gdn_output_gate.restype = i32
    lib.gdn_layer_prefill_workspace_size.argtypes = [i32, i64, i32, i32, i32]
    lib.gdn_layer_prefill_workspace_size.restype = sz
    lib.gdn_layer_prefill.argtypes = [vp, vp, vp, fp, fp, fp, vp, vp, fp, fp, vp, fp, vp, vp, i32, i64, i32, i32,
                                      i32, i32, f32, i32, vp, sz, vp]
    lib.gdn_layer_prefill.restype = i32
    lib.gdn_rope.argtypes = [vp, vp, vp, i32, i64, i32, i32, i32, f32, i32, vp]
    lib.gdn_rope.restype = i32
    lib.gdn_swa_attention.argtypes = [vp, vp, vp, vp, vp, i32, i64, i32, i32, i32, i32, f32, i32, vp, vp]
    lib.gdn_swa_attention.restype = i32
    lib.gdn_session_workspace_size.argtypes = [i32, i32, i32, i32, i32]
    lib.gdn_session_workspace_size.restype = sz
    lib.gdn_session_create.argtypes = [i32, i32, i32, i32, i32, i32, i32, f32, vp, vp]
    lib.gdn_session_create.restype = i32
    lib.gdn_session_prefill.argtypes = [vp, i32, vp]
    lib.gdn_session_prefill.restype = i32
    lib.gdn_session_decode.argtypes = [vp, vp]
    lib.gdn_session_decode.restype = i32
    lib.gdn_session_step_eager.argtypes = [vp, i32, vp]
    lib.gdn_session_step_eager.restype = i32
    lib.gdn_session_graph_count.argtypes = [vp]
    lib.gdn_session_graph_count.restype = i32
    lib.gdn_session_destroy.argtypes = [vp]
    lib.gdn_session_destroy.restype = None
    lib.gdn_status_string.argtypes = [i32]
    lib.gdn_status_string.restype = ctypes.c_char_p
    lib.gdn_read_status.argtypes = [vp, vp, ctypes.POINTER(ctypes.c_int32)]
    lib.gdn_read_status.restype = i32
    lib.gdn_noalloc_read_status.argtypes = [vp, ctypes.POINTER(ctypes.c_int32)]
    lib.gdn_noalloc_read_status.restype = i32
    lib.gdn_set_wait_limit.argtypes = [ctypes.c_uint64]
    lib.gdn_set_wait_limit.restype = None
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


def gdn_read_status(word: torch.Tensor) -> int:
    """Wait for the current stream and return the device status word the
    tensor-core kernels leave (include/gdn.h, gdn_read_status): 0 when every
    wait inside them completed, else the kernel's code.  ``word`` is an int32
    view of the prefill workspace's first word, or gdn_swa_attention's status
    tensor."""
    if word.device.type != "cuda" or word.dtype != torch.int32 or word.numel() < 1:
        raise ValueError("word must be a CUDA int32 tensor")
    code = ctypes.c_int32(0)
    st = _load().gdn_read_status(_ptr(word), _stream(word.device), ctypes.byref(code))
    if st not in (GDN_OK, GDN_ERR_TIMEOUT):
        raise GdnError(st, "gdn_read_status")
    return int(code.value)


WAIT_LIMIT_DEFAULT = 2000000000


def gdn_set_wait_limit(ns: int) -> None:
    """Bound (ns) on the work-loop waits of the tensor-core kernels this host
    thread launches next (include/gdn.h, gdn_set_wait_limit); 0 makes the
    first wait on work in flight give up, WAIT_LIMIT_DEFAULT restores 2 s."""
    _load().gdn_set_wait_limit(int(ns))


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


def gdn_noalloc_read_status(device=None) -> int:
    """Wait for the current stream and return the status word that
    gdn_prefill_noalloc's kernels leave in the library's scratch on
    ``device`` (include/gdn.h, gdn_noalloc_read_status): 0 when every wait
    inside them completed, else the kernel's code."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    code = ctypes.c_int32(0)
    with torch.cuda.device(dev):
        st = _load().gdn_noalloc_read_status(_stream(dev), ctypes.byref(code))
    if st not in (GDN_OK, GDN_ERR_TIMEOUT):
        raise GdnError(st, "gdn_noalloc_read_status")
    return int(code.value)


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


def gdn_preprocess(xq: torch.Tensor, xk: torch.Tensor, xv: torch.Tensor, conv_w: torch.Tensor,
                   a: torch.Tensor, b: torch.Tensor, conv_state_in: Optional[torch.Tensor] = None,
                   cu_seqlens: Optional[torch.Tensor] = None, *, num_seqs: Optional[int] = None,
                   activation: int = ACT_NONE, eps: float = 1e-6, conv_state_out: Optional[torch.Tensor] = None,
                   want_state: bool = True):
    """Raw projections -> gdn_prefill's inputs (include/gdn.h, gdn_preprocess).
    xq, xk, xv [T, H, d]; conv_w [3, H, d, 4] fp32; a, b [T, H] fp32 logits;
    conv_state_in [N, 3, 3, H, d] (dtype of x) or None.  Returns
    (q, k, v, g, beta, conv_state_out); pass conv_state_out=conv_state_in to
    update the convolution state in place."""
    T, H, d = xq.shape
    dev = xq.device
    if dev.type != "cuda":
        raise ValueError("gdn_preprocess needs CUDA tensors")
    if xk.shape != (T, H, d) or xv.shape != (T, H, d):
        raise ValueError("xq/xk/xv shapes disagree")
    if xk.dtype != xq.dtype or xv.dtype != xq.dtype:
        raise ValueError("xq, xk, xv must share a dtype")
    if conv_w.shape != (3, H, d, 4) or conv_w.dtype != torch.float32:
        raise ValueError("conv_w must be fp32 [3, H, d, 4]")
    if a.shape != (T, H) or b.shape != (T, H) or a.dtype != torch.float32 or b.dtype != torch.float32:
        raise ValueError("a and b must be fp32 [T, H]")
    if cu_seqlens is not None:
        if cu_seqlens.dtype != torch.int32 or cu_seqlens.device != dev:
            raise ValueError("cu_seqlens must be int32 on the same device")
        N = cu_seqlens.numel() - 1
    else:
        N = 1 if num_seqs is None else int(num_seqs)
    if conv_state_in is not None and (conv_state_in.shape != (N, 3, 3, H, d) or conv_state_in.dtype != xq.dtype):
        raise ValueError("conv_state_in must be [N, 3, 3, H, d] in the dtype of x")
    for t in (xk, xv, conv_w, a, b, conv_state_in, conv_state_out, cu_seqlens):
        if t is not None and t.device != dev:
            raise ValueError("all tensors must be on %s" % dev)
    q, k, v = (torch.empty_like(xq) for _ in range(3))
    g = torch.empty((T, H), dtype=torch.float32, device=dev)
    beta = torch.empty_like(g)
    if conv_state_out is None and want_state:
        conv_state_out = torch.empty((N, 3, 3, H, d), dtype=xq.dtype, device=dev)
    st = _load().gdn_preprocess(_ptr(xq), _ptr(xk), _ptr(xv), _ptr(conv_w), _ptr(a), _ptr(b),
                                _ptr(conv_state_in), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                _ptr(conv_state_out), _ptr(cu_seqlens), N, T, H, d, int(activation),
                                float(eps), _dtype_code(xq.dtype), _stream(dev))
    if st != GDN_OK:
        raise GdnError(st, "gdn_preprocess")
    return q, k, v, g, beta, conv_state_out


def gdn_output_gate(o: torch.Tensor, z: torch.Tensor, norm_w: Optional[torch.Tensor] = None, *,
                    gate: int = GATE_SIGMOID, eps: float = 1e-6, out: Optional[torch.Tensor] = None):
    """y = n(o) * act(z) over the last dimension (include/gdn.h,
    gdn_output_gate).  o, z [..., dv] of one dtype; norm_w [dv] fp32 or None.
    ``out`` may be ``o`` (in place)."""
    dev = o.device
    if dev.type != "cuda":
        raise ValueError("gdn_output_gate needs CUDA tensors")
    if z.shape != o.shape or z.dtype != o.dtype or z.device != dev:
        raise ValueError("o and z must share shape, dtype and device")
    dv = o.shape[-1]
    if norm_w is not None and (norm_w.shape != (dv,) or norm_w.dtype != torch.float32 or norm_w.device != dev):
        raise ValueError("norm_w must be fp32 [dv] on the same device")
    if out is None:
        out = torch.empty_like(o)
    rows = o.numel() // dv if dv else 0
    st = _load().gdn_output_gate(_ptr(o), _ptr(z), _ptr(norm_w), _ptr(out), rows, dv, int(gate), float(eps),
                                 _dtype_code(o.dtype), _stream(dev))
    if st != GDN_OK:
        raise GdnError(st, "gdn_output_gate")
    return out


def gdn_layer_prefill_workspace_size(num_seqs: int, total_tokens: int, H: int, d: int,
                                     dtype: torch.dtype = torch.bfloat16) -> int:
    return int(_load().gdn_layer_prefill_workspace_size(num_seqs, total_tokens, H, d, _dtype_code(dtype)))


def gdn_layer_prefill(xq: torch.Tensor, xk: torch.Tensor, xv: torch.Tensor, conv_w: torch.Tensor,
                      a: torch.Tensor, b: torch.Tensor, z: torch.Tensor,
                      conv_state_in: Optional[torch.Tensor] = None, state_in: Optional[torch.Tensor] = None,
                      norm_w: Optional[torch.Tensor] = None, cu_seqlens: Optional[torch.Tensor] = None, *,
                      num_seqs: Optional[int] = None, activation: int = ACT_NONE, gate: int = GATE_SIGMOID,
                      eps: float = 1e-6, y: Optional[torch.Tensor] = None,
                      state_out: Optional[torch.Tensor] = None, conv_state_out: Optional[torch.Tensor] = None,
                      workspace: Optional[torch.Tensor] = None, want_state: bool = True,
                      want_conv_state: bool = True):
    """Raw projections -> gated output of one layer's token mixer
    (include/gdn.h, gdn_layer_prefill).  xq, xk, xv, z [T, H, d]; conv_w
    [3, H, d, 4] fp32; a, b [T, H] fp32 logits; conv_state_in [N, 3, 3, H, d]
    or None; state_in [N, H, d, d] fp32 or None; norm_w [d] fp32 or None.
    Returns (y, state_out, conv_state_out); pass state_out=state_in and
    conv_state_out=conv_state_in to carry both states in place."""
    T, H, d = xq.shape
    dev = xq.device
    if dev.type != "cuda":
        raise ValueError("gdn_layer_prefill needs CUDA tensors")
    for t in (xk, xv, z):
        if t.shape != (T, H, d) or t.dtype != xq.dtype:
            raise ValueError("xq, xk, xv and z must share shape [T, H, d] and dtype")
    if conv_w.shape != (3, H, d, 4) or conv_w.dtype != torch.float32:
        raise ValueError("conv_w must be fp32 [3, H, d, 4]")
    if a.shape != (T, H) or b.shape != (T, H) or a.dtype != torch.float32 or b.dtype != torch.float32:
        raise ValueError("a and b must be fp32 [T, H]")
    N = _seq_count(cu_seqlens, num_seqs, dev)
    if conv_state_in is not None and (conv_state_in.shape != (N, 3, 3, H, d) or conv_state_in.dtype != xq.dtype):
        raise ValueError("conv_state_in must be [N, 3, 3, H, d] in the dtype of x")
    if state_in is not None and (state_in.shape != (N, H, d, d) or state_in.dtype != torch.float32):
        raise ValueError("state_in must be fp32 [N, H, d, d]")
    if norm_w is not None and (norm_w.shape != (d,) or norm_w.dtype != torch.float32):
        raise ValueError("norm_w must be fp32 [d]")
    for t in (xk, xv, z, conv_w, a, b, conv_state_in, state_in, norm_w, cu_seqlens, y, state_out,
              conv_state_out, workspace):
        if t is not None and t.device != dev:
            raise ValueError("all tensors must be on %s" % dev)
    if y is None:
        y = torch.empty_like(xq)
    if state_out is None and want_state:
        state_out = torch.empty((N, H, d, d), dtype=torch.float32, device=dev)
    if conv_state_out is None and want_conv_state:
        conv_state_out = torch.empty((N, 3, 3, H, d), dtype=xq.dtype, device=dev)
    need = gdn_layer_prefill_workspace_size(N, T, H, d, xq.dtype)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    ws_bytes = workspace.numel() * workspace.element_size()
    st = _load().gdn_layer_prefill(_ptr(xq), _ptr(xk), _ptr(xv), _ptr(conv_w), _ptr(a), _ptr(b),
                                   _ptr(conv_state_in), _ptr(conv_state_out), _ptr(state_in), _ptr(state_out),
                                   _ptr(z), _ptr(norm_w), _ptr(y), _ptr(cu_seqlens), N, T, H, d, int(activation),
                                   int(gate), float(eps), _dtype_code(xq.dtype), _ptr(workspace), ws_bytes,
                                   _stream(dev))
    if st != GDN_OK:
        raise GdnError(st, "gdn_layer_prefill")
    return y, state_out, conv_state_out


def _seq_count(cu_seqlens: Optional[torch.Tensor], num_seqs: Optional[int], dev) -> int:
    if cu_seqlens is not None:
        if cu_seqlens.dtype != torch.int32 or cu_seqlens.device != dev:
            raise ValueError("cu_seqlens must be int32 on the same device")
        return cu_seqlens.numel() - 1
    return 1 if num_seqs is None else int(num_seqs)


def gdn_rope(x: torch.Tensor, cu_seqlens: Optional[torch.Tensor] = None, *, num_seqs: Optional[int] = None,
             offset: int = 0, base: float = 10000.0, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Rotate-half RoPE of x [T, H, d] at each token's position inside its
    sequence plus ``offset`` (include/gdn.h, gdn_rope).  ``out`` may be ``x``."""
    T, H, d = x.shape
    dev = x.device
    if dev.type != "cuda":
        raise ValueError("gdn_rope needs CUDA tensors")
    N = _seq_count(cu_seqlens, num_seqs, dev)
    if out is None:
        out = torch.empty_like(x)
    elif out.shape != x.shape or out.dtype != x.dtype or out.device != dev:
        raise ValueError("out must match x")
    st = _load().gdn_rope(_ptr(x), _ptr(out), _ptr(cu_seqlens), N, T, H, d, int(offset), float(base),
                          _dtype_code(x.dtype), _stream(dev))
    if st != GDN_OK:
        raise GdnError(st, "gdn_rope")
    return out


def gdn_swa_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, cu_seqlens: Optional[torch.Tensor] = None,
                      *, num_seqs: Optional[int] = None, window: int = 8192, scale: Optional[float] = None,
                      out: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Causal sliding-window attention with grouped key/value heads
    (include/gdn.h, gdn_swa_attention).  q [T, Hq, d], k, v [T, Hkv, d] bf16,
    already rotated.  ``status`` (int32 [1] on the device, cleared by the
    caller) receives a nonzero code if a wait inside the kernel gave up."""
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("gdn_swa_attention needs CUDA tensors")
    if k.shape != (T, Hkv, d) or v.shape != (T, Hkv, d):
        raise ValueError("k and v must be [T, Hkv, d]")
    if k.dtype != q.dtype or v.dtype != q.dtype or k.device != dev or v.device != dev:
        raise ValueError("q, k, v must share dtype and device")
    N = _seq_count(cu_seqlens, num_seqs, dev)
    if out is None:
        out = torch.empty_like(q)
    elif out.shape != q.shape or out.dtype != q.dtype or out.device != dev:
        raise ValueError("out must match q")
    if status is not None and (status.dtype != torch.int32 or status.device != dev):
        raise ValueError("status must be int32 on the same device")
    st = _load().gdn_swa_attention(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(cu_seqlens), N, T, Hq, Hkv, d,
                                   int(window), 0.0 if scale is None else float(scale), _dtype_code(q.dtype),
                                   _ptr(status), _stream(dev))
    if st != GDN_OK:
        raise GdnError(st, "gdn_swa_attention")
    return out


class _SessionBuffers(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("xq", "xk", "xv", "a", "b", "z", "y", "q", "k", "v", "o", "g",
                                                "beta", "state", "conv_state", "conv_w", "norm_w", "workspace")] + \
               [("workspace_bytes", ctypes.c_size_t)]


class GdnSession:
    """Streaming session (include/gdn.h, gdn_session_*): one layer step --
    pre-processing, the recurrence with a carried state, the output gate --
    over buffers allocated here once, captured as a CUDA graph per token
    count and replayed.  Write the next step's inputs into ``xq, xk, xv, a,
    b, z`` (``[num_streams * tokens, ...]`` at the start, stream-major), call
    ``prefill(tokens)`` or ``decode()``, read ``y``.  ``feed`` does the copies."""

    def __init__(self, num_streams: int, H: int, d: int, seg_tokens: int, conv_w: torch.Tensor,
                 norm_w: Optional[torch.Tensor] = None, *, dtype: torch.dtype = torch.bfloat16,
                 activation: int = ACT_NONE, gate: int = GATE_SIGMOID, eps: float = 1e-6, device=None):
        dev = torch.device(device) if device is not None else conv_w.device
        if dev.type != "cuda":
            raise ValueError("GdnSession needs a CUDA device")
        if conv_w.shape != (3, H, d, 4) or conv_w.dtype != torch.float32:
            raise ValueError("conv_w must be fp32 [3, H, d, 4]")
        self.B, self.H, self.d, self.seg, self.dtype = num_streams, H, d, seg_tokens, dtype
        R = num_streams * seg_tokens
        mk = lambda *shape, dt=dtype: torch.zeros(shape, dtype=dt, device=dev)
        self.xq, self.xk, self.xv, self.z, self.y = (mk(R, H, d) for _ in range(5))
        self.a, self.b = mk(R, H, dt=torch.float32), mk(R, H, dt=torch.float32)
        self._scratch = [mk(R, H, d) for _ in range(4)] + [mk(R, H, dt=torch.float32) for _ in range(2)]
        self.state = mk(num_streams, H, d, d, dt=torch.float32)
        self.conv_state = mk(num_streams, 3, 3, H, d)
        self.conv_w = conv_w.to(dev).contiguous().clone()
        self.norm_w = None if norm_w is None else norm_w.to(dev, torch.float32).contiguous().clone()
        lib = _load()
        ws_bytes = int(lib.gdn_session_workspace_size(num_streams, H, d, seg_tokens, _dtype_code(dtype)))
        self.workspace = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
        q, k, v, o, g, beta = self._scratch
        self._buf = _SessionBuffers(*(_ptr(t) for t in (self.xq, self.xk, self.xv, self.a, self.b, self.z, self.y,
                                                         q, k, v, o, g, beta, self.state, self.conv_state,
                                                         self.conv_w, self.norm_w, self.workspace)), ws_bytes)
        self._h = ctypes.c_void_p()
        st = lib.gdn_session_create(num_streams, H, d, seg_tokens, _dtype_code(dtype), int(activation), int(gate),
                                    float(eps), ctypes.byref(self._buf), ctypes.byref(self._h))
        if st != GDN_OK:
            raise GdnError(st, "gdn_session_create")
        self.device = dev

    def prefill(self, tokens: Optional[int] = None, eager: bool = False) -> torch.Tensor:
        tokens = self.seg if tokens is None else int(tokens)
        lib = _load()
        s = _stream(self.device)
        st = lib.gdn_session_step_eager(self._h, tokens, s) if eager else lib.gdn_session_prefill(self._h, tokens, s)
        if st != GDN_OK:
            raise GdnError(st, "gdn_session_prefill")
        return self.y[: self.B * tokens]

    def decode(self, eager: bool = False) -> torch.Tensor:
        lib = _load()
        s = _stream(self.device)
        st = lib.gdn_session_step_eager(self._h, 0, s) if eager else lib.gdn_session_decode(self._h, s)
        if st != GDN_OK:
            raise GdnError(st, "gdn_session_decode")
        return self.y[: self.B]

    def feed(self, xq, xk, xv, a, b, z, eager: bool = False) -> torch.Tensor:
        """Copy one step's inputs ([num_streams * tokens, ...], stream-major;
        tokens = 1 means a decode step) into the staging buffers and run it."""
        n = xq.shape[0]
        if n % self.B != 0:
            raise ValueError("rows must be a multiple of num_streams")
        for dst, src in ((self.xq, xq), (self.xk, xk), (self.xv, xv), (self.a, a), (self.b, b), (self.z, z)):
            dst[:n].copy_(src, non_blocking=True)
        return self.prefill(n // self.B, eager=eager)

    def graph_count(self) -> int:
        return int(_load().gdn_session_graph_count(self._h))

    def reset(self) -> None:
        self.state.zero_()
        self.conv_state.zero_()

    def close(self) -> None:
        if getattr(self, "_h", None) is not None and self._h.value:
            _load().gdn_session_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
