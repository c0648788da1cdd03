"""Gated delta rule on NVIDIA B200 (sm_100a): Python binding of libgdn.so.

This module only marshals arguments: it reads shapes and data pointers from
torch tensors and calls the C ABI declared in ``include/gdn.h``.  Every step
of the computation runs in the library's CUDA kernels; there is no Python or
CPU fallback, and importing the binding fails loudly when ``libgdn.so`` has
not been built (``python -m gated_delta_rule_142_b200.build``).

The operation ("ATMA: Long-Context Language Modeling via Polar Attention and
Gated-Delta Compression Memory", Sec. 3.3), per (batch, head):

    S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,   o_t = S_t q_t,
    alpha_t = exp(log_alpha_t).

Tensors may live on the current CUDA device (used in place) or on the host
(staged by the library through stream-ordered device buffers).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIBRARY = os.path.join(_PKG, "libgdn.so")

GDN_F32 = 0
GDN_BF16 = 1

STATUS = {
    0: "GDN_OK", 1: "GDN_ERR_NULL_PTR", 2: "GDN_ERR_INVALID_SIZE", 3: "GDN_ERR_UNSUPPORTED",
    4: "GDN_ERR_MISALIGNED", 5: "GDN_ERR_ALLOC", 6: "GDN_ERR_LAUNCH", 7: "GDN_ERR_DEVICE_TIMEOUT",
    8: "GDN_ERR_ALIAS", 9: "GDN_ERR_DEVICE", 10: "GDN_ERR_SCRATCH_LIMIT",
}

EXPORTS = ("gdn_forward", "gdn_decode_step", "gdn_forward_plan", "gdn_status_string", "gdn_version",
           "gdn_forward_noalloc", "gdn_scratch_release", "gdn_timing_start", "gdn_timing_stop",
           "gdn_forward_varlen", "gdn_forward_raw", "gdn_forward_varlen_raw", "gdn_decode_step_raw",
           "gdn_backward", "gdn_forward_grouped", "gdn_decode_step_grouped", "gdn_causal_conv",
           "gdn_device_status", "gdn_selftest_device_timeout", "gdn_forward_conv")

# gdn_kernel_kind names, in enum order
KERNEL_KINDS = ("prep", "chain", "transfer", "prefix", "fused", "simt", "decode", "input", "backward",
                "group_out")


class GdnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__("%s: %s (%s)" % (where, STATUS.get(status, status), status_string(status)))


_lib = None


def load(path: str = LIBRARY) -> ctypes.CDLL:
    """Load libgdn.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError("libgdn.so not found at %s: build it with "
                           "`python -m gated_delta_rule_142_b200.build`" % path)
    lib = ctypes.CDLL(path)
    vp, i64 = ctypes.c_void_p, ctypes.c_int64
    for fn in (lib.gdn_forward, lib.gdn_forward_raw):
        fn.argtypes = [vp] * 8 + [i64] * 6 + [vp, ctypes.c_int]
        fn.restype = ctypes.c_int
    for fn in (lib.gdn_decode_step, lib.gdn_decode_step_raw):
        fn.argtypes = [vp] * 7 + [i64] * 4 + [vp, ctypes.c_int]
        fn.restype = ctypes.c_int
    lib.gdn_status_string.argtypes = [ctypes.c_int]
    lib.gdn_status_string.restype = ctypes.c_char_p
    lib.gdn_version.argtypes = []
    lib.gdn_version.restype = ctypes.c_int
    lib.gdn_forward_plan.argtypes = [i64] * 6 + [ctypes.c_int, ctypes.POINTER(i64), ctypes.POINTER(ctypes.c_int)]
    lib.gdn_forward_plan.restype = ctypes.c_int
    for fn in (lib.gdn_forward_varlen, lib.gdn_forward_varlen_raw):
        fn.argtypes = [vp] * 5 + [ctypes.POINTER(i64), i64] + [vp] * 3 + [i64] * 5 + [vp, ctypes.c_int]
        fn.restype = ctypes.c_int
    lib.gdn_backward.argtypes = [vp] * 14 + [i64] * 6 + [vp, ctypes.c_int]
    lib.gdn_device_status.argtypes = [vp]
    lib.gdn_device_status.restype = ctypes.c_int
    lib.gdn_selftest_device_timeout.argtypes = [vp]
    lib.gdn_selftest_device_timeout.restype = ctypes.c_int
    lib.gdn_causal_conv.argtypes = [vp] * 5 + [i64] * 4 + [vp, ctypes.c_int]
    lib.gdn_causal_conv.restype = ctypes.c_int
    lib.gdn_forward_conv.argtypes = [vp] * 11 + [i64] * 7 + [vp, ctypes.c_int]
    lib.gdn_forward_conv.restype = ctypes.c_int
    lib.gdn_forward_grouped.argtypes = [vp] * 8 + [i64] * 7 + [vp, ctypes.c_int]
    lib.gdn_forward_grouped.restype = ctypes.c_int
    lib.gdn_decode_step_grouped.argtypes = [vp] * 7 + [i64] * 5 + [vp, ctypes.c_int]
    lib.gdn_decode_step_grouped.restype = ctypes.c_int
    lib.gdn_backward.restype = ctypes.c_int
    lib.gdn_scratch_release.argtypes = []
    lib.gdn_scratch_release.restype = ctypes.c_int
    lib.gdn_timing_start.argtypes = []
    lib.gdn_timing_start.restype = ctypes.c_int
    lib.gdn_timing_stop.argtypes = [ctypes.POINTER(ctypes.c_double), ctypes.POINTER(i64)]
    lib.gdn_timing_stop.restype = ctypes.c_int
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load().gdn_status_string(int(status)).decode()


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return GDN_F32
    if t.dtype == torch.bfloat16:
        return GDN_BF16
    raise TypeError("q/k/v must be float32 or bfloat16, got %s" % t.dtype)


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr()) if t.numel() > 0 else None


def _pinned(t: torch.Tensor) -> bool:
    return t.device.type == "cpu" and torch.cuda.is_available() and t.is_pinned()


def _stream_handle(device: torch.device, stream) -> ctypes.c_void_p:
    if stream is None:
        if device.type == "cuda":
            stream = torch.cuda.current_stream(device)
        else:
            stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def forward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, log_alpha: torch.Tensor,
            beta: torch.Tensor, S0: Optional[torch.Tensor] = None, chunk: int = 64,
            out: Optional[torch.Tensor] = None, S_final: Optional[torch.Tensor] = None,
            output_final_state: bool = True, stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Chunkwise forward.  q, k [B,T,H,dk], v [B,T,H,dv] (float32 or bfloat16, same dtype);
    log_alpha, beta [B,T,H] float32; S0 [B,H,dv,dk] float32 or None.
    Returns (out [B,T,H,dv] in the input dtype, S_final [B,H,dv,dk] float32 or None)."""
    return _forward("gdn_forward", q, k, v, log_alpha, beta, S0, chunk, out, S_final, output_final_state, stream)


def forward_raw(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, x_alpha: torch.Tensor,
                x_beta: torch.Tensor, S0: Optional[torch.Tensor] = None, chunk: int = 64,
                out: Optional[torch.Tensor] = None, S_final: Optional[torch.Tensor] = None,
                output_final_state: bool = True, stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """forward() with the input stage in the kernels: q, k in any scale (L2-normalised inside),
    x_alpha, x_beta [B,T,H] float32 gate logits (log alpha = -softplus(x_alpha),
    beta = sigmoid(x_beta))."""
    return _forward("gdn_forward_raw", q, k, v, x_alpha, x_beta, S0, chunk, out, S_final, output_final_state,
                    stream)


def _forward(entry, q, k, v, log_alpha, beta, S0, chunk, out, S_final, output_final_state, stream):
    lib = load()
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    for name, t, shape in (("k", k, (B, T, H, dk)), ("v", v, (B, T, H, dv)), ("log_alpha", log_alpha, (B, T, H)),
                           ("beta", beta, (B, T, H)), ("out", out, (B, T, H, dv))):
        if t is not None and tuple(t.shape) != shape:
            raise ValueError("%s has shape %s, expected %s" % (name, tuple(t.shape), shape))
    _dtype_code(q)
    if k.dtype != q.dtype or v.dtype != q.dtype or (out is not None and out.dtype != q.dtype):
        raise TypeError("q, k, v and out must share one dtype")
    for name, t in (("log_alpha", log_alpha), ("beta", beta), ("S0", S0), ("S_final", S_final)):
        if t is not None and t.dtype != torch.float32:
            raise TypeError("%s must be float32" % name)
    for name, t in (("S0", S0), ("S_final", S_final)):
        if t is not None and tuple(t.shape) != (B, H, dv, dk):
            raise ValueError("%s has shape %s, expected %s" % (name, tuple(t.shape), (B, H, dv, dk)))
    for t in (q, k, v, log_alpha, beta, S0, out, S_final):
        if t is not None and not t.is_contiguous():
            raise ValueError("tensors must be contiguous")
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device, pin_memory=_pinned(q))
    if S_final is None and output_final_state:
        S_final = torch.empty((B, H, dv, dk), dtype=torch.float32, device=q.device, pin_memory=_pinned(q))
    with torch.cuda.device(q.device if q.device.type == "cuda" else torch.cuda.current_device()):
        st = getattr(lib, entry)(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(S0), _ptr(out),
                                 _ptr(S_final), B, T, H, dk, dv, int(chunk), _stream_handle(q.device, stream),
                                 _dtype_code(q))
    if st != 0:
        raise GdnError(st, entry)
    return out, S_final


def forward_varlen(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, log_alpha: torch.Tensor,
                   beta: torch.Tensor, cu_seqlens, S0: Optional[torch.Tensor] = None, chunk: int = 64,
                   out: Optional[torch.Tensor] = None, S_final: Optional[torch.Tensor] = None,
                   output_final_state: bool = True, stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Chunkwise forward over N packed sequences.  q, k [T_total,H,dk], v [T_total,H,dv];
    log_alpha, beta [T_total,H] float32; cu_seqlens: N + 1 token offsets (list or CPU int tensor);
    S0 [N,H,dv,dk] float32 or None.  Returns (out [T_total,H,dv], S_final [N,H,dv,dk] or None)."""
    return _forward_varlen("gdn_forward_varlen", q, k, v, log_alpha, beta, cu_seqlens, S0, chunk, out, S_final,
                           output_final_state, stream)


def forward_varlen_raw(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, x_alpha: torch.Tensor,
                       x_beta: torch.Tensor, cu_seqlens, S0: Optional[torch.Tensor] = None, chunk: int = 64,
                       out: Optional[torch.Tensor] = None, S_final: Optional[torch.Tensor] = None,
                       output_final_state: bool = True, stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """forward_varlen() with the input stage in the kernels (see forward_raw)."""
    return _forward_varlen("gdn_forward_varlen_raw", q, k, v, x_alpha, x_beta, cu_seqlens, S0, chunk, out,
                           S_final, output_final_state, stream)


def _forward_varlen(entry, q, k, v, log_alpha, beta, cu_seqlens, S0, chunk, out, S_final, output_final_state,
                    stream):
    lib = load()
    T, H, dk = q.shape
    dv = v.shape[-1]
    cu = [int(x) for x in (cu_seqlens.tolist() if torch.is_tensor(cu_seqlens) else cu_seqlens)]
    N = len(cu) - 1
    if N < 0:
        raise ValueError("cu_seqlens needs at least one entry")
    for name, t, shape in (("k", k, (T, H, dk)), ("v", v, (T, H, dv)), ("log_alpha", log_alpha, (T, H)),
                           ("beta", beta, (T, H)), ("out", out, (T, H, dv))):
        if t is not None and tuple(t.shape) != shape:
            raise ValueError("%s has shape %s, expected %s" % (name, tuple(t.shape), shape))
    _dtype_code(q)
    if k.dtype != q.dtype or v.dtype != q.dtype or (out is not None and out.dtype != q.dtype):
        raise TypeError("q, k, v and out must share one dtype")
    for name, t in (("log_alpha", log_alpha), ("beta", beta), ("S0", S0), ("S_final", S_final)):
        if t is not None and t.dtype != torch.float32:
            raise TypeError("%s must be float32" % name)
    for name, t in (("S0", S0), ("S_final", S_final)):
        if t is not None and tuple(t.shape) != (N, H, dv, dk):
            raise ValueError("%s has shape %s, expected %s" % (name, tuple(t.shape), (N, H, dv, dk)))
    for t in (q, k, v, log_alpha, beta, S0, out, S_final):
        if t is not None and not t.is_contiguous():
            raise ValueError("tensors must be contiguous")
    if out is None:
        out = torch.empty((T, H, dv), dtype=q.dtype, device=q.device, pin_memory=_pinned(q))
    if S_final is None and output_final_state:
        S_final = torch.empty((N, H, dv, dk), dtype=torch.float32, device=q.device, pin_memory=_pinned(q))
    cu_arr = (ctypes.c_int64 * max(len(cu), 1))(*cu)
    with torch.cuda.device(q.device if q.device.type == "cuda" else torch.cuda.current_device()):
        st = getattr(lib, entry)(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), cu_arr, N, _ptr(S0),
                                 _ptr(out), _ptr(S_final), T, H, dk, dv, int(chunk),
                                 _stream_handle(q.device, stream), _dtype_code(q))
    if st != 0:
        raise GdnError(st, entry)
    return out, S_final


def backward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, log_alpha: torch.Tensor, beta: torch.Tensor,
             S0: Optional[torch.Tensor], grad_out: torch.Tensor, grad_S_final: Optional[torch.Tensor] = None,
             chunk: int = 64, want_grad_S0: bool = True, stream=None):
    """Reverse mode of forward().  grad_out [B,T,H,dv] (dtype of q); grad_S_final [B,H,dv,dk] float32 or
    None.  Returns (dq, dk, dv in the input dtype; dlog_alpha, dbeta [B,T,H] float32; dS0 or None)."""
    lib = load()
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    for name, t, shape in (("k", k, (B, T, H, dk)), ("v", v, (B, T, H, dv)), ("log_alpha", log_alpha, (B, T, H)),
                           ("beta", beta, (B, T, H)), ("grad_out", grad_out, (B, T, H, dv)),
                           ("S0", S0, (B, H, dv, dk)), ("grad_S_final", grad_S_final, (B, H, dv, dk))):
        if t is not None and tuple(t.shape) != shape:
            raise ValueError("%s has shape %s, expected %s" % (name, tuple(t.shape), shape))
    _dtype_code(q)
    if k.dtype != q.dtype or v.dtype != q.dtype or grad_out.dtype != q.dtype:
        raise TypeError("q, k, v and grad_out must share one dtype")
    for name, t in (("log_alpha", log_alpha), ("beta", beta), ("S0", S0), ("grad_S_final", grad_S_final)):
        if t is not None and t.dtype != torch.float32:
            raise TypeError("%s must be float32" % name)
    for t in (q, k, v, log_alpha, beta, S0, grad_out, grad_S_final):
        if t is not None and not t.is_contiguous():
            raise ValueError("tensors must be contiguous")
    pin = _pinned(q)
    dq = torch.empty_like(q, pin_memory=pin) if q.device.type == "cpu" else torch.empty_like(q)
    dk_ = torch.empty_like(k, pin_memory=pin) if k.device.type == "cpu" else torch.empty_like(k)
    dv_ = torch.empty_like(v, pin_memory=pin) if v.device.type == "cpu" else torch.empty_like(v)
    dla = torch.empty((B, T, H), dtype=torch.float32, device=q.device, pin_memory=pin)
    dbe = torch.empty((B, T, H), dtype=torch.float32, device=q.device, pin_memory=pin)
    dS0 = (torch.empty((B, H, dv, dk), dtype=torch.float32, device=q.device, pin_memory=pin)
           if want_grad_S0 else None)
    with torch.cuda.device(q.device if q.device.type == "cuda" else torch.cuda.current_device()):
        st = lib.gdn_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(S0), _ptr(grad_out),
                              _ptr(grad_S_final), _ptr(dq), _ptr(dk_), _ptr(dv_), _ptr(dla), _ptr(dbe), _ptr(dS0),
                              B, T, H, dk, dv, int(chunk), _stream_handle(q.device, stream), _dtype_code(q))
    if st != 0:
        raise GdnError(st, "gdn_backward")
    return dq, dk_, dv_, dla, dbe, dS0


def forward_grouped(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, log_alpha: torch.Tensor,
                    beta: torch.Tensor, S0: Optional[torch.Tensor] = None, chunk: int = 64,
                    out: Optional[torch.Tensor] = None, S_final: Optional[torch.Tensor] = None,
                    output_final_state: bool = True, stream=None):
    """Grouped heads: q [B,T,Hq,dk]; k [B,T,Hkv,dk], v [B,T,Hkv,dv], log_alpha, beta [B,T,Hkv];
    S0 [B,Hkv,dv,dk] or None.  Query head h reads the memory of key-value head h // (Hq // Hkv).
    Returns (out [B,T,Hq,dv], S_final [B,Hkv,dv,dk] or None)."""
    lib = load()
    B, T, Hq, dk = q.shape
    Hkv, dv = k.shape[2], v.shape[-1]
    for name, t, shape in (("k", k, (B, T, Hkv, dk)), ("v", v, (B, T, Hkv, dv)),
                           ("log_alpha", log_alpha, (B, T, Hkv)), ("beta", beta, (B, T, Hkv)),
                           ("out", out, (B, T, Hq, dv)), ("S0", S0, (B, Hkv, dv, dk)),
                           ("S_final", S_final, (B, Hkv, dv, dk))):
        if t is not None and tuple(t.shape) != shape:
            raise ValueError("%s has shape %s, expected %s" % (name, tuple(t.shape), shape))
    _dtype_code(q)
    if k.dtype != q.dtype or v.dtype != q.dtype or (out is not None and out.dtype != q.dtype):
        raise TypeError("q, k, v and out must share one dtype")
    for t in (q, k, v, log_alpha, beta, S0, out, S_final):
        if t is not None and not t.is_contiguous():
            raise ValueError("tensors must be contiguous")
    if out is None:
        out = torch.empty((B, T, Hq, dv), dtype=q.dtype, device=q.device, pin_memory=_pinned(q))
    if S_final is None and output_final_state:
        S_final = torch.empty((B, Hkv, dv, dk), dtype=torch.float32, device=q.device, pin_memory=_pinned(q))
    with torch.cuda.device(q.device if q.device.type == "cuda" else torch.cuda.current_device()):
        st = lib.gdn_forward_grouped(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(S0), _ptr(out),
                                     _ptr(S_final), B, T, Hq, Hkv, dk, dv, int(chunk),
                                     _stream_handle(q.device, stream), _dtype_code(q))
    if st != 0:
        raise GdnError(st, "gdn_forward_grouped")
    return out, S_final


def decode_step_grouped(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, log_alpha: torch.Tensor,
                        beta: torch.Tensor, S: torch.Tensor, out: Optional[torch.Tensor] = None,
                        stream=None) -> torch.Tensor:
    """Grouped-heads decode step: q [B,Hq,dk]; k [B,Hkv,dk], v [B,Hkv,dv], gates [B,Hkv];
    S [B,Hkv,dv,dk] float32 updated in place.  Returns out [B,Hq,dv]."""
    lib = load()
    B, Hq, dk = q.shape
    Hkv, dv = k.shape[1], v.shape[-1]
    for name, t, shape in (("k", k, (B, Hkv, dk)), ("v", v, (B, Hkv, dv)), ("log_alpha", log_alpha, (B, Hkv)),
                           ("beta", beta, (B, Hkv)), ("S", S, (B, Hkv, dv, dk)), ("out", out, (B, Hq, dv))):
        if t is not None and tuple(t.shape) != shape:
            raise ValueError("%s has shape %s, expected %s" % (name, tuple(t.shape), shape))
    _dtype_code(q)
    for t in (q, k, v, log_alpha, beta, S, out):
        if t is not None and not t.is_contiguous():
            raise ValueError("tensors must be contiguous")
    if out is None:
        out = torch.empty((B, Hq, dv), dtype=q.dtype, device=q.device, pin_memory=_pinned(q))
    with torch.cuda.device(q.device if q.device.type == "cuda" else torch.cuda.current_device()):
        st = lib.gdn_decode_step_grouped(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(S), _ptr(out),
                                         B, Hq, Hkv, dk, dv, _stream_handle(q.device, stream), _dtype_code(q))
    if st != 0:
        raise GdnError(st, "gdn_decode_step_grouped")
    return out


def causal_conv(x: torch.Tensor, weight: torch.Tensor, state_in: Optional[torch.Tensor] = None,
                out: Optional[torch.Tensor] = None, state_out: Optional[torch.Tensor] = None,
                want_state: bool = True, stream=None):
    """Depthwise causal convolution: x [B,T,C] (or [B,T,H,d], flattened), weight [C,W] float32,
    state_in [B,W-1,C] float32 or None.  Returns (y like x, state_out [B,W-1,C] or None)."""
    lib = load()
    B, T = x.shape[0], x.shape[1]
    C = 1
    for s_ in x.shape[2:]:
        C *= s_
    W = weight.shape[-1]
    if tuple(weight.shape) != (C, W) or weight.dtype != torch.float32:
        raise ValueError("weight must be float32 [C, W] with C = %d" % C)
    for name, t in (("state_in", state_in), ("state_out", state_out)):
        if t is not None and (tuple(t.shape) != (B, W - 1, C) or t.dtype != torch.float32):
            raise ValueError("%s must be float32 [B, W-1, C]" % name)
    _dtype_code(x)
    for t in (x, weight, state_in, out, state_out):
        if t is not None and not t.is_contiguous():
            raise ValueError("tensors must be contiguous")
    if out is None:
        out = torch.empty_like(x, pin_memory=_pinned(x)) if x.device.type == "cpu" else torch.empty_like(x)
    if state_out is None and want_state:
        state_out = torch.empty((B, W - 1, C), dtype=torch.float32, device=x.device, pin_memory=_pinned(x))
    with torch.cuda.device(x.device if x.device.type == "cuda" else torch.cuda.current_device()):
        st = lib.gdn_causal_conv(_ptr(x), _ptr(weight), _ptr(state_in), _ptr(out), _ptr(state_out), B, T, C, W,
                                 _stream_handle(x.device, stream), _dtype_code(x))
    if st != 0:
        raise GdnError(st, "gdn_causal_conv")
    return out, state_out


def forward_conv(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, x_alpha: torch.Tensor, x_beta: torch.Tensor,
                 conv_weight: torch.Tensor, conv_state: Optional[torch.Tensor] = None, S0: Optional[torch.Tensor] = None,
                 chunk: int = 64, out: Optional[torch.Tensor] = None, S_final: Optional[torch.Tensor] = None,
                 conv_state_out: Optional[torch.Tensor] = None, stream=None):
    """The short causal convolution of q, k, v, then the raw forward (gdn_forward_conv).
    conv_weight float32 [3, H*d, W] (q, k, v blocks; dk == dv), conv_state float32 [3, B, W-1, H*d] or
    None.  Device tensors only.  Returns (out, S_final, conv_state_out)."""
    lib = load()
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if dk != dv:
        raise ValueError("this binding takes dk == dv (the C entry point takes separate block sizes)")
    W = conv_weight.shape[-1]
    if tuple(conv_weight.shape) != (3, H * dk, W) or conv_weight.dtype != torch.float32:
        raise ValueError("conv_weight must be float32 [3, H*d, W]")
    for name, t in (("conv_state", conv_state), ("conv_state_out", conv_state_out)):
        if t is not None and (tuple(t.shape) != (3, B, W - 1, H * dk) or t.dtype != torch.float32):
            raise ValueError("%s must be float32 [3, B, W-1, H*d]" % name)
    for name, t, shape in (("k", k, (B, T, H, dk)), ("v", v, (B, T, H, dv)), ("x_alpha", x_alpha, (B, T, H)),
                           ("x_beta", x_beta, (B, T, H)), ("S0", S0, (B, H, dv, dk))):
        if t is not None and tuple(t.shape) != shape:
            raise ValueError("%s has shape %s, expected %s" % (name, tuple(t.shape), shape))
    _dtype_code(q)
    for t in (q, k, v, x_alpha, x_beta, conv_weight, conv_state, S0, out, S_final, conv_state_out):
        if t is not None and (not t.is_contiguous() or t.device.type != "cuda"):
            raise ValueError("tensors must be contiguous CUDA tensors")
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    if S_final is None:
        S_final = torch.empty((B, H, dv, dk), dtype=torch.float32, device=q.device)
    if conv_state_out is None and W > 1:
        conv_state_out = torch.empty((3, B, W - 1, H * dk), dtype=torch.float32, device=q.device)
    with torch.cuda.device(q.device):
        st = lib.gdn_forward_conv(_ptr(q), _ptr(k), _ptr(v), _ptr(x_alpha), _ptr(x_beta), _ptr(conv_weight),
                                  _ptr(conv_state), _ptr(conv_state_out), _ptr(S0), _ptr(out), _ptr(S_final), B, T,
                                  H, dk, dv, W, chunk, _stream_handle(q.device, stream), _dtype_code(q))
    if st != 0:
        raise GdnError(st, "gdn_forward_conv")
    return out, S_final, conv_state_out


def forward_plan(B: int, T: int, H: int, dk: int, dv: int, chunk: int = 64, dtype=torch.bfloat16):
    """(scratch bytes, kernel launches) that gdn_forward takes for these sizes on the current device."""
    lib = load()
    code = GDN_BF16 if dtype == torch.bfloat16 else GDN_F32
    scratch, launches = ctypes.c_int64(0), ctypes.c_int(0)
    st = lib.gdn_forward_plan(B, T, H, dk, dv, int(chunk), code, ctypes.byref(scratch), ctypes.byref(launches))
    if st != 0:
        raise GdnError(st, "gdn_forward_plan")
    return scratch.value, launches.value


def device_status(stream=None) -> int:
    """Synchronise the stream and return GDN_OK (0), or the status of a bounded device-side wait that
    gave up since the last call (GDN_ERR_DEVICE_TIMEOUT = 7)."""
    dev = torch.device("cuda", torch.cuda.current_device())
    return int(load().gdn_device_status(_stream_handle(dev, stream)))


def selftest_device_timeout(stream=None) -> None:
    """Enqueue a kernel whose bounded wait gives up by design (see gdn_selftest_device_timeout)."""
    dev = torch.device("cuda", torch.cuda.current_device())
    st = load().gdn_selftest_device_timeout(_stream_handle(dev, stream))
    if st != 0:
        raise GdnError(st, "gdn_selftest_device_timeout")


def scratch_release() -> None:
    """Return the library's unused pooled device scratch on the current device to the driver."""
    st = load().gdn_scratch_release()
    if st != 0:
        raise GdnError(st, "gdn_scratch_release")


def timing_start() -> None:
    """Start recording per-kernel device times of every launch the library makes."""
    st = load().gdn_timing_start()
    if st != 0:
        raise GdnError(st, "gdn_timing_start")


def timing_stop() -> dict:
    """Stop recording; {kernel kind: (total ms, launches)} for the kinds that ran."""
    n = len(KERNEL_KINDS)
    ms = (ctypes.c_double * n)()
    cnt = (ctypes.c_int64 * n)()
    st = load().gdn_timing_stop(ms, cnt)
    if st != 0:
        raise GdnError(st, "gdn_timing_stop")
    return {KERNEL_KINDS[i]: (ms[i], cnt[i]) for i in range(n) if cnt[i] > 0}


def decode_step(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, log_alpha: torch.Tensor,
                beta: torch.Tensor, S: torch.Tensor, out: Optional[torch.Tensor] = None,
                stream=None) -> torch.Tensor:
    """One token for every (b, h).  q, k [B,H,dk]; v [B,H,dv]; log_alpha, beta [B,H] float32;
    S [B,H,dv,dk] float32 is updated in place.  Returns out [B,H,dv]."""
    return _decode("gdn_decode_step", q, k, v, log_alpha, beta, S, out, stream)


def decode_step_raw(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, x_alpha: torch.Tensor,
                    x_beta: torch.Tensor, S: torch.Tensor, out: Optional[torch.Tensor] = None,
                    stream=None) -> torch.Tensor:
    """decode_step() with the input stage in the kernel (see forward_raw)."""
    return _decode("gdn_decode_step_raw", q, k, v, x_alpha, x_beta, S, out, stream)


def _decode(entry, q, k, v, log_alpha, beta, S, out, stream):
    lib = load()
    B, H, dk = q.shape
    dv = v.shape[-1]
    for name, t, shape in (("k", k, (B, H, dk)), ("v", v, (B, H, dv)), ("log_alpha", log_alpha, (B, H)),
                           ("beta", beta, (B, H)), ("S", S, (B, H, dv, dk)), ("out", out, (B, H, dv))):
        if t is not None and tuple(t.shape) != shape:
            raise ValueError("%s has shape %s, expected %s" % (name, tuple(t.shape), shape))
    _dtype_code(q)
    if k.dtype != q.dtype or v.dtype != q.dtype or (out is not None and out.dtype != q.dtype):
        raise TypeError("q, k, v and out must share one dtype")
    if S.dtype != torch.float32 or log_alpha.dtype != torch.float32 or beta.dtype != torch.float32:
        raise TypeError("S, log_alpha and beta must be float32")
    for t in (q, k, v, log_alpha, beta, S, out):
        if t is not None and not t.is_contiguous():
            raise ValueError("tensors must be contiguous")
    if out is None:
        out = torch.empty((B, H, dv), dtype=q.dtype, device=q.device, pin_memory=_pinned(q))
    with torch.cuda.device(q.device if q.device.type == "cuda" else torch.cuda.current_device()):
        st = getattr(lib, entry)(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(S), _ptr(out),
                                 B, H, dk, dv, _stream_handle(q.device, stream), _dtype_code(q))
    if st != 0:
        raise GdnError(st, entry)
    return out
