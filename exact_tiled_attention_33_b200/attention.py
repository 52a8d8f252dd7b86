"""Python binding of libfattn: argument marshalling only.

Every step of the attention computation runs in the library's CUDA kernels; this module
checks tensor shapes/dtypes/devices, allocates outputs with PyTorch (device memory is
PyTorch's job here) and passes raw pointers and the current CUDA stream to the C ABI.

API shapes follow the pages' usage: ``flash_attn_func(q, k, v, softmax_scale, causal)``
on [batch, seqlen, heads, head_dim] tensors and ``flash_attn_varlen_func`` on packed
[total, heads, head_dim] tensors with cu_seqlens (page "FlashAttention-2的核心设计原理",
sections "FlashAttention-2在PyTorch中的安装与使用" and
"变长序列处理与flash_attn_varlen_func"); the backward pass is reached through autograd
(section "FlashAttention-2反向传播与多GPU训练").
"""

from __future__ import annotations

import math
from typing import Optional

import torch

from . import _lib

_DTYPES = {torch.bfloat16: _lib.FA_BF16, torch.float16: _lib.FA_FP16}


def _stream(t: torch.Tensor) -> int:
    return torch.cuda.current_stream(t.device).cuda_stream


def _check(*ts: torch.Tensor):
    dev = ts[0].device
    dt = ts[0].dtype
    if dev.type != "cuda":
        raise ValueError("attention tensors must be CUDA tensors")
    if dt not in _DTYPES:
        raise ValueError(f"unsupported dtype {dt}; use bfloat16 or float16")
    for t in ts:
        if t.device != dev or t.dtype != dt:
            raise ValueError("all attention tensors must share device and dtype")
        if not t.is_contiguous():
            raise ValueError("attention tensors must be contiguous")
    return _DTYPES[dt]


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def fwd(q, k, v, softmax_scale=None, causal=False, out=None, lse=None):
    """Dense forward. q, k, v: [B, N, H, d]. Returns (o [B,N,H,d], lse [B,H,N] fp32)."""
    if q.dim() != 4 or k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must all be [B, N, H, d] with equal shapes")
    dtype = _check(q, k, v)
    B, N, H, d = q.shape
    scale = 1.0 / math.sqrt(d) if softmax_scale is None else float(softmax_scale)
    o = torch.empty_like(q) if out is None else out
    lse_t = torch.empty((B, H, N), device=q.device, dtype=torch.float32) if lse is None else lse
    lib = _lib.load()
    with torch.cuda.device(q.device):
        st = lib.fa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse_t), B, N, H, d, scale,
                        int(bool(causal)), dtype, _stream(q))
    _lib.check(st, "fa_fwd")
    return o, lse_t


def fwd_f32out(q, k, v, softmax_scale=None, causal=False, window=None):
    """Test hook: fa_fwd (window None) or fa_fwd_local with O returned in fp32 before
    rounding (fa_selftest_fwd_f32).  Returns (o [B,N,H,d] fp32, lse [B,H,N] fp32)."""
    if q.dim() != 4 or k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must all be [B, N, H, d] with equal shapes")
    dtype = _check(q, k, v)
    B, N, H, d = q.shape
    scale = 1.0 / math.sqrt(d) if softmax_scale is None else float(softmax_scale)
    o = torch.empty(q.shape, device=q.device, dtype=torch.float32)
    lse_t = torch.empty((B, H, N), device=q.device, dtype=torch.float32)
    lib = _lib.load()
    with torch.cuda.device(q.device):
        wl, wr = (-1, 0 if causal else -1) if window is None else _window(window)
        st = lib.fa_selftest_fwd_f32(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse_t), B, N, H,
                                     d, scale, wl, wr, dtype, _stream(q))
    _lib.check(st, "fa_selftest_fwd_f32")
    return o, lse_t


def varlen_fwd(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k,
               softmax_scale=None, causal=False, out=None, lse=None):
    """Varlen forward. q: [total_q, H, d]; k, v: [total_k, H, d]; cu_seqlens int32 on device.
    Returns (o [total_q,H,d], lse [H,total_q] fp32)."""
    if q.dim() != 3 or k.dim() != 3 or k.shape != v.shape or q.shape[1:] != k.shape[1:]:
        raise ValueError("q must be [total_q, H, d] and k, v [total_k, H, d]")
    dtype = _check(q, k, v)
    for cu in (cu_seqlens_q, cu_seqlens_k):
        if cu.dtype != torch.int32 or cu.device != q.device or not cu.is_contiguous():
            raise ValueError("cu_seqlens must be contiguous int32 tensors on q's device")
    if cu_seqlens_q.numel() != cu_seqlens_k.numel() or cu_seqlens_q.numel() < 1:
        raise ValueError("cu_seqlens_q and cu_seqlens_k must have num_seqs + 1 entries")
    total_q, H, d = q.shape
    total_k = k.shape[0]
    scale = 1.0 / math.sqrt(d) if softmax_scale is None else float(softmax_scale)
    o = torch.empty_like(q) if out is None else out
    lse_t = torch.empty((H, total_q), device=q.device, dtype=torch.float32) if lse is None else lse
    lib = _lib.load()
    with torch.cuda.device(q.device):
        st = lib.fa_varlen_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse_t), _ptr(cu_seqlens_q),
                               _ptr(cu_seqlens_k), int(max_seqlen_q), int(max_seqlen_k), H, d,
                               scale, int(bool(causal)), cu_seqlens_q.numel() - 1, total_q,
                               total_k, dtype, _stream(q))
    _lib.check(st, "fa_varlen_fwd")
    return o, lse_t


def bwd_workspace(B, N, H, d, device) -> torch.Tensor:
    n = _lib.load().fa_bwd_workspace_size(B, N, H, d)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device)


def varlen_bwd_workspace(total_q, H, d, device) -> torch.Tensor:
    n = _lib.load().fa_varlen_bwd_workspace_size(total_q, H, d)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device)


def _bwd_dense(name, q, k, v, o, lse, dout, scale, window, workspace, dq, dk, dv, deterministic):
    dtype = _check(q, k, v, o, dout)
    B, N, H, d = q.shape
    wl, wr = window
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    ws = bwd_workspace(B, N, H, d, q.device) if workspace is None else workspace
    lib = _lib.load()
    fn = lib.fa_bwd_deterministic if deterministic else lib.fa_bwd_local
    with torch.cuda.device(q.device):
        st = fn(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk),
                _ptr(dv), B, N, H, d, scale, wl, wr, _ptr(ws), ws.numel(), dtype, _stream(q))
    _lib.check(st, "fa_bwd_deterministic" if deterministic else name)
    return dq, dk, dv


def bwd(q, k, v, o, lse, dout, softmax_scale=None, causal=False, workspace=None,
        dq=None, dk=None, dv=None, deterministic=False):
    """Dense backward. Returns (dq, dk, dv), each [B, N, H, d].  deterministic=True runs the
    two-pass backward (fa_bwd_deterministic): bitwise-reproducible dQ."""
    if deterministic:
        d = q.shape[-1]
        scale = 1.0 / math.sqrt(d) if softmax_scale is None else float(softmax_scale)
        return _bwd_dense("fa_bwd", q, k, v, o, lse, dout, scale, (-1, 0 if causal else -1),
                          workspace, dq, dk, dv, True)
    dtype = _check(q, k, v, o, dout)
    B, N, H, d = q.shape
    scale = 1.0 / math.sqrt(d) if softmax_scale is None else float(softmax_scale)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    ws = bwd_workspace(B, N, H, d, q.device) if workspace is None else workspace
    lib = _lib.load()
    with torch.cuda.device(q.device):
        st = lib.fa_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq),
                        _ptr(dk), _ptr(dv), B, N, H, d, scale, int(bool(causal)), _ptr(ws),
                        ws.numel(), dtype, _stream(q))
    _lib.check(st, "fa_bwd")
    return dq, dk, dv


def bwd_noalloc(q, k, v, o, lse, dout, softmax_scale=None, causal=False, dq=None, dk=None,
                dv=None):
    """Dense backward without a workspace (fa_bwd_noalloc): D lives in the library's fixed
    device array, so B*H*N must not exceed its capacity.  Calls on one device must not
    overlap on the GPU."""
    dtype = _check(q, k, v, o, dout)
    B, N, H, d = q.shape
    scale = 1.0 / math.sqrt(d) if softmax_scale is None else float(softmax_scale)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    lib = _lib.load()
    with torch.cuda.device(q.device):
        st = lib.fa_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse),
                                _ptr(dq), _ptr(dk), _ptr(dv), B, N, H, d, scale, int(bool(causal)),
                                dtype, _stream(q))
    _lib.check(st, "fa_bwd_noalloc")
    return dq, dk, dv


def _bwd_varlen_det(q, k, v, o, lse, dout, cu_seqlens_q, cu_seqlens_k, max_seqlen_q,
                    max_seqlen_k, scale, window, workspace, dq, dk, dv):
    dtype = _check(q, k, v, o, dout)
    total_q, H, d = q.shape
    total_k = k.shape[0]
    wl, wr = window
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    ws = varlen_bwd_workspace(total_q, H, d, q.device) if workspace is None else workspace
    lib = _lib.load()
    with torch.cuda.device(q.device):
        st = lib.fa_varlen_bwd_deterministic(
            _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk),
            _ptr(dv), _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), int(max_seqlen_q),
            int(max_seqlen_k), H, d, scale, wl, wr, cu_seqlens_q.numel() - 1, total_q, total_k,
            _ptr(ws), ws.numel(), dtype, _stream(q))
    _lib.check(st, "fa_varlen_bwd_deterministic")
    return dq, dk, dv


def varlen_bwd(q, k, v, o, lse, dout, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k,
               softmax_scale=None, causal=False, workspace=None, dq=None, dk=None, dv=None,
               deterministic=False):
    """Varlen backward. Returns (dq [total_q,H,d], dk, dv [total_k,H,d]).  deterministic=True
    runs fa_varlen_bwd_deterministic."""
    if deterministic:
        d = q.shape[-1]
        scale = 1.0 / math.sqrt(d) if softmax_scale is None else float(softmax_scale)
        return _bwd_varlen_det(q, k, v, o, lse, dout, cu_seqlens_q, cu_seqlens_k, max_seqlen_q,
                               max_seqlen_k, scale, (-1, 0 if causal else -1), workspace, dq, dk,
                               dv)
    dtype = _check(q, k, v, o, dout)
    total_q, H, d = q.shape
    total_k = k.shape[0]
    scale = 1.0 / math.sqrt(d) if softmax_scale is None else float(softmax_scale)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    ws = varlen_bwd_workspace(total_q, H, d, q.device) if workspace is None else workspace
    lib = _lib.load()
    with torch.cuda.device(q.device):
        st = lib.fa_varlen_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq),
                               _ptr(dk), _ptr(dv), _ptr(cu_seqlens_q), _ptr(cu_seqlens_k),
                               int(max_seqlen_q), int(max_seqlen_k), H, d, scale,
                               int(bool(causal)), cu_seqlens_q.numel() - 1, total_q, total_k,
                               _ptr(ws), ws.numel(), dtype, _stream(q))
    _lib.check(st, "fa_varlen_bwd")
    return dq, dk, dv


# ------------------------------------------------------------------ local attention
# Sliding-window attention (page "FlashAttention技术深度解析" (pwwt.cn/news/595117): CUDA
# backend feature table and the section on local attention).  window = (left, right):
# key j is allowed for query i iff i + (Lk - Lq) - left <= j <= i + (Lk - Lq) + right,
# a negative bound meaning no bound; (-1, 0) is causal, (-1, -1) full attention.

def _window(window):
    left, right = (int(x) for x in window)
    return left, right


def fwd_local(q, k, v, window, softmax_scale=None, out=None, lse=None):
    """Dense sliding-window forward (fa_fwd_local). Returns (o, lse) as fwd."""
    if q.dim() != 4 or k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must all be [B, N, H, d] with equal shapes")
    dtype = _check(q, k, v)
    B, N, H, d = q.shape
    wl, wr = _window(window)
    scale = 1.0 / math.sqrt(d) if softmax_scale is None else float(softmax_scale)
    o = torch.empty_like(q) if out is None else out
    lse_t = torch.empty((B, H, N), device=q.device, dtype=torch.float32) if lse is None else lse
    lib = _lib.load()
    with torch.cuda.device(q.device):
        st = lib.fa_fwd_local(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse_t), B, N, H, d, scale,
                              wl, wr, dtype, _stream(q))
    _lib.check(st, "fa_fwd_local")
    return o, lse_t


def varlen_fwd_local(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k, window,
                     softmax_scale=None, out=None, lse=None):
    """Packed sliding-window forward (fa_varlen_fwd_local). Returns (o, lse) as varlen_fwd."""
    if q.dim() != 3 or k.dim() != 3 or k.shape != v.shape or q.shape[1:] != k.shape[1:]:
        raise ValueError("q must be [total_q, H, d] and k, v [total_k, H, d]")
    dtype = _check(q, k, v)
    for cu in (cu_seqlens_q, cu_seqlens_k):
        if cu.dtype != torch.int32 or cu.device != q.device or not cu.is_contiguous():
            raise ValueError("cu_seqlens must be contiguous int32 tensors on q's device")
    if cu_seqlens_q.numel() != cu_seqlens_k.numel() or cu_seqlens_q.numel() < 1:
        raise ValueError("cu_seqlens_q and cu_seqlens_k must have num_seqs + 1 entries")
    total_q, H, d = q.shape
    total_k = k.shape[0]
    wl, wr = _window(window)
    scale = 1.0 / math.sqrt(d) if softmax_scale is None else float(softmax_scale)
    o = torch.empty_like(q) if out is None else out
    lse_t = torch.empty((H, total_q), device=q.device, dtype=torch.float32) if lse is None else lse
    lib = _lib.load()
    with torch.cuda.device(q.device):
        st = lib.fa_varlen_fwd_local(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse_t),
                                     _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), int(max_seqlen_q),
                                     int(max_seqlen_k), H, d, scale, wl, wr,
                                     cu_seqlens_q.numel() - 1, total_q, total_k, dtype,
                                     _stream(q))
    _lib.check(st, "fa_varlen_fwd_local")
    return o, lse_t


def bwd_local(q, k, v, o, lse, dout, window, softmax_scale=None, workspace=None, dq=None,
              dk=None, dv=None, deterministic=False):
    """Dense sliding-window backward (fa_bwd_local, or fa_bwd_deterministic).
    Returns (dq, dk, dv)."""
    d = q.shape[-1]
    scale = 1.0 / math.sqrt(d) if softmax_scale is None else float(softmax_scale)
    return _bwd_dense("fa_bwd_local", q, k, v, o, lse, dout, scale, _window(window), workspace,
                      dq, dk, dv, deterministic)


def varlen_bwd_local(q, k, v, o, lse, dout, cu_seqlens_q, cu_seqlens_k, max_seqlen_q,
                     max_seqlen_k, window, softmax_scale=None, workspace=None, dq=None, dk=None,
                     dv=None, deterministic=False):
    """Packed sliding-window backward (fa_varlen_bwd_local, or
    fa_varlen_bwd_deterministic). Returns (dq, dk, dv)."""
    if deterministic:
        d = q.shape[-1]
        scale = 1.0 / math.sqrt(d) if softmax_scale is None else float(softmax_scale)
        return _bwd_varlen_det(q, k, v, o, lse, dout, cu_seqlens_q, cu_seqlens_k, max_seqlen_q,
                               max_seqlen_k, scale, _window(window), workspace, dq, dk, dv)
    dtype = _check(q, k, v, o, dout)
    total_q, H, d = q.shape
    total_k = k.shape[0]
    wl, wr = _window(window)
    scale = 1.0 / math.sqrt(d) if softmax_scale is None else float(softmax_scale)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    ws = varlen_bwd_workspace(total_q, H, d, q.device) if workspace is None else workspace
    lib = _lib.load()
    with torch.cuda.device(q.device):
        st = lib.fa_varlen_bwd_local(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse),
                                     _ptr(dq), _ptr(dk), _ptr(dv), _ptr(cu_seqlens_q),
                                     _ptr(cu_seqlens_k), int(max_seqlen_q), int(max_seqlen_k), H,
                                     d, scale, wl, wr, cu_seqlens_q.numel() - 1, total_q, total_k,
                                     _ptr(ws), ws.numel(), dtype, _stream(q))
    _lib.check(st, "fa_varlen_bwd_local")
    return dq, dk, dv


# ------------------------------------------------------------------ FP8 forward
# 8-bit (E4M3) inputs with per-tensor dequantisation factors (pages: FP8 attention with an
# 8-bit quantization strategy on Hopper tensor cores).

def _check_fp8(*ts):
    dev = ts[0].device
    if dev.type != "cuda":
        raise ValueError("attention tensors must be CUDA tensors")
    for t in ts:
        if t.dtype not in (torch.float8_e4m3fn, torch.uint8) or t.device != dev or \
                not t.is_contiguous():
            raise ValueError("FP8 inputs must be contiguous float8_e4m3fn (or uint8) tensors "
                             "on one device")


def fwd_fp8(q8, k8, v8, q_descale, k_descale, v_descale, softmax_scale=None, causal=False,
            out_dtype=torch.bfloat16, out=None, lse=None):
    """Dense FP8 forward (fa_fwd_fp8): q8, k8, v8 [B, N, H, 128] E4M3.
    Returns (o [B,N,H,128] out_dtype, lse [B,H,N] fp32)."""
    if q8.dim() != 4 or k8.shape != q8.shape or v8.shape != q8.shape:
        raise ValueError("q, k, v must all be [B, N, H, d] with equal shapes")
    _check_fp8(q8, k8, v8)
    B, N, H, d = q8.shape
    scale = 1.0 / math.sqrt(d) if softmax_scale is None else float(softmax_scale)
    o = torch.empty(q8.shape, dtype=out_dtype, device=q8.device) if out is None else out
    lse_t = torch.empty((B, H, N), device=q8.device, dtype=torch.float32) if lse is None else lse
    lib = _lib.load()
    with torch.cuda.device(q8.device):
        st = lib.fa_fwd_fp8(_ptr(q8), _ptr(k8), _ptr(v8), _ptr(o), _ptr(lse_t), B, N, H, d, scale,
                            float(q_descale), float(k_descale), float(v_descale),
                            int(bool(causal)), _DTYPES[o.dtype], _stream(q8))
    _lib.check(st, "fa_fwd_fp8")
    return o, lse_t


def varlen_fwd_fp8(q8, k8, v8, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k,
                   q_descale, k_descale, v_descale, softmax_scale=None, causal=False,
                   out_dtype=torch.bfloat16, out=None, lse=None):
    """Packed FP8 forward (fa_varlen_fwd_fp8). Returns (o, lse) as varlen_fwd."""
    if q8.dim() != 3 or k8.dim() != 3 or k8.shape != v8.shape or q8.shape[1:] != k8.shape[1:]:
        raise ValueError("q must be [total_q, H, d] and k, v [total_k, H, d]")
    _check_fp8(q8, k8, v8)
    total_q, H, d = q8.shape
    total_k = k8.shape[0]
    scale = 1.0 / math.sqrt(d) if softmax_scale is None else float(softmax_scale)
    o = torch.empty(q8.shape, dtype=out_dtype, device=q8.device) if out is None else out
    lse_t = torch.empty((H, total_q), device=q8.device, dtype=torch.float32) if lse is None else lse
    lib = _lib.load()
    with torch.cuda.device(q8.device):
        st = lib.fa_varlen_fwd_fp8(_ptr(q8), _ptr(k8), _ptr(v8), _ptr(o), _ptr(lse_t),
                                   _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), int(max_seqlen_q),
                                   int(max_seqlen_k), H, d, scale, float(q_descale),
                                   float(k_descale), float(v_descale), int(bool(causal)),
                                   cu_seqlens_q.numel() - 1, total_q, total_k,
                                   _DTYPES[o.dtype], _stream(q8))
    _lib.check(st, "fa_varlen_fwd_fp8")
    return o, lse_t


# ------------------------------------------------------------------ KV-cache decode
# One incremental-decoding step over a KV cache (page "FlashAttention技术深度解析"
# (pwwt.cn/news/595117): KV caches for incremental decoding, paged KV caches).  The Nq
# new tokens are the last Nq positions of each sequence's cache.

def decode_workspace(B, Nq, H, d, max_seqlen_k, device) -> Optional[torch.Tensor]:
    n = _lib.load().fa_decode_workspace_size(B, Nq, H, d, max_seqlen_k)
    return None if n == 0 else torch.empty(n, dtype=torch.uint8, device=device)


def _check_seqlens(t, B, device, name):
    if t.dtype != torch.int32 or t.device != device or not t.is_contiguous() or t.dim() != 1 \
            or t.numel() != B:
        raise ValueError(f"{name} must be a contiguous int32 [B] tensor on q's device")


def decode(q, k_cache, v_cache, cache_seqlens, max_seqlen_k=None, softmax_scale=None,
           causal=True, out=None, lse=None, workspace=None):
    """Decode step over a contiguous cache (fa_decode).  q: [B, Nq, H, d];
    k_cache, v_cache: [B, capacity, H, d]; cache_seqlens: int32 [B] on the device.
    max_seqlen_k: host bound on the lengths (default: the capacity).
    Returns (o [B, Nq, H, d], lse [B, H, Nq] fp32)."""
    if q.dim() != 4 or k_cache.dim() != 4 or k_cache.shape != v_cache.shape or \
            k_cache.shape[0] != q.shape[0] or k_cache.shape[2:] != q.shape[2:]:
        raise ValueError("q must be [B, Nq, H, d] and the caches [B, capacity, H, d]")
    dtype = _check(q, k_cache, v_cache)
    B, Nq, H, d = q.shape
    cap = k_cache.shape[1]
    _check_seqlens(cache_seqlens, B, q.device, "cache_seqlens")
    max_len = cap if max_seqlen_k is None else int(max_seqlen_k)
    scale = 1.0 / math.sqrt(d) if softmax_scale is None else float(softmax_scale)
    o = torch.empty_like(q) if out is None else out
    lse_t = torch.empty((B, H, Nq), device=q.device, dtype=torch.float32) if lse is None else lse
    ws = decode_workspace(B, Nq, H, d, max_len, q.device) if workspace is None else workspace
    lib = _lib.load()
    with torch.cuda.device(q.device):
        st = lib.fa_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(o), _ptr(lse_t),
                           _ptr(cache_seqlens), B, Nq, H, d, cap, max_len, scale,
                           int(bool(causal)), _ptr(ws), 0 if ws is None else ws.numel(), dtype,
                           _stream(q))
    _lib.check(st, "fa_decode")
    return o, lse_t


def decode_paged(q, k_pages, v_pages, block_table, cache_seqlens, max_seqlen_k=None,
                 softmax_scale=None, causal=True, out=None, lse=None, workspace=None):
    """Decode step over a paged cache (fa_decode_paged).  q: [B, Nq, H, d];
    k_pages, v_pages: [num_pages, page_size, H, d]; block_table: int32 [B, max_blocks];
    cache_seqlens: int32 [B].  Returns (o, lse) as decode()."""
    if q.dim() != 4 or k_pages.dim() != 4 or k_pages.shape != v_pages.shape or \
            k_pages.shape[2:] != q.shape[2:]:
        raise ValueError("q must be [B, Nq, H, d] and the pages [num_pages, page_size, H, d]")
    dtype = _check(q, k_pages, v_pages)
    B, Nq, H, d = q.shape
    num_pages, page_size = k_pages.shape[0], k_pages.shape[1]
    if block_table.dtype != torch.int32 or block_table.device != q.device or \
            block_table.dim() != 2 or block_table.shape[0] != B or not block_table.is_contiguous():
        raise ValueError("block_table must be a contiguous int32 [B, max_blocks] tensor")
    _check_seqlens(cache_seqlens, B, q.device, "cache_seqlens")
    max_blocks = block_table.shape[1]
    max_len = max_blocks * page_size if max_seqlen_k is None else int(max_seqlen_k)
    scale = 1.0 / math.sqrt(d) if softmax_scale is None else float(softmax_scale)
    o = torch.empty_like(q) if out is None else out
    lse_t = torch.empty((B, H, Nq), device=q.device, dtype=torch.float32) if lse is None else lse
    ws = decode_workspace(B, Nq, H, d, max_len, q.device) if workspace is None else workspace
    lib = _lib.load()
    with torch.cuda.device(q.device):
        st = lib.fa_decode_paged(_ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(o), _ptr(lse_t),
                                 _ptr(block_table), _ptr(cache_seqlens), B, Nq, H, d, page_size,
                                 num_pages, max_blocks, max_len, scale, int(bool(causal)),
                                 _ptr(ws), 0 if ws is None else ws.numel(), dtype, _stream(q))
    _lib.check(st, "fa_decode_paged")
    return o, lse_t


def device_status(stream: Optional[int] = None) -> int:
    """Synchronise and return the library status word (0 = ok, 4 = a wait timed out)."""
    lib = _lib.load()
    s = torch.cuda.current_stream().cuda_stream if stream is None else stream
    return lib.fa_get_device_status(s)


class FlashAttnFunction(torch.autograd.Function):
    """Autograd wrapper: forward saves (q, k, v, o, lse); backward recomputes P.
    window None: the causal flag decides; else the sliding-window calls."""

    @staticmethod
    def forward(ctx, q, k, v, softmax_scale, causal, window, deterministic):
        if window is None:
            o, lse = fwd(q, k, v, softmax_scale, causal)
        else:
            o, lse = fwd_local(q, k, v, window, softmax_scale)
        ctx.save_for_backward(q, k, v, o, lse)
        ctx.args = (softmax_scale, causal, window, deterministic)
        return o

    @staticmethod
    def backward(ctx, do):
        q, k, v, o, lse = ctx.saved_tensors
        scale, causal, window, det = ctx.args
        if window is None:
            dq, dk, dv = bwd(q, k, v, o, lse, do.contiguous(), scale, causal, deterministic=det)
        else:
            dq, dk, dv = bwd_local(q, k, v, o, lse, do.contiguous(), window, scale,
                                   deterministic=det)
        return dq, dk, dv, None, None, None, None


class FlashAttnVarlenFunction(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, cu_q, cu_k, max_q, max_k, softmax_scale, causal, window,
                deterministic):
        if window is None:
            o, lse = varlen_fwd(q, k, v, cu_q, cu_k, max_q, max_k, softmax_scale, causal)
        else:
            o, lse = varlen_fwd_local(q, k, v, cu_q, cu_k, max_q, max_k, window, softmax_scale)
        ctx.save_for_backward(q, k, v, o, lse, cu_q, cu_k)
        ctx.args = (max_q, max_k, softmax_scale, causal, window, deterministic)
        return o

    @staticmethod
    def backward(ctx, do):
        q, k, v, o, lse, cu_q, cu_k = ctx.saved_tensors
        max_q, max_k, scale, causal, window, det = ctx.args
        if window is None:
            dq, dk, dv = varlen_bwd(q, k, v, o, lse, do.contiguous(), cu_q, cu_k, max_q, max_k,
                                    scale, causal, deterministic=det)
        else:
            dq, dk, dv = varlen_bwd_local(q, k, v, o, lse, do.contiguous(), cu_q, cu_k, max_q,
                                          max_k, window, scale, deterministic=det)
        return dq, dk, dv, None, None, None, None, None, None, None, None


def flash_attn_func(q, k, v, softmax_scale=None, causal=False, window=None,
                    deterministic=False):
    """[batch, seqlen, heads, head_dim] attention with autograd.  window=(left, right)
    selects sliding-window attention (and overrides causal); deterministic=True makes the
    backward bitwise reproducible (the pages' deterministic mode)."""
    return FlashAttnFunction.apply(q, k, v, softmax_scale, causal,
                                   None if window is None else _window(window), deterministic)


def flash_attn_varlen_func(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k,
                           softmax_scale=None, causal=False, window=None, deterministic=False):
    """Packed variable-length attention with autograd (window and deterministic as in
    flash_attn_func)."""
    return FlashAttnVarlenFunction.apply(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q,
                                         max_seqlen_k, softmax_scale, causal,
                                         None if window is None else _window(window),
                                         deterministic)
