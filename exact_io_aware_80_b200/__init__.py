"""Exact IO-aware attention on one B200: PyTorch-facing wrappers of libfa.so.

The wrappers only check tensor metadata, allocate outputs and workspaces with
PyTorch, and pass raw device pointers plus the current CUDA stream to the C
entry points of the same names (see ``_lib``).  Every step of the attention
computation runs in the CUDA kernels of libfa.so; there is no CPU or PyTorch
fallback, and calling any of these without the built library or without a
CUDA device raises.

Layout (BSHD): q, o [B, Nq, Hq, d]; k, v [B, Nk, Hkv, d]; lse [B, Hq, Nq] fp32.
"""
from __future__ import annotations

import math

from . import _lib
from ._lib import (FAError, fa_bwd, fa_bwd_dkdv, fa_bwd_dq, fa_bwd_preprocess, fa_bwd_workspace_bytes,  # noqa: F401
                   fa_decode_chunk, fa_decode_combine, fa_decode_num_splits, fa_decode_splitkv,
                   fa_decode_workspace_bytes, fa_fp8_quantize_qk, fa_fp8_quantize_qkv, fa_fp8_quantize_v,
                   fa_fp8_v_workspace_bytes, fa_fwd,
                   fa_bwd_dropout, fa_fwd_blocksparse, fa_fwd_dropout, fa_fwd_fp8, fa_get_device_status, fa_version)

__all__ = [
    "attention_fwd", "attention_bwd", "decode", "decode_splitkv", "decode_combine", "device_status",
    "fa_fwd", "fa_bwd", "fa_bwd_preprocess", "fa_bwd_dkdv", "fa_bwd_dq", "fa_decode_splitkv", "fa_decode_combine", "fa_decode_num_splits",
    "fa_decode_workspace_bytes", "fa_bwd_workspace_bytes", "fa_decode_chunk", "fa_get_device_status",
    "fp8_quantize_qk", "fp8_quantize_v", "fp8_quantize_qkv", "attention_fwd_fp8", "fa_fp8_quantize_qk",
    "fa_fp8_quantize_qkv", "fa_fp8_quantize_v",
    "fa_fp8_v_workspace_bytes", "fa_fwd_fp8", "attention_fwd_blocksparse", "fa_fwd_blocksparse",
    "attention_fwd_dropout", "attention_bwd_dropout", "fa_fwd_dropout", "fa_bwd_dropout", "FAError",
]


def _torch():
    import torch
    return torch


def _dt(t):
    torch = _torch()
    if t.dtype == torch.bfloat16:
        return _lib.FA_BF16
    if t.dtype == torch.float16:
        return _lib.FA_FP16
    raise TypeError(f"attention tensors must be fp16 or bf16, got {t.dtype}")


def _dev(*ts):
    for t in ts:
        if not t.is_cuda:
            raise ValueError("libfa.so takes CUDA tensors only (no CPU path)")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous (BSHD)")
    return ts[0].device


def _stream(device):
    return _torch().cuda.current_stream(device).cuda_stream


def attention_fwd(q, k, v, causal: bool = False, scale: float | None = None, out=None, lse=None):
    """O, LSE = softmax(scale q k^T + mask) v, via ``fa_fwd``."""
    torch = _torch()
    dev = _dev(q, k, v)
    B, Nq, Hq, d = q.shape
    _, Nk, Hkv, _ = k.shape
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    o = torch.empty_like(q) if out is None else out
    l = torch.empty(B, Hq, Nq, device=dev, dtype=torch.float32) if lse is None else lse
    fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), l.data_ptr(), B, Hq, Hkv, Nq, Nk, d,
           causal, scale, _dt(q), _stream(dev))
    return o, l


def attention_fwd_dropout(q, k, v, p_drop: float, seed: int, offset: int = 0, causal: bool = False,
                          scale: float | None = None):
    """O, LSE with dropout on P (mask from Philox4x32-10, see include/fa.h), via ``fa_fwd_dropout``."""
    torch = _torch()
    dev = _dev(q, k, v)
    B, Nq, Hq, d = q.shape
    _, Nk, Hkv, _ = k.shape
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    o = torch.empty_like(q)
    lse = torch.empty(B, Hq, Nq, device=dev, dtype=torch.float32)
    fa_fwd_dropout(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, Hq, Hkv, Nq, Nk, d,
                   causal, scale, p_drop, seed, offset, _dt(q), _stream(dev))
    return o, lse


def attention_bwd_dropout(q, k, v, o, do, lse, p_drop: float, seed: int, offset: int = 0, causal: bool = False,
                          scale: float | None = None):
    """dQ, dK, dV for attention_fwd_dropout with the same p_drop, seed and offset, via ``fa_bwd_dropout``."""
    torch = _torch()
    dev = _dev(q, k, v, o, do, lse)
    B, Nq, Hq, d = q.shape
    _, Nk, Hkv, _ = k.shape
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(fa_bwd_workspace_bytes(B, Hq, Nq), device=dev, dtype=torch.uint8)
    fa_bwd_dropout(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(), lse.data_ptr(), dq.data_ptr(),
                   dk.data_ptr(), dv.data_ptr(), ws.data_ptr(), B, Hq, Hkv, Nq, Nk, d, causal, scale, p_drop, seed,
                   offset, _dt(q), _stream(dev))
    return dq, dk, dv


def attention_fwd_blocksparse(q, k, v, block_mask, causal: bool = False, scale: float | None = None):
    """O, LSE of attention restricted to a 128 x 128 block pattern, via ``fa_fwd_blocksparse``.

    ``block_mask``: uint8 CUDA tensor [B, Hq, ceil(Nq/128), ceil(Nk/128)], nonzero = computed.
    """
    torch = _torch()
    dev = _dev(q, k, v, block_mask)
    B, Nq, Hq, d = q.shape
    _, Nk, Hkv, _ = k.shape
    if block_mask.dtype != torch.uint8 or tuple(block_mask.shape) != (B, Hq, -(-Nq // 128), -(-Nk // 128)):
        raise ValueError("block_mask must be uint8 [B, Hq, ceil(Nq/128), ceil(Nk/128)]")
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    o = torch.empty_like(q)
    lse = torch.empty(B, Hq, Nq, device=dev, dtype=torch.float32)
    fa_fwd_blocksparse(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), block_mask.data_ptr(),
                       B, Hq, Hkv, Nq, Nk, d, causal, scale, _dt(q), _stream(dev))
    return o, lse


def fp8_quantize_qk(x, signs=None):
    """E4M3 codes [B, N, H, d] (uint8) and block scales [B, H, ceil(N/128)] of Q or K, via ``fa_fp8_quantize_qk``.

    ``signs``: optional float32 CUDA tensor of d values +-1 (rotation before quantization).
    """
    torch = _torch()
    dev = _dev(x) if signs is None else _dev(x, signs)
    B, N, H, d = x.shape
    x8 = torch.empty(B, N, H, d, device=dev, dtype=torch.uint8)
    sc = torch.empty(B, H, (N + 127) // 128, device=dev, dtype=torch.float32)
    fa_fp8_quantize_qk(x.data_ptr(), x8.data_ptr(), sc.data_ptr(), 0 if signs is None else signs.data_ptr(),
                       B, H, N, d, _dt(x), _stream(dev))
    return x8, sc


def fp8_quantize_v(v):
    """Transposed E4M3 codes [B, Hkv, d, Nk_pad] and per-head scales [B, Hkv] of V, via ``fa_fp8_quantize_v``."""
    torch = _torch()
    dev = _dev(v)
    B, Nk, H, d = v.shape
    v8t = torch.empty(B, H, d, (Nk + 15) // 16 * 16, device=dev, dtype=torch.uint8)
    sc = torch.empty(B, H, device=dev, dtype=torch.float32)
    ws = torch.empty(fa_fp8_v_workspace_bytes(B, H, Nk), device=dev, dtype=torch.uint8)
    fa_fp8_quantize_v(v.data_ptr(), v8t.data_ptr(), sc.data_ptr(), ws.data_ptr(), B, H, Nk, d, _dt(v), _stream(dev))
    return v8t, sc


def fp8_quantize_qkv(q, k, v, signs=None):
    """Q, K, V quantized together (``fa_fp8_quantize_qkv``): (q8, q_scale, k8, k_scale, v8t, v_scale)."""
    torch = _torch()
    dev = _dev(q, k, v) if signs is None else _dev(q, k, v, signs)
    B, Nq, Hq, d = q.shape
    _, Nk, Hkv, _ = k.shape
    q8 = torch.empty(B, Nq, Hq, d, device=dev, dtype=torch.uint8)
    k8 = torch.empty(B, Nk, Hkv, d, device=dev, dtype=torch.uint8)
    v8t = torch.empty(B, Hkv, d, (Nk + 15) // 16 * 16, device=dev, dtype=torch.uint8)
    qs = torch.empty(B, Hq, (Nq + 127) // 128, device=dev, dtype=torch.float32)
    ks = torch.empty(B, Hkv, (Nk + 127) // 128, device=dev, dtype=torch.float32)
    vs = torch.empty(B, Hkv, device=dev, dtype=torch.float32)
    ws = torch.empty(fa_fp8_v_workspace_bytes(B, Hkv, Nk), device=dev, dtype=torch.uint8)
    fa_fp8_quantize_qkv(q.data_ptr(), k.data_ptr(), v.data_ptr(), q8.data_ptr(), k8.data_ptr(), v8t.data_ptr(),
                        qs.data_ptr(), ks.data_ptr(), vs.data_ptr(), 0 if signs is None else signs.data_ptr(),
                        ws.data_ptr(), B, Hq, Hkv, Nq, Nk, d, _dt(q), _stream(dev))
    return q8, qs, k8, ks, v8t, vs


def attention_fwd_fp8(q8, q_scale, k8, k_scale, v8t, v_scale, Nk: int, causal: bool = False,
                      scale: float | None = None, rotated: bool = False, out_dtype=None):
    """FP8 forward (``fa_fwd_fp8``) on quantized operands; returns O [B, Nq, Hq, d] and LSE [B, Hq, Nq]."""
    torch = _torch()
    dev = _dev(q8, q_scale, k8, k_scale, v8t, v_scale)
    B, Nq, Hq, d = q8.shape
    Hkv = k8.shape[2]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    out_dtype = torch.bfloat16 if out_dtype is None else out_dtype
    o = torch.empty(B, Nq, Hq, d, device=dev, dtype=out_dtype)
    lse = torch.empty(B, Hq, Nq, device=dev, dtype=torch.float32)
    fa_fwd_fp8(q8.data_ptr(), q_scale.data_ptr(), k8.data_ptr(), k_scale.data_ptr(), v8t.data_ptr(),
               v_scale.data_ptr(), o.data_ptr(), lse.data_ptr(), B, Hq, Hkv, Nq, Nk, d, causal, scale, rotated,
               _dt(o), _stream(dev))
    return o, lse


def attention_bwd(q, k, v, o, do, lse, causal: bool = False, scale: float | None = None, workspace=None,
                  dq=None, dk=None, dv=None):
    """dQ, dK, dV of sum(dO * O), P recomputed from ``lse``, via ``fa_bwd``."""
    torch = _torch()
    dev = _dev(q, k, v, o, do, lse)
    B, Nq, Hq, d = q.shape
    _, Nk, Hkv, _ = k.shape
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if workspace is None:
        workspace = torch.empty(fa_bwd_workspace_bytes(B, Hq, Nq), device=dev, dtype=torch.uint8)
    fa_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(), lse.data_ptr(), dq.data_ptr(),
           dk.data_ptr(), dv.data_ptr(), workspace.data_ptr(), B, Hq, Hkv, Nq, Nk, d, causal, scale, _dt(q),
           _stream(dev))
    return dq, dk, dv


def decode_splitkv(q, k_cache, v_cache, seqlens_k, num_splits: int, scale: float | None = None, workspace=None):
    """Per-split partials of one-token decode (``fa_decode_splitkv``); returns the workspace."""
    torch = _torch()
    dev = _dev(q, k_cache, v_cache, seqlens_k)
    B, _, Hq, d = q.shape
    _, Nk_max, Hkv, _ = k_cache.shape
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    if workspace is None:
        workspace = torch.empty(fa_decode_workspace_bytes(B, Hq, num_splits, d), device=dev, dtype=torch.uint8)
    fa_decode_splitkv(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), seqlens_k.data_ptr(), B, Hq, Hkv,
                      Nk_max, d, scale, num_splits, workspace.data_ptr(), _dt(q), _stream(dev))
    return workspace


def decode_combine(workspace, seqlens_k, B, Hq, d, num_splits, dtype, out=None, lse=None):
    """Log-sum-exp merge of the split partials (``fa_decode_combine``)."""
    torch = _torch()
    dev = _dev(workspace, seqlens_k)
    o = torch.empty(B, 1, Hq, d, device=dev, dtype=dtype) if out is None else out
    l = torch.empty(B, Hq, 1, device=dev, dtype=torch.float32) if lse is None else lse
    dt = _lib.FA_BF16 if dtype == torch.bfloat16 else _lib.FA_FP16
    fa_decode_combine(workspace.data_ptr(), o.data_ptr(), l.data_ptr(), seqlens_k.data_ptr(), B, Hq, num_splits, d,
                      dt, _stream(dev))
    return o, l


def decode(q, k_cache, v_cache, seqlens_k, num_splits: int | None = None, scale: float | None = None,
           workspace=None, out=None, lse=None):
    """One-token split-KV decode: partial pass then combine."""
    B, _, Hq, d = q.shape
    _, Nk_max, Hkv, _ = k_cache.shape
    if num_splits is None:
        num_splits = fa_decode_num_splits(B, Hkv, Nk_max, d, 0)
    ws = decode_splitkv(q, k_cache, v_cache, seqlens_k, num_splits, scale, workspace)
    return decode_combine(ws, seqlens_k, B, Hq, d, num_splits, q.dtype, out, lse)


def device_status(stream=None) -> int:
    """Synchronise and return (then clear) the kernels' device status word."""
    s = _stream(_torch().cuda.current_device()) if stream is None else stream
    return fa_get_device_status(s)
