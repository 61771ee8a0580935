"""Python binding of the C ABI in include/attn_b200.h, one function per entry point.

Argument marshalling only: tensors become device pointers, the current
torch CUDA stream becomes the stream argument, and a non-OK status raises
``AttnError``.  Every step of the computation runs in libattn_b200.so.
"""
from __future__ import annotations

import math

import torch

from . import _lib
from ._lib import AttnError

__all__ = ["attn_prefill", "attn_prefill_f32", "attn_prefill_lse", "attn_prefill_f32_lse",
           "attn_prefill_paged", "attn_decode_paged", "attn_decode_paged_noalloc",
           "attn_decode_paged_workspace_size",
           "attn_device_status", "attn_status_string", "attn_version", "AttnError"]


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes_void(stream.cuda_stream)


def ctypes_void(x):
    import ctypes

    return ctypes.c_void_p(int(x))


def _ptr(t):
    return None if t is None else ctypes_void(t.data_ptr())


def _check(name, st):
    if st != 0:
        raise AttnError(name, st)


def _need_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("tensors must be CUDA tensors on the current device")
        if t is not None and not t.is_contiguous():
            raise ValueError("tensors must be contiguous")


def attn_status_string(status: int) -> str:
    return _lib.load().attn_status_string(int(status)).decode()


def attn_version() -> int:
    return int(_lib.load().attn_version())


def _prefill(name, dtype, q, k, v, causal, window, scale, out, stream):
    if q.dtype != dtype or k.dtype != dtype or v.dtype != dtype:
        raise ValueError(f"{name} expects {dtype} q, k, v")
    B, Hq, Sq, D = q.shape
    _, Hkv, Skv, _ = k.shape
    if out is None:
        out = torch.empty_like(q)
    _need_cuda(q, k, v, out)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    fn = getattr(_lib.load(), name)
    _check(name, fn(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, Hq, Hkv, Sq, Skv, D, float(scale),
                    int(bool(causal)), int(window), _stream(stream)))
    return out


def attn_prefill(q, k, v, *, causal=False, window=0, scale=None, out=None, stream=None):
    """bf16 prefill: q [B,Hq,Sq,D], k/v [B,Hkv,Skv,D] -> out [B,Hq,Sq,D] (tcgen05 kernel)."""
    return _prefill("attn_prefill", torch.bfloat16, q, k, v, causal, window, scale, out, stream)


def attn_prefill_f32(q, k, v, *, causal=False, window=0, scale=None, out=None, stream=None):
    """fp32 prefill (CUDA-core kernel), same layouts as attn_prefill."""
    return _prefill("attn_prefill_f32", torch.float32, q, k, v, causal, window, scale, out, stream)


def _prefill_lse(name, dtype, q, k, v, causal, window, scale, out, lse, stream):
    if q.dtype != dtype or k.dtype != dtype or v.dtype != dtype:
        raise ValueError(f"{name} expects {dtype} q, k, v")
    B, Hq, Sq, D = q.shape
    _, Hkv, Skv, _ = k.shape
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=q.device)
    _need_cuda(q, k, v, out, lse)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    fn = getattr(_lib.load(), name)
    _check(name, fn(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv, Sq, Skv, D, float(scale),
                    int(bool(causal)), int(window), _stream(stream)))
    return out, lse


def attn_prefill_lse(q, k, v, *, causal=False, window=0, scale=None, out=None, lse=None, stream=None):
    """bf16 prefill returning (out, lse); lse [B,Hq,Sq] fp32 natural-log log-sum-exp per row."""
    return _prefill_lse("attn_prefill_lse", torch.bfloat16, q, k, v, causal, window, scale, out, lse, stream)


def attn_prefill_f32_lse(q, k, v, *, causal=False, window=0, scale=None, out=None, lse=None, stream=None):
    """fp32 prefill returning (out, lse)."""
    return _prefill_lse("attn_prefill_f32_lse", torch.float32, q, k, v, causal, window, scale, out, lse, stream)


def attn_prefill_paged(q, k_pool, v_pool, page_table, seq_lens, *, max_seq_len, causal=True, window=0,
                       scale=None, out=None, lse=None, want_lse=False, stream=None):
    """Chunked prefill over a paged cache: q [B,Hq,Sq,D] are the last Sq tokens of each sequence.

    Returns out, or (out, lse) with want_lse (or an lse tensor given).
    """
    B, Hq, Sq, D = q.shape
    num_pages, Hkv, page_size, _ = k_pool.shape
    max_pages = page_table.shape[1]
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    _need_cuda(q, k_pool, v_pool, page_table, seq_lens, out, lse)
    if page_table.dtype != torch.int32 or seq_lens.dtype != torch.int32:
        raise ValueError("page_table and seq_lens must be int32")
    _check("attn_prefill_paged", _lib.load().attn_prefill_paged(
        _ptr(q), _ptr(k_pool), _ptr(v_pool), _ptr(page_table), _ptr(seq_lens), page_size, B, Hq, Hkv, Sq, D,
        num_pages, max_pages, int(max_seq_len), float(scale), int(bool(causal)), int(window), _ptr(out), _ptr(lse),
        _stream(stream)))
    return (out, lse) if lse is not None else out


def attn_decode_paged_workspace_size(N, Hq, D, max_seq_len, page_size) -> int:
    return int(_lib.load().attn_decode_paged_workspace_size(int(N), int(Hq), int(D), int(max_seq_len),
                                                            int(page_size)))


def attn_decode_paged(q, k_pool, v_pool, page_table, seq_lens, *, max_seq_len, scale=None, window=0,
                      workspace=None, out=None, stream=None):
    """Paged decode: q [N,Hq,D], pools [P,Hkv,page,D], page_table [N,max_pages] i32, seq_lens [N] i32."""
    N, Hq, D = q.shape
    num_pages, Hkv, page_size, _ = k_pool.shape
    max_pages = page_table.shape[1]
    if out is None:
        out = torch.empty_like(q)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    need = attn_decode_paged_workspace_size(N, Hq, D, max_seq_len, page_size)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    _need_cuda(q, k_pool, v_pool, page_table, seq_lens, out, workspace)
    if page_table.dtype != torch.int32 or seq_lens.dtype != torch.int32:
        raise ValueError("page_table and seq_lens must be int32")
    lib = _lib.load()
    _check("attn_decode_paged", lib.attn_decode_paged(
        _ptr(q), _ptr(k_pool), _ptr(v_pool), _ptr(page_table), _ptr(seq_lens), page_size, N, Hq, Hkv, D,
        num_pages, max_pages, int(max_seq_len), float(scale), int(window), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(out), _stream(stream)))
    return out


def attn_decode_paged_noalloc(q, k_pool, v_pool, page_table, seq_lens, *, max_seq_len, scale=None, window=0,
                              out=None, stream=None):
    """attn_decode_paged with the library's fixed 32 MiB scratch instead of a workspace.

    For callers that cannot allocate device memory when they decode.  Calls
    that overlap on the GPU share (and race on) that scratch.
    """
    N, Hq, D = q.shape
    num_pages, Hkv, page_size, _ = k_pool.shape
    max_pages = page_table.shape[1]
    if out is None:
        out = torch.empty_like(q)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    _need_cuda(q, k_pool, v_pool, page_table, seq_lens, out)
    if page_table.dtype != torch.int32 or seq_lens.dtype != torch.int32:
        raise ValueError("page_table and seq_lens must be int32")
    _check("attn_decode_paged_noalloc", _lib.load().attn_decode_paged_noalloc(
        _ptr(q), _ptr(k_pool), _ptr(v_pool), _ptr(page_table), _ptr(seq_lens), page_size, N, Hq, Hkv, D,
        num_pages, max_pages, int(max_seq_len), float(scale), int(window), _ptr(out), _stream(stream)))
    return out


def attn_device_status(clear: bool = True) -> int:
    """Status recorded by the kernels since the last clear (synchronises the device)."""
    return int(_lib.load().attn_device_status(int(bool(clear))))
