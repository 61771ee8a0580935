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
           "attn_prefill_paged", "attn_prefill_host", "attn_decode_paged", "attn_decode_paged_noalloc",
           "attn_decode_step_host",
           "attn_decode_paged_workspace_size", "attn_decode_paged_fp8", "attn_kv_append", "attn_kv_append_fp8",
           "PagePool",
           "attn_device_status", "attn_selftest_wait_timeout", "attn_status_string", "attn_version", "AttnError"]


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
    dev = None
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("tensors must be CUDA tensors on the current device")
        if dev is None:
            dev = torch.cuda.current_device()
        if t.device.index != dev:
            raise ValueError(f"tensor on {t.device}, but the current device is cuda:{dev}")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")


def _expect(t, name, shape, dtype):
    """Host-side check that a tensor argument has the layout the C ABI will assume."""
    if t is None:
        return
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")


def attn_status_string(status: int) -> str:
    return _lib.load().attn_status_string(int(status)).decode()


def attn_version() -> int:
    return int(_lib.load().attn_version())


def _prefill(name, dtype, q, k, v, causal, window, scale, out, stream):
    if q.dtype != dtype or k.dtype != dtype or v.dtype != dtype:
        raise ValueError(f"{name} expects {dtype} q, k, v")
    B, Hq, Sq, D = q.shape
    _, Hkv, Skv, _ = k.shape
    _expect(k, "k", (B, Hkv, Skv, D), dtype)
    _expect(v, "v", (B, Hkv, Skv, D), dtype)
    if out is None:
        out = torch.empty_like(q)
    _expect(out, "out", q.shape, dtype)
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


_COPY_STREAMS: dict = {}
# Host tensors of attn_prefill_host calls whose copies may still be in flight, each
# with an event recorded on the call's stream after its last copy.  The library
# copies them with its own cudaMemcpyAsync calls, which torch's pinned-memory
# allocator does not track, so a host tensor the caller drops could otherwise be
# handed out again (and overwritten or read) while a copy still uses it.
_HOST_IN_FLIGHT: list = []


def _copy_streams(dev):
    """The (host-to-device, device-to-host) copy streams of a device, created on first use."""
    pair = _COPY_STREAMS.get(dev)
    if pair is None:
        with torch.cuda.device(dev):
            pair = (torch.cuda.Stream(), torch.cuda.Stream())
        _COPY_STREAMS[dev] = pair
    return pair


def _release_finished_host_calls():
    while _HOST_IN_FLIGHT and _HOST_IN_FLIGHT[0][0].query():
        _HOST_IN_FLIGHT.pop(0)


def attn_prefill_host(q, k, v, *, causal=False, window=0, scale=None, out=None, chunks=0, device_buffers=None,
                      stream=None, copy_streams="auto"):
    """bf16 prefill whose q [B,Hq,Sq,D], k/v [B,Hkv,Skv,D] and output are host (CPU) tensors.

    The C call copies the inputs to the device, runs the prefill and copies
    the output back, in `chunks` pieces (0: one per 48 MB of input, 2 to 8) so that the copies overlap
    the kernels; page-locked host tensors (``pin_memory()``) are needed for
    the overlap.  `device_buffers` = (q_dev, k_dev, v_dev, out_dev) CUDA
    tensors of the same shapes, allocated here if None.  `copy_streams` =
    (copy_in, copy_out) torch streams, "auto" for two per device, or None to
    copy on `stream`.  The returned host tensor is complete once `stream`
    (default: the current stream) has completed.  This binding keeps q, k,
    v and out referenced until then, so the caller may drop them at once.
    """
    for t, name in ((q, "q"), (k, "k"), (v, "v")):
        if t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous bf16 host tensor")
    B, Hq, Sq, D = q.shape
    _, Hkv, Skv, _ = k.shape
    _expect(k, "k", (B, Hkv, Skv, D), torch.bfloat16)
    _expect(v, "v", (B, Hkv, Skv, D), torch.bfloat16)
    if out is None:
        out = torch.empty(q.shape, dtype=torch.bfloat16, pin_memory=q.is_pinned())
    if out.is_cuda or not out.is_contiguous():
        raise ValueError("out must be a contiguous host tensor")
    _expect(out, "out", q.shape, torch.bfloat16)
    dev = torch.cuda.current_device()
    own_buffers = device_buffers is None
    if own_buffers:
        device_buffers = (torch.empty(q.shape, dtype=torch.bfloat16, device=dev),
                          torch.empty(k.shape, dtype=torch.bfloat16, device=dev),
                          torch.empty(v.shape, dtype=torch.bfloat16, device=dev),
                          torch.empty(q.shape, dtype=torch.bfloat16, device=dev))
    qd, kd, vd, od = device_buffers
    for t, ref, name in ((qd, q, "q_dev"), (kd, k, "k_dev"), (vd, v, "v_dev"), (od, q, "out_dev")):
        _expect(t, name, ref.shape, torch.bfloat16)
    _need_cuda(qd, kd, vd, od)
    if copy_streams == "auto":
        copy_streams = _copy_streams(dev)
    cin, cout = copy_streams if copy_streams is not None else (None, None)
    kernel_stream = torch.cuda.current_stream() if stream is None else stream
    users = [cs for cs in (cin, cout) if cs is not None]
    if own_buffers and kernel_stream != torch.cuda.current_stream():
        users.append(kernel_stream)   # allocated on the current stream, used on another
    for t in (qd, kd, vd, od):   # the copy streams use the buffers too: keep them from early reuse
        for cs in users:
            t.record_stream(cs)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    _release_finished_host_calls()
    _check("attn_prefill_host",
           _lib.load().attn_prefill_host(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(qd), _ptr(kd), _ptr(vd),
                                         _ptr(od), B, Hq, Hkv, Sq, Skv, D, float(scale), int(bool(causal)),
                                         int(window), int(chunks), _stream(stream),
                                         None if cin is None else ctypes_void(cin.cuda_stream),
                                         None if cout is None else ctypes_void(cout.cuda_stream)))
    # the call joins its copy streams into `stream` before returning: an event
    # recorded there completes after every copy that reads or writes the host tensors
    done = torch.cuda.Event()
    done.record(kernel_stream)
    _HOST_IN_FLIGHT.append((done, (q, k, v, out)))
    return out


def attn_prefill_f32(q, k, v, *, causal=False, window=0, scale=None, out=None, stream=None):
    """fp32 prefill (CUDA-core kernel), same layouts as attn_prefill."""
    return _prefill("attn_prefill_f32", torch.float32, q, k, v, causal, window, scale, out, stream)


def _prefill_lse(name, dtype, q, k, v, causal, window, scale, out, lse, stream):
    if q.dtype != dtype or k.dtype != dtype or v.dtype != dtype:
        raise ValueError(f"{name} expects {dtype} q, k, v")
    B, Hq, Sq, D = q.shape
    _, Hkv, Skv, _ = k.shape
    _expect(k, "k", (B, Hkv, Skv, D), dtype)
    _expect(v, "v", (B, Hkv, Skv, D), dtype)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=q.device)
    _expect(out, "out", q.shape, dtype)
    _expect(lse, "lse", (B, Hq, Sq), torch.float32)
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
    _expect(q, "q", (B, Hq, Sq, D), torch.bfloat16)
    _expect(k_pool, "k_pool", (num_pages, Hkv, page_size, D), torch.bfloat16)
    _expect(v_pool, "v_pool", (num_pages, Hkv, page_size, D), torch.bfloat16)
    _expect(page_table, "page_table", (B, max_pages), torch.int32)
    _expect(seq_lens, "seq_lens", (B,), torch.int32)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=q.device)
    _expect(out, "out", q.shape, torch.bfloat16)
    _expect(lse, "lse", (B, Hq, Sq), torch.float32)
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


def _check_decode_args(q, k_pool, v_pool, page_table, seq_lens, pool_dtype):
    if q.dim() != 3 or k_pool.dim() != 4 or page_table.dim() != 2:
        raise ValueError("q must be [N,Hq,D], the pools [num_pages,Hkv,page_size,D], page_table [N,max_pages]")
    N, Hq, D = q.shape
    num_pages, Hkv, page_size, _ = k_pool.shape
    _expect(q, "q", (N, Hq, D), torch.bfloat16)
    _expect(k_pool, "k_pool", (num_pages, Hkv, page_size, D), pool_dtype)
    _expect(v_pool, "v_pool", (num_pages, Hkv, page_size, D), pool_dtype)
    _expect(page_table, "page_table", (N, page_table.shape[1]), torch.int32)
    _expect(seq_lens, "seq_lens", (N,), torch.int32)


def attn_decode_paged_workspace_size(N, Hq, D, max_seq_len, page_size) -> int:
    return int(_lib.load().attn_decode_paged_workspace_size(int(N), int(Hq), int(D), int(max_seq_len),
                                                            int(page_size)))


def attn_decode_paged(q, k_pool, v_pool, page_table, seq_lens, *, max_seq_len, scale=None, window=0,
                      workspace=None, out=None, stream=None):
    """Paged decode: q [N,Hq,D], pools [P,Hkv,page,D], page_table [N,max_pages] i32, seq_lens [N] i32."""
    N, Hq, D = q.shape
    num_pages, Hkv, page_size, _ = k_pool.shape
    max_pages = page_table.shape[1]
    _check_decode_args(q, k_pool, v_pool, page_table, seq_lens, torch.bfloat16)
    if out is None:
        out = torch.empty_like(q)
    _expect(out, "out", q.shape, torch.bfloat16)
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


def attn_decode_paged_fp8(q, k_pool, v_pool, page_table, seq_lens, *, max_seq_len, k_scale, v_scale, scale=None,
                          window=0, workspace=None, out=None, stream=None):
    """Paged decode over an 8-bit cache: pools are uint8 E4M3 codes [P,Hkv,page,D]; element = scale * e4m3(code)."""
    N, Hq, D = q.shape
    num_pages, Hkv, page_size, _ = k_pool.shape
    max_pages = page_table.shape[1]
    _check_decode_args(q, k_pool, v_pool, page_table, seq_lens, torch.uint8)
    if out is None:
        out = torch.empty_like(q)
    _expect(out, "out", q.shape, torch.bfloat16)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    need = attn_decode_paged_workspace_size(N, Hq, D, max_seq_len, page_size)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    _need_cuda(q, k_pool, v_pool, page_table, seq_lens, out, workspace)
    if page_table.dtype != torch.int32 or seq_lens.dtype != torch.int32:
        raise ValueError("page_table and seq_lens must be int32")
    _check("attn_decode_paged_fp8", _lib.load().attn_decode_paged_fp8(
        _ptr(q), _ptr(k_pool), _ptr(v_pool), _ptr(page_table), _ptr(seq_lens), page_size, N, Hq, Hkv, D,
        num_pages, max_pages, int(max_seq_len), float(scale), float(k_scale), float(v_scale), int(window),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(out), _stream(stream)))
    return out


def attn_decode_step_host(q, k_new, v_new, k_pool, v_pool, page_table, seq_lens, *, max_seq_len, scale=None,
                          window=0, out=None, device_buffers=None, workspace=None, stream=None):
    """One decode step whose inputs and output are host tensors: copy in, append, decode, copy out.

    q [N,Hq,D] and the new token's k_new/v_new [N,Hkv,1,D] are bf16 host
    tensors (page-locked for asynchronous copies); the pools, page_table and
    seq_lens (already counting the new token) are the device-resident cache.
    `device_buffers` = (q_dev, k_new_dev, v_new_dev, out_dev), allocated here
    if None.  The returned host tensor is complete once `stream` (default: the
    current stream) has completed; this binding keeps the host tensors
    referenced until then.
    """
    for t, name in ((q, "q"), (k_new, "k_new"), (v_new, "v_new")):
        if t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous bf16 host tensor")
    N, Hq, D = q.shape
    num_pages, Hkv, page_size, _ = k_pool.shape
    _expect(k_new, "k_new", (N, Hkv, 1, D), torch.bfloat16)
    _expect(v_new, "v_new", (N, Hkv, 1, D), torch.bfloat16)
    _expect(k_pool, "k_pool", (num_pages, Hkv, page_size, D), torch.bfloat16)
    _expect(v_pool, "v_pool", (num_pages, Hkv, page_size, D), torch.bfloat16)
    _expect(page_table, "page_table", (N, page_table.shape[1]), torch.int32)
    _expect(seq_lens, "seq_lens", (N,), torch.int32)
    if out is None:
        out = torch.empty(q.shape, dtype=torch.bfloat16, pin_memory=q.is_pinned())
    if out.is_cuda or not out.is_contiguous():
        raise ValueError("out must be a contiguous host tensor")
    _expect(out, "out", q.shape, torch.bfloat16)
    dev = torch.cuda.current_device()
    own = device_buffers is None
    if own:
        device_buffers = (torch.empty(q.shape, dtype=torch.bfloat16, device=dev),
                          torch.empty(k_new.shape, dtype=torch.bfloat16, device=dev),
                          torch.empty(v_new.shape, dtype=torch.bfloat16, device=dev),
                          torch.empty(q.shape, dtype=torch.bfloat16, device=dev))
    qd, kd, vd, od = device_buffers
    for t, ref, name in ((qd, q, "q_dev"), (kd, k_new, "k_new_dev"), (vd, v_new, "v_new_dev"), (od, q, "out_dev")):
        _expect(t, name, ref.shape, torch.bfloat16)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    need = attn_decode_paged_workspace_size(N, Hq, D, max_seq_len, page_size)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    _need_cuda(qd, kd, vd, od, k_pool, v_pool, page_table, seq_lens, workspace)
    kernel_stream = torch.cuda.current_stream() if stream is None else stream
    if kernel_stream != torch.cuda.current_stream():
        for t in ((qd, kd, vd, od) if own else ()) + ((workspace,) if workspace is not None else ()):
            t.record_stream(kernel_stream)
    _release_finished_host_calls()
    _check("attn_decode_step_host", _lib.load().attn_decode_step_host(
        _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(out), _ptr(qd), _ptr(kd), _ptr(vd), _ptr(od), _ptr(k_pool),
        _ptr(v_pool), _ptr(page_table), _ptr(seq_lens), page_size, N, Hq, Hkv, D, num_pages, page_table.shape[1],
        int(max_seq_len), float(scale), int(window), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _stream(stream)))
    done = torch.cuda.Event()
    done.record(kernel_stream)
    _HOST_IN_FLIGHT.append((done, (q, k_new, v_new, out)))
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
    _check_decode_args(q, k_pool, v_pool, page_table, seq_lens, torch.bfloat16)
    if out is None:
        out = torch.empty_like(q)
    _expect(out, "out", q.shape, torch.bfloat16)
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


def attn_kv_append(k_new, v_new, k_pool, v_pool, page_table, seq_lens, *, stream=None):
    """Write k_new/v_new [B,Hkv,S_new,D] into the pools at positions seq_lens[b] - S_new + i (seq_lens: after)."""
    B, Hkv, S_new, D = k_new.shape
    num_pages, Hkv_p, page_size, D_p = k_pool.shape
    if tuple(v_new.shape) != tuple(k_new.shape) or tuple(v_pool.shape) != tuple(k_pool.shape):
        raise ValueError("k_new/v_new and k_pool/v_pool must have matching shapes")
    if Hkv_p != Hkv or D_p != D:
        raise ValueError("the pools' head count and head dim must match k_new")
    if k_new.dtype != torch.bfloat16 or v_new.dtype != torch.bfloat16 or k_pool.dtype != torch.bfloat16 \
            or v_pool.dtype != torch.bfloat16:
        raise ValueError("k_new, v_new and the pools must be bfloat16")
    _expect(page_table, "page_table", (B, page_table.shape[1]), torch.int32)
    _expect(seq_lens, "seq_lens", (B,), torch.int32)
    _need_cuda(k_new, v_new, k_pool, v_pool, page_table, seq_lens)
    if page_table.dtype != torch.int32 or seq_lens.dtype != torch.int32:
        raise ValueError("page_table and seq_lens must be int32")
    _check("attn_kv_append", _lib.load().attn_kv_append(
        _ptr(k_new), _ptr(v_new), _ptr(k_pool), _ptr(v_pool), _ptr(page_table), _ptr(seq_lens), page_size, B, Hkv,
        S_new, D, num_pages, page_table.shape[1], _stream(stream)))


def attn_kv_append_fp8(k_new, v_new, k_pool, v_pool, page_table, seq_lens, *, k_scale, v_scale, stream=None):
    """attn_kv_append into uint8 E4M3 pools: code = nearest E4M3 to x * (1/scale) (float32, ties to even)."""
    B, Hkv, S_new, D = k_new.shape
    num_pages, Hkv_p, page_size, D_p = k_pool.shape
    if tuple(v_new.shape) != tuple(k_new.shape) or tuple(v_pool.shape) != tuple(k_pool.shape):
        raise ValueError("k_new/v_new and k_pool/v_pool must have matching shapes")
    if Hkv_p != Hkv or D_p != D:
        raise ValueError("the pools' head count and head dim must match k_new")
    if k_new.dtype != torch.bfloat16 or v_new.dtype != torch.bfloat16:
        raise ValueError("k_new and v_new must be bfloat16")
    if k_pool.dtype != torch.uint8 or v_pool.dtype != torch.uint8:
        raise ValueError("the pools must hold uint8 E4M3 codes")
    _expect(page_table, "page_table", (B, page_table.shape[1]), torch.int32)
    _expect(seq_lens, "seq_lens", (B,), torch.int32)
    _need_cuda(k_new, v_new, k_pool, v_pool, page_table, seq_lens)
    if page_table.dtype != torch.int32 or seq_lens.dtype != torch.int32:
        raise ValueError("page_table and seq_lens must be int32")
    _check("attn_kv_append_fp8", _lib.load().attn_kv_append_fp8(
        _ptr(k_new), _ptr(v_new), _ptr(k_pool), _ptr(v_pool), _ptr(page_table), _ptr(seq_lens), page_size, B, Hkv,
        S_new, D, num_pages, page_table.shape[1], float(k_scale), float(v_scale), _stream(stream)))


class PagePool:
    """Host-side page allocator of the C ABI (attn_page_pool_*): page ids and per-sequence page tables.

    ``resize(seq, len)`` grows or shrinks a sequence (all or nothing),
    ``release(seq)`` returns its pages, ``export()`` gives host copies of the
    table [max_seqs, max_pages_per_seq] and lengths [max_seqs], and
    ``upload(page_table, seq_lens)`` copies the changed rows into device int32
    tensors of those shapes on the current stream.
    """

    def __init__(self, num_pages, page_size, max_seqs, max_pages_per_seq):
        import ctypes

        self._lib = _lib.load()
        handle = ctypes.c_void_p()
        _check("attn_page_pool_create", self._lib.attn_page_pool_create(
            int(num_pages), int(page_size), int(max_seqs), int(max_pages_per_seq), ctypes.byref(handle)))
        self._h = handle
        self.num_pages, self.page_size = int(num_pages), int(page_size)
        self.max_seqs, self.max_pages_per_seq = int(max_seqs), int(max_pages_per_seq)

    def close(self):
        if getattr(self, "_h", None) is not None and self._h.value:
            self._lib.attn_page_pool_destroy(self._h)
        self._h = None

    def __del__(self):
        self.close()

    def resize(self, seq, length):
        _check("attn_page_pool_resize", self._lib.attn_page_pool_resize(self._h, int(seq), int(length)))

    def release(self, seq):
        _check("attn_page_pool_release", self._lib.attn_page_pool_release(self._h, int(seq)))

    @property
    def free_pages(self) -> int:
        return int(self._lib.attn_page_pool_free_pages(self._h))

    def seq_len(self, seq) -> int:
        return int(self._lib.attn_page_pool_seq_len(self._h, int(seq)))

    def export(self):
        table = torch.empty((self.max_seqs, self.max_pages_per_seq), dtype=torch.int32)
        lens = torch.empty((self.max_seqs,), dtype=torch.int32)
        _check("attn_page_pool_export", self._lib.attn_page_pool_export(self._h, _ptr(table), _ptr(lens)))
        return table, lens

    def upload(self, page_table, seq_lens, stream=None):
        if tuple(page_table.shape) != (self.max_seqs, self.max_pages_per_seq) or \
                tuple(seq_lens.shape) != (self.max_seqs,):
            raise ValueError("page_table must be [max_seqs, max_pages_per_seq] and seq_lens [max_seqs]")
        if page_table.dtype != torch.int32 or seq_lens.dtype != torch.int32:
            raise ValueError("page_table and seq_lens must be int32")
        _need_cuda(page_table, seq_lens)
        _check("attn_page_pool_upload", self._lib.attn_page_pool_upload(
            self._h, _ptr(page_table), _ptr(seq_lens), _stream(stream)))


def attn_selftest_wait_timeout(limit_ms=20, stream=None):
    """Run a kernel whose bounded wait expires after limit_ms; attn_device_status() then reports a timeout."""
    _check("attn_selftest_wait_timeout", _lib.load().attn_selftest_wait_timeout(int(limit_ms), _stream(stream)))
