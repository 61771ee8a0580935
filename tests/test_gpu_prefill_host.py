"""GPU tests of the prefill from and to host memory (attn_prefill_host).

The call cuts the work into pieces of (batch, kv head) pairs and overlaps
their copies with the kernels; each piece's kernel is the same prefill, so
the output must equal the device-buffer prefill bit for bit, for every way
of cutting, and match the float64 oracle.
"""
import numpy as np
import pytest
import torch

from conftest import assert_parity
from oracle import sdpa
from scaled_dot_product_prefill_b200 import api, inputs

pytestmark = pytest.mark.gpu


def host_inputs(shape, seed, pinned=True):
    B, Hq, Hkv, Sq, Skv, D = shape
    inp = inputs.prefill_inputs(B, Hq, Hkv, Sq, Skv, D, seed=seed)
    if pinned:
        return inp, inp.q.pin_memory(), inp.k.pin_memory(), inp.v.pin_memory()
    return inp, inp.q, inp.k, inp.v


def device_reference(inp, causal, window):
    out = api.attn_prefill(inp.q.cuda(), inp.k.cuda(), inp.v.cuda(), causal=causal, window=window)
    torch.cuda.synchronize()
    return out.cpu()


SHAPES = [
    # B, Hq, Hkv, Sq, Skv, D, causal, window, chunks
    ((2, 12, 12, 300, 300, 64), True, 0, 0),       # the library's choice
    ((2, 12, 12, 300, 300, 64), True, 0, 5),       # uneven pieces
    ((2, 12, 12, 300, 300, 64), True, 0, 24),      # one (batch, kv head) pair per piece
    ((3, 8, 2, 257, 257, 128), True, 0, 4),        # GQA; pieces cross batch boundaries
    ((1, 8, 2, 520, 520, 128), True, 129, 2),      # sliding window, one batch element cut by kv head
    ((2, 4, 1, 200, 333, 64), False, 0, 2),        # MQA, Sq < Skv, non-causal
]


@pytest.mark.parametrize("case", SHAPES, ids=[str(c) for c in SHAPES])
def test_host_prefill_equals_device_prefill_and_the_oracle(case):
    shape, causal, window, chunks = case
    inp, qh, kh, vh = host_inputs(shape, seed=sum(shape) + chunks)
    out = api.attn_prefill_host(qh, kh, vh, causal=causal, window=window, chunks=chunks)
    torch.cuda.synchronize()
    assert api.attn_device_status(clear=True) == 0
    assert torch.equal(out, device_reference(inp, causal, window))
    D = shape[-1]
    assert_parity(out, sdpa.attention(inp.q, inp.k, inp.v, 1.0 / np.sqrt(D), causal, window), "bf16", str(case))


def test_single_stream_and_pageable_memory_give_the_same_result():
    shape = (2, 8, 4, 300, 300, 128)
    inp, qh, kh, vh = host_inputs(shape, seed=3)
    ref = device_reference(inp, True, 0)
    a = api.attn_prefill_host(qh, kh, vh, causal=True, chunks=3, copy_streams=None)
    torch.cuda.synchronize()
    _, qp, kp, vp = host_inputs(shape, seed=3, pinned=False)
    b = api.attn_prefill_host(qp, kp, vp, causal=True, chunks=3)
    torch.cuda.synchronize()
    assert torch.equal(a, ref) and torch.equal(b, ref)


def test_back_to_back_calls_reusing_device_buffers():
    """Each call's copies wait for the previous call's kernels on the same stream."""
    shape = (2, 12, 12, 256, 256, 64)
    B, Hq, Hkv, Sq, Skv, D = shape
    bufs = tuple(torch.empty(s, dtype=torch.bfloat16, device="cuda")
                 for s in ((B, Hq, Sq, D), (B, Hkv, Skv, D), (B, Hkv, Skv, D), (B, Hq, Sq, D)))
    outs, refs, hosts = [], [], []
    for seed in (11, 12, 13):
        inp, qh, kh, vh = host_inputs(shape, seed=seed)
        outs.append(api.attn_prefill_host(qh, kh, vh, causal=True, chunks=6, device_buffers=bufs))
        refs.append(inp)
        hosts.append((qh, kh, vh))   # held here until the copies are known to be done
    torch.cuda.synchronize()
    for out, inp in zip(outs, refs):
        assert torch.equal(out, device_reference(inp, True, 0))


def test_dropped_host_inputs_are_kept_until_the_copies_finish():
    """The binding holds the host tensors until the call's stream has passed it.

    The caller drops its pinned inputs right after each call and fills freshly
    pinned buffers of the same size with NaN: had a dropped block been handed
    out again while its copy was still queued, NaN would reach the output.
    """
    shape = (4, 8, 8, 512, 512, 64)
    refs, outs = [], []
    blocker = torch.empty(64 << 20, dtype=torch.uint8, device="cuda")
    for seed in (21, 22, 23, 24):
        blocker.zero_()   # keeps the stream busy, so that the copies are still queued below
        inp, qh, kh, vh = host_inputs(shape, seed=seed)
        outs.append(api.attn_prefill_host(qh, kh, vh, causal=True, chunks=4))
        refs.append(inp)
        del qh, kh, vh
        junk = [torch.full(t.shape, float("nan"), dtype=torch.bfloat16).pin_memory() for t in (inp.q, inp.k, inp.v)]
        del junk
    torch.cuda.synchronize()
    for out, inp in zip(outs, refs):
        assert torch.equal(out, device_reference(inp, True, 0))


def test_no_keys_gives_zeros():
    inp, qh, _, _ = host_inputs((1, 4, 2, 100, 1, 64), seed=5)
    k0 = torch.empty((1, 2, 0, 64), dtype=torch.bfloat16)
    out = api.attn_prefill_host(qh, k0, k0.clone(), causal=False, chunks=2)
    torch.cuda.synchronize()
    assert torch.count_nonzero(out) == 0


def test_rejects_device_tensors_and_bad_pieces():
    inp, qh, kh, vh = host_inputs((1, 4, 2, 64, 64, 64), seed=1)
    with pytest.raises(ValueError):
        api.attn_prefill_host(qh.cuda(), kh, vh)
    with pytest.raises(api.AttnError):
        api.attn_prefill_host(qh, kh, vh, chunks=3)   # only 2 (batch, kv head) pairs
