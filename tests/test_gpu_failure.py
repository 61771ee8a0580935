"""Failure detection on the GPU without a fault: a bounded wait that nothing completes gives up,
the host reads the timeout from the device error word, and the context stays usable."""
import pytest
import torch

from conftest import assert_parity
from oracle import sdpa
from scaled_dot_product_prefill_b200 import api, inputs

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_reports_a_timeout():
    api.attn_device_status(clear=True)
    api.attn_selftest_wait_timeout(20)           # one thread waits 20 ms for a phase nobody completes
    assert api.attn_device_status(clear=True) == 4    # ATTN_ERR_TIMEOUT
    assert api.attn_device_status(clear=True) == 0    # cleared
    # the context is intact: the next calls run and are right
    inp = inputs.prefill_inputs(1, 4, 2, 300, 300, 64, seed=4)
    out = api.attn_prefill(inp.q.cuda(), inp.k.cuda(), inp.v.cuda(), causal=True)
    torch.cuda.synchronize()
    assert api.attn_device_status(clear=True) == 0
    assert_parity(out, sdpa.attention(inp.q, inp.k, inp.v, 0.125, True, 0), "bf16", "after a timeout")


def test_timeout_is_reported_once_per_clear_and_does_not_leak_into_later_calls():
    api.attn_device_status(clear=True)
    api.attn_selftest_wait_timeout(5)
    api.attn_selftest_wait_timeout(5)
    assert api.attn_device_status(clear=False) == 4   # read without clearing
    assert api.attn_device_status(clear=True) == 4
    p = inputs.paged_inputs(2, 8, 2, 128, 16, seed=6, seq_lens=[100, 200])
    dev = [t.cuda() for t in (p.q, p.k_pool, p.v_pool, p.page_table, p.seq_lens)]
    api.attn_decode_paged(*dev, max_seq_len=200)
    torch.cuda.synchronize()
    assert api.attn_device_status(clear=True) == 0
