"""GPU tests of one decode step from and to host memory (attn_decode_step_host).

The step copies the new token's query and key/value in, appends the key/value
to the paged cache, decodes and copies the output back.  Its output must equal
the same append and decode run from device buffers bit for bit, the cache
must hold the appended token afterwards, and the output must match the
float64 oracle on the appended cache.
"""
import numpy as np
import pytest
import torch

from conftest import assert_parity
from oracle import sdpa
from scaled_dot_product_prefill_b200 import api, inputs

pytestmark = pytest.mark.gpu

CASES = [
    # N, Hq, Hkv, D, page, seq_lens (after the append)
    (4, 8, 2, 128, 16, [1, 16, 17, 300]),
    (3, 16, 2, 64, 32, [900, 1, 65]),
    (64, 32, 8, 128, 16, None),                  # the decode workload's shape
]


@pytest.mark.parametrize("case", CASES, ids=[str(c[:5]) for c in CASES])
def test_host_step_equals_device_append_and_decode_and_the_oracle(case):
    N, Hq, Hkv, D, page, lens = case
    if lens is None:
        lens = np.random.default_rng(3).integers(512, 8193, N).tolist()
    p = inputs.paged_inputs(N, Hq, Hkv, D, page, seed=N + D, seq_lens=lens, spare_pages=3, poison=True)
    q = inputs.normal((N, Hq, D), seed=91)
    k_new = inputs.normal((N, Hkv, 1, D), seed=92)
    v_new = inputs.normal((N, Hkv, 1, D), seed=93)
    table, sl = p.page_table.cuda(), p.seq_lens.cuda()
    # device path: append, then decode
    kp1, vp1 = p.k_pool.cuda(), p.v_pool.cuda()
    api.attn_kv_append(k_new.cuda(), v_new.cuda(), kp1, vp1, table, sl)
    ref_dev = api.attn_decode_paged(q.cuda(), kp1, vp1, table, sl, max_seq_len=max(lens))
    # host path, on a fresh copy of the cache
    kp2, vp2 = p.k_pool.cuda(), p.v_pool.cuda()
    out = api.attn_decode_step_host(q.pin_memory(), k_new.pin_memory(), v_new.pin_memory(), kp2, vp2, table, sl,
                                    max_seq_len=max(lens))
    torch.cuda.synchronize()
    assert api.attn_device_status(clear=True) == 0
    assert torch.equal(out, ref_dev.cpu())
    # the pools hold NaN in unused slots: compare bit patterns
    assert torch.equal(kp1.view(torch.int16), kp2.view(torch.int16))
    assert torch.equal(vp1.view(torch.int16), vp2.view(torch.int16))
    K = sdpa.append_pages(p.k_pool.double().numpy(), p.page_table.numpy(), lens, k_new.double().numpy(), page)
    V = sdpa.append_pages(p.v_pool.double().numpy(), p.page_table.numpy(), lens, v_new.double().numpy(), page)
    want = sdpa.decode_paged(q, K, V, p.page_table, lens, page, 1 / np.sqrt(D))
    assert_parity(out, want, "bf16", str(case[:5]))


def test_host_step_rejects_device_tensors():
    p = inputs.paged_inputs(2, 8, 2, 128, 16, seed=1, seq_lens=[5, 9])
    q = inputs.normal((2, 8, 128), seed=2)
    kn = inputs.normal((2, 2, 1, 128), seed=3)
    with pytest.raises(ValueError):
        api.attn_decode_step_host(q.cuda(), kn, kn.clone(), p.k_pool.cuda(), p.v_pool.cuda(), p.page_table.cuda(),
                                  p.seq_lens.cuda(), max_seq_len=9)
