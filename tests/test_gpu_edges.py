"""Edge cases of the entry points on the GPU: calls with no keys at all."""
import pytest
import torch

from scaled_dot_product_prefill_b200 import api, inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_prefill_with_no_keys_gives_zeros_and_minus_infinity_lse(dtype):
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    q = inputs.normal((2, 4, 70, 64), seed=1, dtype=dtype).cuda()
    k = torch.empty((2, 2, 0, 64), dtype=tdt, device="cuda")
    v = torch.empty_like(k)
    fn = api.attn_prefill_lse if dtype == "bf16" else api.attn_prefill_f32_lse
    out, lse = fn(q, k, v, causal=False)
    torch.cuda.synchronize()
    assert (out == 0).all()
    assert torch.isneginf(lse).all()


def test_paged_prefill_and_decode_with_empty_caches():
    p = inputs.paged_inputs(3, 8, 2, 128, 16, seed=3, seq_lens=[0, 0, 0], max_pages=2)
    # the pools need at least one page to have an address; nothing is read from them
    kp = torch.zeros((1, 2, 16, 128), dtype=torch.bfloat16, device="cuda")
    table = torch.full((3, 2), -1, dtype=torch.int32, device="cuda")
    lens = torch.zeros(3, dtype=torch.int32, device="cuda")
    q = inputs.normal((3, 8, 5, 128), seed=4).cuda()
    out, lse = api.attn_prefill_paged(q, kp, kp, table, lens, max_seq_len=0, want_lse=True)
    qd = p.q.cuda()
    dec = api.attn_decode_paged(qd, kp, kp, table, lens, max_seq_len=0)
    torch.cuda.synchronize()
    assert api.attn_device_status(clear=True) == 0
    assert (out == 0).all() and torch.isneginf(lse).all()
    assert (dec == 0).all()


def test_append_of_nothing_is_a_no_op():
    kp = torch.zeros((4, 2, 16, 64), dtype=torch.bfloat16, device="cuda")
    before = kp.clone()
    k_new = torch.empty((2, 2, 0, 64), dtype=torch.bfloat16, device="cuda")
    table = torch.zeros((2, 4), dtype=torch.int32, device="cuda")
    lens = torch.zeros(2, dtype=torch.int32, device="cuda")
    api.attn_kv_append(k_new, k_new, kp, kp, table, lens)
    torch.cuda.synchronize()
    assert torch.equal(kp, before)
