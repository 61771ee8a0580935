"""The Python binding's host-side checks: shapes, dtypes and devices are refused before any
pointer reaches the library (a page table with too few rows would otherwise be read out of
bounds by the kernel).  CPU only: the checks run before the first CUDA call."""
import pytest
import torch

from scaled_dot_product_prefill_b200 import api

bf = torch.bfloat16


def t(*shape, dtype=bf):
    return torch.zeros(shape, dtype=dtype)


def test_prefill_refuses_mismatched_shapes_and_dtypes():
    q = t(2, 4, 64, 64)
    with pytest.raises(ValueError, match="k must have shape"):
        api.attn_prefill(q, t(2, 2, 64, 128), t(2, 2, 64, 64))
    with pytest.raises(ValueError, match="v must have shape"):
        api.attn_prefill(q, t(2, 2, 64, 64), t(2, 2, 65, 64))
    with pytest.raises(ValueError, match="out must have shape"):
        api.attn_prefill(q, t(2, 2, 64, 64), t(2, 2, 64, 64), out=t(2, 4, 63, 64))
    with pytest.raises(ValueError, match="expects"):
        api.attn_prefill(q.float(), t(2, 2, 64, 64), t(2, 2, 64, 64))
    with pytest.raises(ValueError, match="lse must have shape"):
        api.attn_prefill_lse(q, t(2, 2, 64, 64), t(2, 2, 64, 64), lse=t(2, 4, 32, dtype=torch.float32))
    with pytest.raises(ValueError, match="CUDA"):
        api.attn_prefill(q, t(2, 2, 64, 64), t(2, 2, 64, 64))


def test_decode_refuses_short_page_tables_and_wrong_pools():
    q = t(4, 8, 128)
    kp = t(10, 2, 16, 128)
    ok_table = t(4, 3, dtype=torch.int32)
    lens = t(4, dtype=torch.int32)
    with pytest.raises(ValueError, match="page_table must have shape"):
        api.attn_decode_paged(q, kp, kp, t(3, 3, dtype=torch.int32), lens, max_seq_len=48)
    with pytest.raises(ValueError, match="seq_lens must have shape"):
        api.attn_decode_paged(q, kp, kp, ok_table, t(3, dtype=torch.int32), max_seq_len=48)
    with pytest.raises(ValueError, match="page_table must be"):
        api.attn_decode_paged(q, kp, kp, ok_table.long(), lens, max_seq_len=48)
    with pytest.raises(ValueError, match="v_pool must have shape"):
        api.attn_decode_paged(q, kp, t(10, 2, 16, 64), ok_table, lens, max_seq_len=48)
    with pytest.raises(ValueError, match="k_pool must be"):
        api.attn_decode_paged_fp8(q, kp, kp, ok_table, lens, max_seq_len=48, k_scale=1, v_scale=1)
    with pytest.raises(ValueError, match="q must have shape|q must be"):
        api.attn_decode_paged(q.float(), kp, kp, ok_table, lens, max_seq_len=48)


def test_paged_prefill_and_append_refuse_mismatched_tables():
    q = t(2, 4, 32, 64)
    kp = t(10, 2, 16, 64)
    with pytest.raises(ValueError, match="page_table must have shape"):
        api.attn_prefill_paged(q, kp, kp, t(1, 4, dtype=torch.int32), t(2, dtype=torch.int32), max_seq_len=64)
    with pytest.raises(ValueError, match="seq_lens must have shape"):
        api.attn_kv_append(t(2, 2, 5, 64), t(2, 2, 5, 64), kp, kp, t(2, 4, dtype=torch.int32),
                           t(1, dtype=torch.int32))
    with pytest.raises(ValueError, match="page_table must have shape"):
        api.attn_kv_append_fp8(t(2, 2, 5, 64), t(2, 2, 5, 64), kp.view(torch.uint8)[..., :64].contiguous(),
                               kp.view(torch.uint8)[..., :64].contiguous(), t(3, 4, dtype=torch.int32),
                               t(2, dtype=torch.int32), k_scale=1, v_scale=1)


def test_host_prefill_refuses_bad_host_tensors_before_touching_the_gpu():
    q, k, v = t(2, 4, 64, 64), t(2, 2, 64, 64), t(2, 2, 64, 64)
    with pytest.raises(ValueError, match="q must be"):
        api.attn_prefill_host(q.float(), k, v)
    with pytest.raises(ValueError, match="k must be"):
        api.attn_prefill_host(q, t(2, 2, 64, 128)[..., ::2], v)      # not contiguous
    with pytest.raises(ValueError, match="v must have shape"):
        api.attn_prefill_host(q, k, t(2, 2, 65, 64))
    with pytest.raises(ValueError, match="out must have shape"):
        api.attn_prefill_host(q, k, v, out=t(2, 4, 64, 32))
