"""GPU parity of the chunked prefill over a paged KV cache (attn_prefill_paged)."""
import numpy as np
import pytest
import torch

from conftest import assert_parity
from oracle import sdpa
from scaled_dot_product_prefill_b200 import api, inputs

pytestmark = pytest.mark.gpu


def oracle_paged_prefill(q, p, scale, causal, window):
    """Per sequence: gather its cache from the pool, then the plain definition (bottom-right causal)."""
    B, Hq, Sq, D = q.shape
    out = np.zeros((B, Hq, Sq, D))
    lse = np.full((B, Hq, Sq), -np.inf)
    for b, L in enumerate(p.seq_lens.tolist()):
        if L == 0:
            continue
        K = sdpa.gather_pages(p.k_pool, p.page_table[b].numpy(), L, p.page_size).transpose(1, 0, 2)[None]
        V = sdpa.gather_pages(p.v_pool, p.page_table[b].numpy(), L, p.page_size).transpose(1, 0, 2)[None]
        o, l = sdpa.attention(q[b:b + 1], K, V, scale, causal, window, return_lse=True)
        out[b], lse[b] = o[0], l[0]
    return out, lse


CASES = [
    # B, Hq, Hkv, Sq, D, page, seq_lens, causal, window
    (3, 8, 2, 77, 128, 16, [77, 300, 1000], True, 0),
    (2, 4, 4, 256, 64, 32, [256, 700], True, 0),
    (3, 8, 1, 130, 128, 64, [40, 130, 513], True, 0),      # a cache shorter than the chunk
    (2, 8, 2, 300, 64, 128, [300, 1500], True, 200),       # sliding window
    (2, 4, 2, 200, 128, 256, [600, 201], False, 0),        # non-causal over the whole cache
    (2, 4, 2, 100, 64, 256, [129, 250], True, 0),          # 127 and 6 NaN slots in the last 128-row box
    (1, 2, 2, 64, 64, 16, [0], True, 0),                   # an empty cache
]


@pytest.mark.parametrize("case", CASES, ids=[str(c[:6]) for c in CASES])
def test_paged_prefill_matches_oracle(case):
    B, Hq, Hkv, Sq, D, page, lens, causal, window = case
    # unreferenced pages and the slots past each last token hold NaN: none may reach the output
    p = inputs.paged_inputs(B, Hq, Hkv, D, page, seed=sum(lens) + D, seq_lens=lens, spare_pages=3, poison=True)
    q = inputs.normal((B, Hq, Sq, D), seed=99 + B)
    dev = [t.cuda() for t in (p.k_pool, p.v_pool, p.page_table, p.seq_lens)]
    out, lse = api.attn_prefill_paged(q.cuda(), *dev, max_seq_len=max(max(lens), 1), causal=causal,
                                      window=window, want_lse=True)
    torch.cuda.synchronize()
    assert api.attn_device_status(clear=True) == 0
    ref, ref_lse = oracle_paged_prefill(q, p, 1 / np.sqrt(D), causal, window)
    assert_parity(out, ref, "bf16", str(case))
    got = lse.cpu().double().numpy()
    empty = np.isneginf(ref_lse)
    assert np.array_equal(np.isneginf(got), empty)
    if (~empty).any():
        assert np.abs(got[~empty] - ref_lse[~empty]).max() <= 1e-3


def test_paged_prefill_equals_dense_prefill_on_the_gathered_cache():
    B, Hq, Hkv, D, page, L = 2, 8, 2, 128, 16, 640
    p = inputs.paged_inputs(B, Hq, Hkv, D, page, seed=31, seq_lens=[L, L])
    q = inputs.normal((B, Hq, L, D), seed=5)
    paged = api.attn_prefill_paged(q.cuda(), p.k_pool.cuda(), p.v_pool.cuda(), p.page_table.cuda(),
                                   p.seq_lens.cuda(), max_seq_len=L, causal=True)
    k = torch.stack([torch.from_numpy(sdpa.gather_pages(p.k_pool, p.page_table[b].numpy(), L, page))
                     .permute(1, 0, 2) for b in range(B)]).to(torch.bfloat16)
    v = torch.stack([torch.from_numpy(sdpa.gather_pages(p.v_pool, p.page_table[b].numpy(), L, page))
                     .permute(1, 0, 2) for b in range(B)]).to(torch.bfloat16)
    dense = api.attn_prefill(q.cuda(), k.contiguous().cuda(), v.contiguous().cuda(), causal=True)
    torch.cuda.synchronize()
    # same tiles, same arithmetic: the two paths agree exactly
    assert torch.equal(paged, dense)


def test_paged_prefill_reports_a_bad_page_without_reading_it():
    p = inputs.paged_inputs(2, 4, 2, 64, 16, seed=2, seq_lens=[100, 60])
    table = p.page_table.clone()
    table[0, 3] = p.num_pages + 77
    q = inputs.normal((2, 4, 32, 64), seed=3)
    api.attn_device_status(clear=True)
    out = api.attn_prefill_paged(q.cuda(), p.k_pool.cuda(), p.v_pool.cuda(), table.cuda(), p.seq_lens.cuda(),
                                 max_seq_len=100, causal=True)
    torch.cuda.synchronize()
    assert api.attn_device_status(clear=True) == 5      # ATTN_ERR_BAD_PAGE
    ref, _ = oracle_paged_prefill(q, p, 1 / 8.0, True, 0)
    assert_parity(out[1:], ref[1:], "bf16", "untouched sequence")


def test_paged_prefill_never_reads_entries_past_the_last_page():
    """Table entries after a sequence's last page hold junk (ids out of the pool, or NaN pages): no error, no NaN."""
    lens = [201, 37, 300]
    p = inputs.paged_inputs(3, 4, 2, 128, 16, seed=41, seq_lens=lens, spare_pages=4, poison=True, max_pages=40)
    table = p.page_table.clone()
    spare = sorted(set(range(p.num_pages)) - set(table[table >= 0].tolist()))
    for b, L in enumerate(lens):
        used = (L + 15) // 16
        table[b, used::2] = 1 << 30
        table[b, used + 1::2] = spare[b % len(spare)]
    q = inputs.normal((3, 4, 64, 128), seed=42)
    api.attn_device_status(clear=True)
    out = api.attn_prefill_paged(q.cuda(), p.k_pool.cuda(), p.v_pool.cuda(), table.cuda(), p.seq_lens.cuda(),
                                 max_seq_len=300, causal=False)
    torch.cuda.synchronize()
    assert api.attn_device_status(clear=True) == 0
    ref, _ = oracle_paged_prefill(q, p, 1 / np.sqrt(128), False, 0)
    assert_parity(out, ref, "bf16", "junk past the last page")


def test_paged_prefill_chunk_at_the_end_of_a_long_cache():
    """A 512-token chunk whose cache holds 20k tokens in 64-token pages."""
    L, Sq = 20000, 512
    p = inputs.paged_inputs(1, 8, 2, 128, 64, seed=13, seq_lens=[L], spare_pages=3, poison=True)
    q = inputs.normal((1, 8, Sq, 128), seed=14)
    out = api.attn_prefill_paged(q.cuda(), p.k_pool.cuda(), p.v_pool.cuda(), p.page_table.cuda(), p.seq_lens.cuda(),
                                 max_seq_len=L, causal=True)
    torch.cuda.synchronize()
    assert api.attn_device_status(clear=True) == 0
    ref, _ = oracle_paged_prefill(q, p, 1 / np.sqrt(128), True, 0)
    assert_parity(out, ref, "bf16", "20k cache, 512-token chunk")


def test_chunked_prefill_workload_every_output():
    """The benchmark's chunked prefill, in the launch it times, compared on all B*Hq*Sq*D outputs."""
    import oracle_blocks
    from scaled_dot_product_prefill_b200 import workloads

    spec = workloads.EXTRA_WORKLOADS["chunked_prefill_paged_gqa"]
    p = inputs.paged_inputs(spec.B, spec.Hq, spec.Hkv, spec.D, spec.page_size, spec.seed, seq_lens=[spec.L] * spec.B)
    q = inputs.normal((spec.B, spec.Hq, spec.Sq, spec.D), seed=spec.seed + 1)
    dev = [t.cuda() for t in (p.k_pool, p.v_pool, p.page_table, p.seq_lens)]
    out = api.attn_prefill_paged(q.cuda(), *dev, max_seq_len=spec.L, causal=True, scale=spec.scale)
    torch.cuda.synchronize()
    assert api.attn_device_status(clear=True) == 0
    # each sequence's cache gathered from the pool into [B, Hkv, L, D], then the blocked oracle
    K = np.stack([sdpa.gather_pages(p.k_pool, p.page_table[b].numpy(), spec.L, spec.page_size).transpose(1, 0, 2)
                  for b in range(spec.B)])
    V = np.stack([sdpa.gather_pages(p.v_pool, p.page_table[b].numpy(), spec.L, spec.page_size).transpose(1, 0, 2)
                  for b in range(spec.B)])
    ref = oracle_blocks.attention_all_rows(q, K, V, spec.scale, True, 0)
    assert_parity(out.cpu(), ref, "bf16", spec.name, report=True)
