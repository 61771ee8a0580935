"""GPU parity of the paged decode (split-KV + combine) against the float64 oracle."""
import numpy as np
import pytest
import torch

from conftest import assert_parity
from oracle import sdpa
from scaled_dot_product_prefill_b200 import api, inputs, workloads

pytestmark = pytest.mark.gpu


def run_decode(p, window=0, scale=None, max_seq_len=None):
    dev = [t.cuda() for t in (p.q, p.k_pool, p.v_pool, p.page_table, p.seq_lens)]
    msl = p.max_seq_len if max_seq_len is None else max_seq_len
    out = api.attn_decode_paged(*dev, max_seq_len=msl, scale=scale, window=window)
    torch.cuda.synchronize()
    return out


SMALL = [
    # N, Hq, Hkv, D, page, seq_lens, window
    (4, 8, 2, 128, 16, [1, 16, 17, 300], 0),
    (3, 4, 4, 64, 16, [5, 513, 1000], 0),
    (2, 8, 1, 128, 32, [700, 33], 0),            # MQA, 32-token pages
    (3, 16, 2, 128, 64, [2000, 64, 65], 0),      # group of 8, 64-token pages
    (5, 32, 8, 128, 16, [4096, 1, 511, 512, 2500], 0),
    (4, 8, 2, 128, 16, [300, 1200, 20, 4000], 100),   # sliding window over the cache
    (2, 8, 4, 64, 16, [1, 0], 0),                # an empty cache gives zeros
    (3, 16, 4, 64, 16, [2100, 47, 900], 0),      # group of 4 at D = 64 (two score pieces per lane)
]


@pytest.mark.parametrize("case", SMALL, ids=[str(c[:5]) for c in SMALL])
def test_decode_matches_oracle(case):
    N, Hq, Hkv, D, page, lens, window = case
    p = inputs.paged_inputs(N, Hq, Hkv, D, page, seed=len(lens) * 7 + D, seq_lens=lens, spare_pages=3,
                            poison=True)
    out = run_decode(p, window)
    assert api.attn_device_status(clear=True) == 0
    ref = sdpa.decode_paged(p.q, p.k_pool, p.v_pool, p.page_table, p.seq_lens, page, 1 / np.sqrt(D), window)
    assert_parity(out, ref, "bf16", str(case))


def test_paged_decode_workload_full():
    spec = workloads.WORKLOADS["paged_decode_gqa"]
    p = inputs.paged_inputs(spec.N, spec.Hq, spec.Hkv, spec.D, spec.page_size, spec.seed, len_range=spec.len_range)
    out = run_decode(p, spec.window, spec.scale)
    assert api.attn_device_status(clear=True) == 0
    ref = sdpa.decode_paged(p.q, p.k_pool, p.v_pool, p.page_table, p.seq_lens, spec.page_size, spec.scale,
                            spec.window)
    assert_parity(out, ref, "bf16", spec.name, report=True)


def test_page_permutation_and_poison_do_not_change_the_result():
    p = inputs.paged_inputs(6, 16, 4, 128, 16, seed=21, seq_lens=[33, 1000, 17, 4097, 250, 64])
    base = run_decode(p)
    # same cache, pages moved to other physical slots, unused pages poisoned with NaN
    rng = np.random.default_rng(0)
    extra = 7
    perm = torch.as_tensor(rng.permutation(p.num_pages + extra))
    k2 = torch.full((p.num_pages + extra,) + tuple(p.k_pool.shape[1:]), float("nan"), dtype=p.k_pool.dtype)
    v2 = k2.clone()
    k2[perm[:p.num_pages]] = p.k_pool
    v2[perm[:p.num_pages]] = p.v_pool
    t2 = torch.where(p.page_table >= 0, perm[p.page_table.clamp(min=0).long()].to(torch.int32), p.page_table)
    q2 = inputs.PagedInputs(p.q, k2, v2, t2.contiguous(), p.seq_lens, 16, p.used_pages, 0)
    moved = run_decode(q2)
    assert torch.equal(base, moved)


def test_decode_equals_last_row_of_causal_prefill():
    """The cache path and the recompute path give the same last-token output (within bf16 tolerance)."""
    L, Hq, Hkv, D = 777, 8, 2, 128
    pre = inputs.prefill_inputs(1, Hq, Hkv, L, L, D, seed=4)
    full = api.attn_prefill(pre.q.cuda(), pre.k.cuda(), pre.v.cuda(), causal=True)
    page = 16
    npg = (L + page - 1) // page
    k_pool = torch.zeros(npg, Hkv, page, D, dtype=torch.bfloat16)
    v_pool = torch.zeros_like(k_pool)
    order = torch.randperm(npg, generator=torch.Generator().manual_seed(1))
    for t in range(0, L, page):
        n = min(page, L - t)
        k_pool[order[t // page], :, :n] = pre.k[0, :, t:t + n]
        v_pool[order[t // page], :, :n] = pre.v[0, :, t:t + n]
    p = inputs.PagedInputs(pre.q[0, :, L - 1].contiguous()[None], k_pool, v_pool,
                           order.to(torch.int32)[None].contiguous(), torch.tensor([L], dtype=torch.int32), page,
                           npg, 0)
    dec = run_decode(p)
    ref = sdpa.attention_rows(pre.q[0, 0, L - 1][None], pre.k[0, 0], pre.v[0, 0], [L - 1], L, 1 / np.sqrt(D),
                              True)  # head 0, anchored to the oracle
    assert_parity(dec[0, :1], ref[:1], "bf16", "decode vs oracle")
    assert (dec[0].float() - full[0, :, L - 1].float()).abs().max() < 2e-2


def test_out_of_pool_page_is_reported_not_read():
    p = inputs.paged_inputs(2, 8, 2, 128, 16, seed=2, seq_lens=[100, 40])
    table = p.page_table.clone()
    table[0, 2] = p.num_pages + 1000     # outside the pool
    bad = inputs.PagedInputs(p.q, p.k_pool, p.v_pool, table, p.seq_lens, 16, p.used_pages, 0)
    api.attn_device_status(clear=True)
    out = run_decode(bad)
    assert api.attn_device_status(clear=True) == 5     # ATTN_ERR_BAD_PAGE
    assert torch.isfinite(out.float()).all()
    # the other sequence is untouched by the bad entry
    ref = sdpa.decode_paged(p.q, p.k_pool, p.v_pool, p.page_table, p.seq_lens, 16, 1 / np.sqrt(128))
    assert_parity(out[1:], ref[1:], "bf16", "good sequence")


def test_sequence_longer_than_hint_is_reported():
    p = inputs.paged_inputs(2, 8, 2, 128, 16, seed=3, seq_lens=[600, 100])
    api.attn_device_status(clear=True)
    run_decode(p, max_seq_len=300)
    assert api.attn_device_status(clear=True) == 5


def test_long_and_short_sequences_in_one_batch():
    """A 70k-token sequence makes the workspace hold 137 splits (of 512 keys) per row; the short sequences
    beside it take the combine's one-round-trip path (at most 16 splits, no window), the long one the
    general path."""
    p = inputs.paged_inputs(4, 8, 2, 128, 16, seed=78, seq_lens=[70001, 300, 1, 3000], spare_pages=4, poison=True)
    out = run_decode(p)
    assert api.attn_device_status(clear=True) == 0
    ref = sdpa.decode_paged(p.q, p.k_pool, p.v_pool, p.page_table, p.seq_lens, 16, 1 / np.sqrt(128))
    assert_parity(out, ref, "bf16", "long and short")


def test_long_context_decode_merges_more_than_32_splits():
    """Two sequences of up to 70k tokens take 274 splits of 256 keys: the combine walks them in blocks of 32."""
    p = inputs.paged_inputs(2, 8, 2, 128, 16, seed=77, seq_lens=[40000, 70001], spare_pages=4, poison=True)
    out = run_decode(p)
    assert api.attn_device_status(clear=True) == 0
    ref = sdpa.decode_paged(p.q, p.k_pool, p.v_pool, p.page_table, p.seq_lens, 16, 1 / np.sqrt(128))
    assert_parity(out, ref, "bf16", "long context")
    # with a window the first split is not split 0
    out_w = run_decode(p, window=30000)
    ref_w = sdpa.decode_paged(p.q, p.k_pool, p.v_pool, p.page_table, p.seq_lens, 16, 1 / np.sqrt(128), 30000)
    assert_parity(out_w, ref_w, "bf16", "long context, window")
