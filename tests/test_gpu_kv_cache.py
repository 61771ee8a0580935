"""GPU tests of the paged KV cache: the append kernel, and the page pool driving prefill and decode."""
import numpy as np
import pytest
import torch

from conftest import assert_parity
from oracle import sdpa
from scaled_dot_product_prefill_b200 import PagePool, api, inputs

pytestmark = pytest.mark.gpu


def bits(t):
    """Raw 16-bit patterns of a bf16 tensor, as numpy (for bit-exact comparison of copies)."""
    return t.cpu().view(torch.int16).numpy()


APPEND_CASES = [
    # B, Hkv, S_new, D, page, seq_lens after the append
    (64, 8, 1, 128, 16, None),                 # one decode step of the decode workload's shape
    (3, 2, 100, 64, 16, [100, 250, 37]),       # a prefill chunk; sequence 2 is shorter than the chunk
    (2, 4, 300, 128, 64, [300, 1000]),
    (2, 1, 7, 64, 256, [7, 600]),
    (1, 2, 1, 128, 8, [1]),                    # the first token of a sequence
]


@pytest.mark.parametrize("case", APPEND_CASES, ids=[str(c[:5]) for c in APPEND_CASES])
def test_append_is_a_bit_exact_scatter_through_the_page_table(case):
    B, Hkv, S_new, D, page, lens = case
    if lens is None:
        lens = np.random.default_rng(5).integers(1, 3000, B).tolist()
    p = inputs.paged_inputs(B, 1, Hkv, D, page, seed=B + S_new, seq_lens=lens, spare_pages=5, poison=True)
    k_new = inputs.normal((B, Hkv, S_new, D), seed=77)
    v_new = inputs.normal((B, Hkv, S_new, D), seed=78)
    kp, vp = p.k_pool.cuda(), p.v_pool.cuda()
    api.attn_device_status(clear=True)
    api.attn_kv_append(k_new.cuda(), v_new.cuda(), kp, vp, p.page_table.cuda(), p.seq_lens.cuda())
    torch.cuda.synchronize()
    assert api.attn_device_status(clear=True) == 0
    table, sl = p.page_table.numpy(), p.seq_lens.numpy()
    want_k = sdpa.append_pages(bits(p.k_pool), table, sl, bits(k_new), page)
    want_v = sdpa.append_pages(bits(p.v_pool), table, sl, bits(v_new), page)
    np.testing.assert_array_equal(bits(kp), want_k)      # NaN slots included: compared as bit patterns
    np.testing.assert_array_equal(bits(vp), want_v)


def test_append_reports_a_bad_page_and_writes_the_rest():
    B, Hkv, D, page = 2, 2, 64, 16
    p = inputs.paged_inputs(B, 1, Hkv, D, page, seed=9, seq_lens=[40, 40])
    table = p.page_table.clone()
    table[0, 1] = p.num_pages + 3                # tokens 16..31 of sequence 0 have no valid page
    k_new = inputs.normal((B, Hkv, 40, D), seed=1)
    kp, vp = p.k_pool.cuda(), p.v_pool.cuda()
    api.attn_device_status(clear=True)
    api.attn_kv_append(k_new.cuda(), k_new.cuda(), kp, vp, table.cuda(), p.seq_lens.cuda())
    torch.cuda.synchronize()
    assert api.attn_device_status(clear=True) == 5
    # sequence 1 and the valid pages of sequence 0 are written exactly
    np.testing.assert_array_equal(bits(kp)[table[1, :3].numpy()],
                                  sdpa.append_pages(bits(p.k_pool), p.page_table.numpy(), [40, 40],
                                                    bits(k_new), page)[table[1, :3].numpy()])
    got0 = bits(kp)[table[0, 0].item()]
    np.testing.assert_array_equal(got0, bits(k_new)[0, :, :16])


class Sequence:
    """Host-side history of one sequence: its tokens' q, k, v (bf16)."""

    def __init__(self, Hq, Hkv, D, seed):
        self.q = torch.empty((Hq, 0, D), dtype=torch.bfloat16)
        self.k = torch.empty((Hkv, 0, D), dtype=torch.bfloat16)
        self.v = torch.empty((Hkv, 0, D), dtype=torch.bfloat16)
        self.seed = seed
        self.step = 0

    def new_tokens(self, n):
        self.step += 1
        base = 1000 * self.seed + 3 * self.step
        q = inputs.normal((self.q.shape[0], n, self.q.shape[2]), base)
        k = inputs.normal((self.k.shape[0], n, self.k.shape[2]), base + 1)
        v = inputs.normal((self.v.shape[0], n, self.v.shape[2]), base + 2)
        self.q, self.k, self.v = torch.cat([self.q, q], 1), torch.cat([self.k, k], 1), torch.cat([self.v, v], 1)
        return q, k, v


def test_serving_loop_with_page_reuse_matches_the_oracle():
    """Admit, prefill in chunks, decode, finish and re-admit through the page pool; every output vs the oracle."""
    Hq, Hkv, D, page = 8, 2, 128, 16
    max_seqs, max_pages, num_pages = 4, 24, 48
    scale = 1 / np.sqrt(D)
    pool = PagePool(num_pages, page, max_seqs, max_pages)
    # the pools start as NaN: only appended tokens may ever be read into an output
    k_pool = torch.full((num_pages, Hkv, page, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    v_pool = torch.full_like(k_pool, float("nan"))
    d_table = torch.empty((max_seqs, max_pages), dtype=torch.int32, device="cuda")
    d_lens = torch.empty((max_seqs,), dtype=torch.int32, device="cuda")
    seqs = {}

    def upload():
        pool.upload(d_table, d_lens)
        table, lens = pool.export()
        torch.cuda.synchronize()
        assert torch.equal(d_table.cpu(), table) and torch.equal(d_lens.cpu(), lens)

    def prefill_chunk(s, n):
        sq = seqs[s]
        q, k, v = sq.new_tokens(n)
        pool.resize(s, pool.seq_len(s) + n)
        upload()
        L = pool.seq_len(s)
        row_t, row_l = d_table[s:s + 1], d_lens[s:s + 1]
        api.attn_kv_append(k[None].cuda(), v[None].cuda(), k_pool, v_pool, row_t, row_l)
        out = api.attn_prefill_paged(q[None].cuda(), k_pool, v_pool, row_t, row_l, max_seq_len=L, causal=True)
        torch.cuda.synchronize()
        assert api.attn_device_status(clear=True) == 0
        ref = sdpa.attention(q[None], sq.k[None], sq.v[None], scale, causal=True)
        assert_parity(out, ref, "bf16", f"prefill chunk of seq {s} ending at {L}")

    def decode_step():
        live = [s for s in range(max_seqs) if s in seqs]
        q_all = torch.zeros((max_seqs, Hq, D), dtype=torch.bfloat16)
        k_all = torch.zeros((max_seqs, Hkv, 1, D), dtype=torch.bfloat16)
        v_all = torch.zeros_like(k_all)
        for s in live:
            q, k, v = seqs[s].new_tokens(1)
            q_all[s], k_all[s, :, 0], v_all[s, :, 0] = q[:, 0], k[:, 0], v[:, 0]
            pool.resize(s, pool.seq_len(s) + 1)
        upload()
        # one batched append and one batched decode over every slot; empty slots append nothing, output 0
        api.attn_kv_append(k_all.cuda(), v_all.cuda(), k_pool, v_pool, d_table, d_lens)
        msl = max(pool.seq_len(s) for s in range(max_seqs))
        out = api.attn_decode_paged(q_all.cuda(), k_pool, v_pool, d_table, d_lens, max_seq_len=msl)
        torch.cuda.synchronize()
        assert api.attn_device_status(clear=True) == 0
        out = out.cpu()
        for s in range(max_seqs):
            if s not in live:
                assert (out[s] == 0).all()
                continue
            sq = seqs[s]
            ref = sdpa.attention(sq.q[None, :, -1:], sq.k[None], sq.v[None], scale, causal=True)[0, :, 0]
            assert_parity(out[s], ref, "bf16", f"decode seq {s} at {pool.seq_len(s)}")

    upload()
    for s, prompt in [(0, 150), (1, 40), (2, 260)]:
        seqs[s] = Sequence(Hq, Hkv, D, seed=s + 1)
        for start in range(0, prompt, 96):
            prefill_chunk(s, min(96, prompt - start))
    for _ in range(3):
        decode_step()
    # sequence 2 finishes; a new one in slot 3 reuses its pages
    freed = set(pool.export()[0][2][:pages_needed(pool.seq_len(2), page)].tolist())
    pool.release(2)
    del seqs[2]
    seqs[3] = Sequence(Hq, Hkv, D, seed=9)
    prefill_chunk(3, 200)
    reused = set(pool.export()[0][3][:pages_needed(200, page)].tolist())
    assert reused & freed
    for _ in range(3):
        decode_step()
    # sequence 1 rolls back 10 tokens (its last page is reclaimed when emptied), then continues
    sq = seqs[1]
    pool.resize(1, pool.seq_len(1) - 10)
    sq.q, sq.k, sq.v = sq.q[:, :-10], sq.k[:, :-10], sq.v[:, :-10]
    decode_step()


def pages_needed(n, page):
    return -(-n // page)
