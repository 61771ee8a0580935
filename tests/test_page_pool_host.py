"""The host-side page pool of the C ABI (attn_page_pool_*): allocation, reclaim and page tables.  CPU only.

The "Attention From Scratch" README ("Paged KV Cache") asks for a global pool
of fixed-size pages, a page table per sequence, and pages allocated as a
sequence grows and reclaimed when it ends; "LLM core technology"
("PagedAttention") lets a sequence's pages sit anywhere in the pool.  These
tests drive the library through long random sequences of requests and check
the pool against a plain model of that bookkeeping after every one.
"""
import numpy as np
import pytest

from scaled_dot_product_prefill_b200 import PagePool
from scaled_dot_product_prefill_b200._lib import AttnError

OUT_OF_PAGES, INVALID = 7, 1


def pages_for(n, page):
    return -(-n // page)


def check_state(pool, model_lens, model_pages):
    table, lens = pool.export()
    table, lens = table.numpy(), lens.numpy()
    held = []
    for s in range(pool.max_seqs):
        n = pages_for(model_lens[s], pool.page_size)
        assert lens[s] == model_lens[s] == pool.seq_len(s)
        row = table[s]
        assert (row[n:] == -1).all()
        assert (row[:n] >= 0).all() and (row[:n] < pool.num_pages).all()
        # pages a sequence keeps never move: the model's prefix is the table's prefix
        assert row[:n].tolist() == model_pages[s]
        held += row[:n].tolist()
    # every page is held by at most one sequence, and the rest are free
    assert len(held) == len(set(held))
    assert pool.free_pages == pool.num_pages - len(held)


def test_fresh_pool_is_empty():
    pool = PagePool(12, 16, 3, 5)
    table, lens = pool.export()
    assert (table == -1).all() and (lens == 0).all()
    assert pool.free_pages == 12


def test_growth_takes_pages_and_release_returns_them_most_recent_first():
    pool = PagePool(10, 16, 3, 4)
    pool.resize(0, 33)                 # 3 pages
    pool.resize(1, 16)                 # 1 page, exactly full
    table, lens = pool.export()
    assert table[0, :3].tolist() == [0, 1, 2] and table[1, 0] == 3
    assert lens.tolist() == [33, 16, 0]
    assert pool.free_pages == 6
    pool.resize(0, 48)                 # same page count: nothing moves
    assert pool.free_pages == 6
    pool.release(0)
    assert pool.free_pages == 9 and pool.seq_len(0) == 0
    pool.resize(2, 17)                 # the page freed last (sequence 0's first) comes back first
    assert pool.export()[0][2, :2].tolist() == [0, 1]


def test_a_request_that_does_not_fit_changes_nothing():
    pool = PagePool(6, 16, 3, 8)
    pool.resize(0, 40)
    pool.resize(1, 20)
    before = [t.clone() for t in pool.export()]
    with pytest.raises(AttnError) as e:
        pool.resize(2, 16 * 3)         # needs 3 pages, 1 left
    assert e.value.status == OUT_OF_PAGES
    after = pool.export()
    assert all((a == b).all() for a, b in zip(before, after))
    assert pool.free_pages == 1
    pool.resize(2, 16)                 # 1 page still fits
    assert pool.free_pages == 0


def test_pages_of_a_sequence_need_not_be_contiguous():
    """Finished sequences leave holes; a new long sequence is built from them (PagedAttention)."""
    pool = PagePool(16, 16, 16, 16)
    for s in range(16):
        pool.resize(s, 16)             # one page each: page s
    for s in range(0, 16, 2):
        pool.release(s)                # free every other page
    pool.resize(0, 8 * 16)             # all 8 scattered free pages
    row = pool.export()[0][0, :8].tolist()
    assert sorted(row) == list(range(0, 16, 2))
    assert pool.free_pages == 0


@pytest.mark.parametrize("bad", [dict(num_pages=0), dict(page_size=0), dict(max_seqs=-1),
                                 dict(max_pages_per_seq=0)])
def test_create_rejects_bad_sizes(bad):
    kw = dict(num_pages=4, page_size=16, max_seqs=2, max_pages_per_seq=2)
    kw.update(bad)
    with pytest.raises(AttnError) as e:
        PagePool(**kw)
    assert e.value.status == INVALID


def test_resize_rejects_bad_arguments():
    pool = PagePool(8, 16, 2, 3)
    for seq, n in [(-1, 1), (2, 1), (0, -5), (0, 3 * 16 + 1)]:
        with pytest.raises(AttnError) as e:
            pool.resize(seq, n)
        assert e.value.status == INVALID
    pool.resize(0, 3 * 16)             # the largest length that fits the table row


def test_null_pool_is_rejected_by_the_c_functions():
    from scaled_dot_product_prefill_b200 import _lib

    lib = _lib.load()
    assert lib.attn_page_pool_free_pages(None) == -1
    assert lib.attn_page_pool_seq_len(None, 0) == -1
    assert lib.attn_page_pool_resize(None, 0, 1) == INVALID
    assert lib.attn_page_pool_export(None, None, None) == INVALID
    assert lib.attn_page_pool_upload(None, None, None, None) == INVALID
    assert lib.attn_page_pool_create(4, 16, 1, 1, None) == INVALID
    lib.attn_page_pool_destroy(None)   # a no-op


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_random_requests_keep_the_bookkeeping_consistent(seed):
    """Grow, shrink and release at random (a serving loop's admissions, decode steps and finishes)."""
    rng = np.random.default_rng(seed)
    num_pages, page, seqs, max_pages = 64, 16, 8, 20
    pool = PagePool(num_pages, page, seqs, max_pages)
    lens = [0] * seqs
    pages = [[] for _ in range(seqs)]
    free = list(range(num_pages - 1, -1, -1))      # the model's free stack
    refused = 0
    for _ in range(400):
        s = int(rng.integers(seqs))
        op = rng.random()
        if op < 0.15:
            n = 0                                   # the sequence finishes
        elif op < 0.25:
            n = int(rng.integers(0, lens[s] + 1))   # roll back some tokens
        elif op < 0.75:
            n = min(lens[s] + 1, max_pages * page)  # one decode step
        else:
            n = min(lens[s] + int(rng.integers(1, 200)), max_pages * page)   # a prefill chunk
        want = pages_for(n, page)
        if want - len(pages[s]) > len(free):
            with pytest.raises(AttnError) as e:
                pool.resize(s, n)
            assert e.value.status == OUT_OF_PAGES
            refused += 1
        else:
            pool.resize(s, n)
            while len(pages[s]) < want:
                pages[s].append(free.pop())
            while len(pages[s]) > want:
                free.append(pages[s].pop())
            lens[s] = n
        check_state(pool, lens, pages)
    assert refused > 0                             # the pool ran full at some point
