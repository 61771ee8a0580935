"""Pins for the float64 oracle: closed forms, invariants and the pages' printed values.

Each test fixes the oracle to something other than itself, so that a
dropped term, a wrong sign or index, or a transposed operand in
``oracle/`` fails at least one of them.  CPU only.
"""
import math

import numpy as np
import pytest

from conftest import read_golden
from oracle import brute, sdpa
from scaled_dot_product_prefill_b200 import inputs, workloads

RNG = np.random.default_rng(12345)


def rand(*shape):
    return RNG.standard_normal(shape)


# --------------------------------------------------------------------------
# independent brute force on tiny shapes


TINY = [
    # B, Hq, Hkv, Sq, Skv, D
    (1, 1, 1, 5, 5, 4),
    (2, 4, 2, 7, 7, 8),
    (1, 4, 1, 6, 9, 3),     # Sq < Skv: bottom-right causal alignment
    (1, 2, 2, 8, 5, 4),     # Sq > Skv: leading rows see nothing under causal
    (1, 4, 4, 3, 1, 5),     # a single key
]


@pytest.mark.parametrize("shape", TINY)
@pytest.mark.parametrize("causal,window", [(False, 0), (True, 0), (True, 1), (True, 3)])
def test_numpy_oracle_matches_brute_force(shape, causal, window):
    B, Hq, Hkv, Sq, Skv, D = shape
    q, k, v = rand(B, Hq, Sq, D), rand(B, Hkv, Skv, D), rand(B, Hkv, Skv, D)
    scale = 0.37
    got = sdpa.attention(q, k, v, scale, causal, window)
    ref = np.array(brute.attention(q, k, v, scale, causal, window))
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def test_paged_decode_matches_brute_force():
    p = inputs.paged_inputs(3, 4, 2, 8, page_size=4, seed=7, seq_lens=[5, 1, 11], spare_pages=2,
                            dtype="f32")
    for window in (0, 3):
        got = sdpa.decode_paged(p.q, p.k_pool, p.v_pool, p.page_table, p.seq_lens, 4, 0.3, window)
        ref = np.array(brute.decode_paged(p.q, p.k_pool, p.v_pool, p.page_table, p.seq_lens, 4, 0.3,
                                          window))
        np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


# --------------------------------------------------------------------------
# softmax and masking, as the pages state them


def test_weights_rows_sum_to_one_and_causal_upper_triangle_is_zero():
    q, k = rand(9, 6), rand(9, 6)
    P, _ = sdpa.weights(q, k, 0.5, causal=True)
    np.testing.assert_allclose(P.sum(-1), 1.0, rtol=0, atol=1e-14)
    assert np.all(P[np.triu_indices(9, 1)] == 0.0)          # exactly zero, not small
    assert np.all(P[np.tril_indices(9)] > 0.0)
    np.testing.assert_array_equal(P[0], np.eye(9)[0])          # first row attends only to itself


def test_printed_6x6_causal_matrix_structure():
    """The page's 6x6 causal weights: lower triangular, first row e0, rows sum to 1 (2-decimal print)."""
    M = np.array([[float(x) for x in r] for r in read_golden("anat_causal_weights_6x6.txt")])
    assert M.shape == (6, 6)
    assert np.all(M[np.triu_indices(6, 1)] == 0.0)
    np.testing.assert_array_equal(M[0], np.eye(6)[0])
    np.testing.assert_allclose(M.sum(-1), 1.0, atol=6 * 0.005)
    # the oracle's causal weights on 6 tokens have the same zero pattern and exact row sums
    P, _ = sdpa.weights(rand(6, 16), rand(6, 16), 0.25, causal=True)
    np.testing.assert_array_equal(P == 0.0, M == 0.0)
    np.testing.assert_allclose(P.sum(-1), 1.0, atol=1e-14)


def test_stable_softmax_survives_large_logits():
    """exp(800) overflows; the max-subtracted form returns [1, e^-800] without NaN."""
    P, lse = sdpa.softmax_rows(np.array([[800.0, 0.0], [-np.inf, 3.0]]))
    assert np.all(np.isfinite(P))
    np.testing.assert_allclose(P[0], [1.0, math.exp(-800.0)], rtol=0, atol=1e-300)
    np.testing.assert_array_equal(P[1], [0.0, 1.0])
    assert lse[0] == pytest.approx(800.0)
    assert lse[1] == pytest.approx(3.0)


def test_masked_logit_gets_exactly_zero_weight_even_when_logit_would_be_zero():
    """A mask must put -inf on the logit; a visible logit of 0 still gets positive weight."""
    q = np.zeros((2, 4))
    k = rand(2, 4)
    P, _ = sdpa.weights(q, k, 1.0, causal=True)      # all logits 0; row 0 sees only key 0
    np.testing.assert_array_equal(P, [[1.0, 0.0], [0.5, 0.5]])


def test_fully_masked_rows_give_zero_output():
    q, k, v = rand(1, 1, 6, 4), rand(1, 1, 3, 4), rand(1, 1, 3, 4)
    out, lse = sdpa.attention(q, k, v, 0.5, causal=True, return_lse=True)
    # Sq=6 > Skv=3, bottom-right: rows 0..2 have i + (3 - 6) < 0, no visible key
    np.testing.assert_array_equal(out[0, 0, :3], 0.0)
    assert np.all(np.isneginf(lse[0, 0, :3]))
    assert np.all(np.isfinite(out[0, 0, 3:]))


# --------------------------------------------------------------------------
# closed forms


def test_identical_keys_give_mean_of_values():
    kvec = rand(1, 8)
    k = np.repeat(kvec, 10, axis=0)[None, None]
    v = rand(1, 1, 10, 8)
    q = rand(1, 1, 4, 8)
    out = sdpa.attention(q, k, v, 0.9, causal=False)
    np.testing.assert_allclose(out[0, 0], np.broadcast_to(v[0, 0].mean(0), (4, 8)), atol=1e-14)


def test_single_key_returns_its_value():
    q, k, v = rand(2, 3, 5, 8), rand(2, 3, 1, 8), rand(2, 3, 1, 8)
    out = sdpa.attention(q, k, v, 1.3, causal=False)
    np.testing.assert_allclose(out, np.broadcast_to(v, out.shape), atol=1e-15)


def test_zero_scale_gives_mean_of_visible_values():
    q, k, v = rand(1, 1, 7, 4), rand(1, 1, 7, 4), rand(1, 1, 7, 4)
    out = sdpa.attention(q, k, v, 0.0, causal=True, window=3)
    for i in range(7):
        lo = max(0, i - 2)
        np.testing.assert_allclose(out[0, 0, i], v[0, 0, lo:i + 1].mean(0), atol=1e-14)


def test_first_causal_row_is_first_value():
    q, k, v = rand(2, 2, 5, 8), rand(2, 2, 5, 8), rand(2, 2, 5, 8)
    out = sdpa.attention(q, k, v, 0.35, causal=True)
    np.testing.assert_allclose(out[:, :, 0], v[:, :, 0], atol=1e-15)


def test_window_one_returns_own_value_and_wide_window_is_causal():
    q, k, v = rand(1, 2, 9, 4), rand(1, 2, 9, 4), rand(1, 2, 9, 4)
    np.testing.assert_allclose(sdpa.attention(q, k, v, 0.5, True, 1), v, atol=1e-15)
    np.testing.assert_allclose(sdpa.attention(q, k, v, 0.5, True, 9),
                               sdpa.attention(q, k, v, 0.5, True, 0), atol=1e-15)
    np.testing.assert_allclose(sdpa.attention(q, k, v, 0.5, True, 50),
                               sdpa.attention(q, k, v, 0.5, True, 0), atol=1e-15)


def test_window_rows_see_exactly_w_keys():
    vis = sdpa.visible(20, 20, True, 4)
    counts = vis.sum(-1)
    np.testing.assert_array_equal(counts, np.minimum(np.arange(20) + 1, 4))
    for i in range(20):  # the W visible keys are the query itself and the W-1 before it
        np.testing.assert_array_equal(np.nonzero(vis[i])[0], np.arange(max(0, i - 3), i + 1))


# --------------------------------------------------------------------------
# invariants


def test_shift_invariance_with_large_shift():
    """K' = K + 1 u^T adds the row constant q_i.u*scale to every logit of row i."""
    q, k, v = rand(1, 2, 6, 8), rand(1, 2, 6, 8), rand(1, 2, 6, 8)
    u = 400.0 * np.sign(rand(8))
    base = sdpa.attention(q, k, v, 0.5, causal=True)
    shifted = sdpa.attention(q, k + u, v, 0.5, causal=True)
    assert np.all(np.isfinite(shifted))
    np.testing.assert_allclose(shifted, base, atol=1e-9)


def test_gqa_with_equal_heads_is_mha_and_matches_repeat_interleave():
    B, Hq, S, D = 2, 8, 7, 4
    q = rand(B, Hq, S, D)
    for Hkv in (8, 4, 2, 1):
        k, v = rand(B, Hkv, S, D), rand(B, Hkv, S, D)
        rep = Hq // Hkv
        kr, vr = np.repeat(k, rep, axis=1), np.repeat(v, rep, axis=1)   # repeat_interleave order
        np.testing.assert_allclose(sdpa.attention(q, k, v, 0.5, True),
                                   sdpa.attention(q, kr, vr, 0.5, True), atol=1e-15)
    # MQA: one kv head is the same as MHA with that head copied to every query head
    k1, v1 = rand(B, 1, S, D), rand(B, 1, S, D)
    np.testing.assert_allclose(sdpa.attention(q, k1, v1, 0.5, False),
                               sdpa.attention(q, np.tile(k1, (1, Hq, 1, 1)),
                                              np.tile(v1, (1, Hq, 1, 1)), 0.5, False), atol=1e-15)
    # the map is contiguous groups (h // rep), not round robin (h % Hkv)
    assert [sdpa.kv_head(h, 8, 2) for h in range(8)] == [0, 0, 0, 0, 1, 1, 1, 1]


def test_attention_rows_match_full_output():
    q, k, v = rand(1, 1, 40, 8), rand(1, 1, 40, 8), rand(1, 1, 40, 8)
    full = sdpa.attention(q, k, v, 0.4, True, 9)
    rows = [0, 5, 8, 9, 39]
    got = sdpa.attention_rows(q[0, 0, rows], k[0, 0], v[0, 0], rows, 40, 0.4, True, 9)
    np.testing.assert_allclose(got, full[0, 0, rows], atol=1e-14)


def test_paged_equals_contiguous_and_ignores_page_order_and_poison():
    p = inputs.paged_inputs(4, 8, 2, 16, page_size=4, seed=3, seq_lens=[1, 4, 9, 17], spare_pages=5,
                            poison=True, dtype="f32")
    out = sdpa.decode_paged(p.q, p.k_pool, p.v_pool, p.page_table, p.seq_lens, 4, 0.25)
    assert np.all(np.isfinite(out))
    q64 = p.q.double().numpy()
    for b, L in enumerate(p.seq_lens.tolist()):
        K = sdpa.gather_pages(p.k_pool, p.page_table[b].numpy(), L, 4)     # [L, Hkv, D]
        V = sdpa.gather_pages(p.v_pool, p.page_table[b].numpy(), L, 4)
        kc = K.transpose(1, 0, 2)[None]
        vc = V.transpose(1, 0, 2)[None]
        ref = sdpa.attention(q64[b][None, :, None, :], kc, vc, 0.25, causal=True)[0, :, 0]
        np.testing.assert_allclose(out[b], ref, atol=1e-14)
    # moving the pages to other physical slots (and the table with them) changes nothing
    perm = np.random.default_rng(1).permutation(p.num_pages)
    inv = np.argsort(perm)
    k2, v2 = p.k_pool.numpy()[perm], p.v_pool.numpy()[perm]
    t2 = np.where(p.page_table.numpy() >= 0, inv[np.maximum(p.page_table.numpy(), 0)], -1)
    out2 = sdpa.decode_paged(p.q, k2, v2, t2, p.seq_lens, 4, 0.25)
    np.testing.assert_allclose(out2, out, atol=0)


def test_incremental_kv_cache_decode_equals_full_recompute():
    """Decoding token by token against a growing cache equals causal attention over the sequence."""
    S, H, D = 12, 2, 8
    q, k, v = rand(1, H, S, D), rand(1, H, S, D), rand(1, H, S, D)
    full = sdpa.attention(q, k, v, 0.3, causal=True)
    page = 4
    npg = (S + page - 1) // page
    k_pool = np.zeros((npg, H, page, D))
    v_pool = np.zeros((npg, H, page, D))
    table = np.arange(npg)[::-1].copy()[None]     # pages stored in reverse order
    for t in range(S):
        k_pool[table[0, t // page], :, t % page] = k[0, :, t]
        v_pool[table[0, t // page], :, t % page] = v[0, :, t]
        step = sdpa.decode_paged(q[0, :, t][None], k_pool, v_pool, table, [t + 1], page, 0.3)
        np.testing.assert_allclose(step[0], full[0, :, t], atol=1e-14)


def test_decode_with_window_equals_last_windowed_prefill_row():
    S, H, D, W = 13, 2, 8, 5
    q, k, v = rand(1, H, S, D), rand(1, H, S, D), rand(1, H, S, D)
    full = sdpa.attention(q, k, v, 0.3, causal=True, window=W)
    k_pool = k[0].transpose(1, 0, 2)[:, :, None, :].copy()     # page size 1: [S, H, 1, D]
    v_pool = v[0].transpose(1, 0, 2)[:, :, None, :].copy()
    out = sdpa.decode_paged(q[0, :, S - 1][None], k_pool, v_pool, np.arange(S)[None], [S], 1, 0.3, W)
    np.testing.assert_allclose(out[0], full[0, :, S - 1], atol=1e-14)


# --------------------------------------------------------------------------
# the pages' printed numbers


def test_scale_table_statistics():
    """Variance, entropy and max-probability of softmax over 64 N(0,1) keys, raw vs 1/sqrt(d).

    The page's random stream is unknown, so the check is statistical: our
    estimate over 2048 repeats against its printed 256-repeat means, within
    about three standard errors of the page's own estimate.
    """
    rng = np.random.default_rng(2024)
    for row in read_golden("anat_scale_table.txt"):
        d = int(row[0])
        var_raw, var_sc, h_raw, h_sc, mp_raw, mp_sc = map(float, row[1:])
        reps = 2048
        q = rng.standard_normal((reps, d))
        k = rng.standard_normal((reps, 64, d))
        stats = {}
        for name, scale in (("raw", 1.0), ("scaled", 1.0 / math.sqrt(d))):
            P = np.stack([sdpa.weights(q[r:r + 1], k[r], scale, causal=False)[0][0] for r in range(reps)])
            logits = np.einsum("rd,rkd->rk", q, k) * scale
            H = -np.sum(np.where(P > 0, P * np.log(np.where(P > 0, P, 1.0)), 0.0), axis=-1).mean()
            stats[name] = (logits.var(), H, P.max(-1).mean())
        assert stats["raw"][0] == pytest.approx(var_raw, rel=0.06)
        assert stats["scaled"][0] == pytest.approx(var_sc, abs=0.05)
        assert stats["scaled"][1] == pytest.approx(h_sc, abs=0.03)
        assert stats["scaled"][2] == pytest.approx(mp_sc, abs=0.008)
        assert stats["raw"][1] == pytest.approx(h_raw, rel=0.25)
        assert stats["raw"][2] == pytest.approx(mp_raw, abs=0.03)
        assert abs(stats["scaled"][1] - math.log(64)) < 0.6        # near uniform, unlike raw at large d


def test_flop_accounting_matches_the_kv_cache_flop_table():
    """The page's last-step FLOPs are projections plus 4 * n_q * n_k * D for attention."""
    D = 64
    for n, no_cache, cache in read_golden("anat_kv_cache_flops.txt"):
        n, no_cache, cache = int(n), int(no_cache), int(cache)
        full_attn = workloads.attention_flops(1, 1, n, n, D, causal=False)
        assert 6 * n * D * D + full_attn + 2 * D * D == no_cache
        one_query = workloads.attention_flops(1, 1, 1, n, D, causal=False)
        assert one_query + 8 * D * D == cache


def test_kv_byte_accounting_matches_the_kv_cache_byte_tables():
    rows = read_golden("anat_kv_cache_bytes.txt")
    for r in rows:
        if r[0].isdigit():
            n, nbytes = int(r[0]), int(r[1])
            assert workloads.kv_bytes([n], Hkv=1, D=64, elem_bytes=4) == nbytes
        else:
            _, heads, kb = r
            per_layer = workloads.kv_bytes([1], Hkv=int(heads), D=128, elem_bytes=2)
            assert 32 * per_layer == int(kb) * 1024


def test_visible_pair_counts_match_the_oracle_predicate():
    for Sq, Skv, causal, W in [(17, 17, True, 0), (17, 17, False, 0), (33, 33, True, 5),
                               (5, 12, True, 0), (12, 5, True, 0), (12, 5, True, 2), (1, 40, True, 7)]:
        assert workloads.visible_pairs(Sq, Skv, causal, W) == int(sdpa.visible(Sq, Skv, causal, W).sum())
    # the sliding-window workload: min(i + 1, 4096) keys per query over 16384 queries
    assert workloads.visible_pairs(16384, 16384, True, 4096) == 58_722_304
    assert workloads.prefill_flops(workloads.WORKLOADS["gqa_swa_16k"]) == 4 * 128 * 32 * 58_722_304
    # the chunked prefill: query i of the last 1024 of 4096 tokens sees 3072 + i + 1 keys
    spec = workloads.EXTRA_WORKLOADS["chunked_prefill_paged_gqa"]
    pairs = 1024 * 3072 + 1024 * 1025 // 2
    assert workloads.visible_pairs(1024, 4096, True, 0) == pairs
    assert workloads.paged_prefill_flops(spec) == 4 * 128 * 4 * 32 * pairs


def test_lse_matches_python_log_sum_exp_and_merges_disjoint_key_sets():
    """lse_i = log sum_j exp(s_ij) over visible keys (math.fsum in pure Python), -inf when none is visible;
    merging two disjoint key sets by their lse reproduces attention over their union."""
    q, k, v = rand(1, 2, 7, 4), rand(1, 2, 9, 4), rand(1, 2, 9, 4)
    for causal, window in ((False, 0), (True, 0), (True, 3)):
        _, lse = sdpa.attention(q, k, v, 0.6, causal, window, return_lse=True)
        vis = sdpa.visible(7, 9, causal, window)
        for h in range(2):
            for i in range(7):
                s = [0.6 * sum(q[0, h, i, d] * k[0, h, j, d] for d in range(4)) for j in range(9) if vis[i, j]]
                want = math.log(math.fsum(math.exp(x) for x in s)) if s else -math.inf
                assert lse[0, h, i] == pytest.approx(want, abs=1e-12)
    o1, l1 = sdpa.attention(q, k[:, :, :4], v[:, :, :4], 0.6, False, return_lse=True)
    o2, l2 = sdpa.attention(q, k[:, :, 4:], v[:, :, 4:], 0.6, False, return_lse=True)
    full, lf = sdpa.attention(q, k, v, 0.6, False, return_lse=True)
    w1, w2 = np.exp(l1 - lf)[..., None], np.exp(l2 - lf)[..., None]
    np.testing.assert_allclose(w1 * o1 + w2 * o2, full, atol=1e-13)
    np.testing.assert_allclose(np.logaddexp(l1, l2), lf, atol=1e-13)


# --------------------------------------------------------------------------
# appending to the paged cache


def _random_table(rng, B, max_pages, num_pages):
    perm = rng.permutation(num_pages)[:B * max_pages]
    return perm.reshape(B, max_pages).astype(np.int64)


def test_append_then_gather_returns_the_appended_tokens():
    """Chunks appended one after another read back, through the page table, as their concatenation."""
    rng = np.random.default_rng(7)
    B, Hkv, D, page = 3, 2, 4, 4
    table = _random_table(rng, B, 6, 30)           # non-contiguous, shuffled pages
    pool = np.full((30, Hkv, page, D), np.nan)
    written = [[] for _ in range(B)]
    lens = np.zeros(B, dtype=np.int64)
    for S_new in (5, 1, 1, 3, 7):                  # a prefill chunk, decode steps, more chunks
        new = rng.standard_normal((B, Hkv, S_new, D))
        lens = lens + S_new
        pool = sdpa.append_pages(pool, table, lens, new, page)
        for b in range(B):
            written[b].append(new[b].transpose(1, 0, 2))        # [S_new, Hkv, D]
    for b in range(B):
        want = np.concatenate(written[b])
        got = sdpa.gather_pages(pool, table[b], int(lens[b]), page)
        np.testing.assert_array_equal(got, want)
    # nothing else was written: exactly the appended slots lost their NaN
    assert np.count_nonzero(~np.isnan(pool)) == int(lens.sum()) * Hkv * D


def test_append_of_a_chunk_longer_than_the_cache_keeps_only_its_last_tokens():
    B, Hkv, D, page = 2, 1, 2, 4
    table = np.array([[3, 1], [0, 2]])
    pool = np.full((4, Hkv, page, D), np.nan)
    new = np.arange(B * Hkv * 5 * D, dtype=np.float64).reshape(B, Hkv, 5, D)
    out = sdpa.append_pages(pool, table, [2, 5], new, page)
    # sequence 0 holds 2 tokens: the chunk's tokens 3 and 4 at positions 0 and 1
    np.testing.assert_array_equal(out[3, 0, :2], new[0, 0, 3:])
    assert np.isnan(out[3, 0, 2:]).all() and np.isnan(out[1]).all()
    np.testing.assert_array_equal(sdpa.gather_pages(out, table[1], 5, page), new[1].transpose(1, 0, 2))


def test_append_then_decode_equals_full_causal_recompute():
    """Prefill a prompt into the cache, then decode token by token: each step equals the causal row."""
    S, P, H, D, page = 11, 4, 2, 8, 4
    q, k, v = rand(1, H, S, D), rand(1, H, S, D), rand(1, H, S, D)
    full = sdpa.attention(q, k, v, 0.3, causal=True)
    table = np.array([[5, 0, 3]])
    k_pool = np.full((6, H, page, D), np.nan)
    v_pool = np.full((6, H, page, D), np.nan)
    k_pool = sdpa.append_pages(k_pool, table, [P], k[:, :, :P], page)
    v_pool = sdpa.append_pages(v_pool, table, [P], v[:, :, :P], page)
    for t in range(P, S):
        k_pool = sdpa.append_pages(k_pool, table, [t + 1], k[:, :, t:t + 1], page)
        v_pool = sdpa.append_pages(v_pool, table, [t + 1], v[:, :, t:t + 1], page)
        step = sdpa.decode_paged(q[0, :, t][None], k_pool, v_pool, table, [t + 1], page, 0.3)
        np.testing.assert_allclose(step[0], full[0, :, t], atol=1e-14)


# --------------------------------------------------------------------------
# 8-bit codes of the fp8 cache


def test_e4m3_values_at_the_format_landmarks():
    from oracle import fp8

    v = fp8.e4m3_value(np.array([0x00, 0x80, 0x01, 0x07, 0x08, 0x38, 0xB8, 0x3C, 0x7E, 0xFE, 0x7F, 0xFF], np.uint8))
    want = [0.0, -0.0, 2.0 ** -9, 7 * 2.0 ** -9, 2.0 ** -6, 1.0, -1.0, 1.5, 448.0, -448.0]
    np.testing.assert_array_equal(v[:10], want)
    assert np.signbit(v[1])
    assert np.isnan(v[10]) and np.isnan(v[11])
    # the positive finite codes are strictly increasing; the step up from code c is one ulp of
    # c's binade, 2^(max(e, 1) - 10) for exponent field e (subnormals share the first binade's ulp)
    pos = fp8.e4m3_value(np.arange(0x7F, dtype=np.uint8))
    steps = np.diff(pos)
    assert (steps > 0).all()
    e = np.maximum(np.arange(0, 0x7E) >> 3, 1)
    np.testing.assert_array_equal(steps, 2.0 ** (e - 10.0))


def test_e4m3_values_match_torch_float8_for_every_code():
    import torch

    from oracle import fp8

    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = fp8.e4m3_value(codes)
    np.testing.assert_array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    np.testing.assert_array_equal(got[ok], ref[ok])


def test_e4m3_rounding_round_trips_ties_to_even_and_saturates():
    from oracle import fp8

    codes = np.arange(256, dtype=np.uint8)
    codes = codes[(codes & 0x7F) != 0x7F]
    np.testing.assert_array_equal(fp8.e4m3_round(fp8.e4m3_value(codes)), codes)
    pos = fp8.e4m3_value(np.arange(0x7F, dtype=np.uint8))
    mid = (pos[:-1] + pos[1:]) / 2                       # exact halfway points (in float64)
    got = fp8.e4m3_round(mid)
    lower = np.arange(0x7E)
    np.testing.assert_array_equal(got, np.where(lower % 2 == 0, lower, lower + 1))
    eps = np.diff(pos) / 8
    np.testing.assert_array_equal(fp8.e4m3_round(mid - eps), lower)
    np.testing.assert_array_equal(fp8.e4m3_round(mid + eps), lower + 1)
    np.testing.assert_array_equal(fp8.e4m3_round([448.0, 449.0, 1e30, -1e30, -0.0, -1e-9]),
                                  [0x7E, 0x7E, 0x7E, 0xFE, 0x80, 0x80])


def test_e4m3_rounding_matches_torch_float8_in_range():
    import torch

    from oracle import fp8

    x = np.float32(np.random.default_rng(3).standard_normal(200000) * 60)
    x = x[np.abs(x) <= 448]
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(fp8.e4m3_round(x), want)
